"""CPU tests of the C-ABI library: it loads without a GPU, exports every symbol
include/hstu.h declares, builds the same time-bucket thresholds as the oracle,
and rejects bad arguments synchronously, before anything is enqueued.

The rejection cases pass placeholder device addresses; every case violates one
rule, so the library returns before it touches them (no CUDA call is made).
"""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from pointwise_attention_b200 import build
    build.build()
    import pointwise_attention_b200 as pa
    return pa


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "hstu.h")).read()
    return sorted(set(re.findall(r"HSTU_API\s+[\w\s\*]*?\b(hstu_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 7
    so = lib.load_library()
    for n in names:
        assert hasattr(so, n), n
    assert set(names) == set(lib.EXPORTED)


def test_thresholds_match_oracle_golden(lib):
    rows = [l.split() for l in open(os.path.join(ROOT, "tests", "golden",
                                                 "time_bucket_thresholds.txt"))
            if not l.startswith("#")]
    golden = np.array([int(r[1]) for r in rows], dtype=np.int64)
    got = lib.hstu_time_bucket_thresholds(128)
    assert np.array_equal(got, golden)
    # a capped table keeps the first NB-1 thresholds
    assert np.array_equal(lib.hstu_time_bucket_thresholds(10), golden[:9])
    with pytest.raises(lib.HSTUError):
        lib.hstu_time_bucket_thresholds(129)


def test_status_strings(lib):
    for code in range(7):
        assert lib.status_string(code).startswith("HSTU_")
    assert "unknown" in lib.status_string(99)


FAKE = 0x7F0000000000   # placeholder device address, 256-byte aligned; never dereferenced


def problem(lib, **kw):
    p = lib.hstu_problem_t()
    host_off = kw.pop("offsets_host", None)
    p.dtype = kw.pop("dtype", 1)
    p.batch = kw.pop("batch", 2)
    p.total_tokens = kw.pop("total_tokens", 300)
    p.max_seq_len = kw.pop("max_seq_len", 200)
    p.num_heads = kw.pop("num_heads", 4)
    p.d_qk = kw.pop("d_qk", 128)
    p.d_v = kw.pop("d_v", 128)
    p.offsets = kw.pop("offsets", FAKE)
    p.timestamps = kw.pop("timestamps", None)
    p.rab_pos = kw.pop("rab_pos", None)
    p.rab_pos_len = kw.pop("rab_pos_len", 0)
    p.rab_time = kw.pop("rab_time", None)
    p.num_time_buckets = kw.pop("num_time_buckets", 0)
    p.norm_len = kw.pop("norm_len", 0)
    p.ln_eps = kw.pop("ln_eps", 1e-5)
    assert not kw, kw
    keep = None
    if host_off is not None:
        keep = (ctypes.c_int32 * len(host_off))(*host_off)
        p.offsets_host = ctypes.cast(keep, ctypes.c_void_p).value
    return p, keep


def call_fwd(lib, p, ws_bytes=None, ws=FAKE, q=FAKE, save=(None, None, None), y=FAKE):
    so = lib.load_library()
    if ws_bytes is None:
        ws_bytes = 1 << 20
    vp = ctypes.c_void_p
    return so.hstu_attn_fwd(ctypes.byref(p), vp(q), vp(FAKE), vp(FAKE), vp(FAKE), vp(y),
                            *(vp(x) if x else None for x in save), vp(ws) if ws else None,
                            ws_bytes, None)


@pytest.mark.parametrize("field,value", [
    ("dtype", 7), ("num_heads", 0), ("d_qk", 0), ("batch", -1), ("ln_eps", 0.0),
    ("ln_eps", float("nan")), ("norm_len", -3), ("offsets", None), ("max_seq_len", -1),
])
def test_fwd_rejects_bad_problem(lib, field, value):
    p, keep = problem(lib, **{field: value})
    assert call_fwd(lib, p) == 1


@pytest.mark.parametrize("host", [
    [0, 200, 100],          # decreasing
    [1, 100, 300],          # offsets[0] != 0
    [0, 100, 299],          # offsets[B] != T
    [0, 50, 300],           # a length above max_seq_len
])
def test_fwd_rejects_bad_host_offsets(lib, host):
    p, keep = problem(lib, offsets_host=host)
    assert call_fwd(lib, p) == 1


def test_fwd_rejects_bias_shapes(lib):
    p, _ = problem(lib, rab_pos=FAKE, rab_pos_len=100)        # L < max_seq_len
    assert call_fwd(lib, p) == 1
    p, _ = problem(lib, rab_pos=FAKE, rab_pos_len=200, max_seq_len=200,
                   offsets_host=[0, 99, 300])                   # n_b = 201 > max_seq_len
    assert call_fwd(lib, p) == 1
    p, _ = problem(lib, rab_time=FAKE, num_time_buckets=128)  # no timestamps
    assert call_fwd(lib, p) == 1
    p, _ = problem(lib, rab_time=FAKE, timestamps=FAKE, num_time_buckets=129)
    assert call_fwd(lib, p) == 1


def test_fwd_rejects_pointers(lib):
    p, _ = problem(lib)
    assert call_fwd(lib, p, q=None) == 1
    assert call_fwd(lib, p, q=FAKE + 8) == 1                  # not 16-byte aligned
    assert call_fwd(lib, p, y=FAKE + 2) == 1
    assert call_fwd(lib, p, save=(FAKE, None, None)) == 1     # all three saved outputs or none


@pytest.mark.parametrize("kw", [
    dict(d_qk=64, d_v=64), dict(num_heads=9), dict(dtype=0, d_qk=256), dict(dtype=0, d_v=200),
    dict(dtype=0, num_heads=16, d_v=128),
])
def test_fwd_unsupported(lib, kw):
    p, _ = problem(lib, **kw)
    assert call_fwd(lib, p) == 2


def test_fwd_workspace(lib):
    p, _ = problem(lib)
    need = lib.hstu_attn_workspace_size(p, False)
    assert need >= 256 and need % 256 == 0
    assert call_fwd(lib, p, ws=None) == 5
    assert call_fwd(lib, p, ws_bytes=need - 1) == 5
    assert call_fwd(lib, p, ws=FAKE + 16) == 5


def test_bwd_workspace_size_and_rejections(lib):
    p, _ = problem(lib, total_tokens=300)
    need = lib.hstu_attn_workspace_size(p, True)
    # status word + dO (bf16, T*H*dv)
    assert need >= 256 + 300 * 4 * 128 * 2
    so = lib.load_library()
    vp = ctypes.c_void_p
    args = [vp(FAKE)] * 12
    # d_rab_pos requested without a position table
    rc = so.hstu_attn_bwd(ctypes.byref(p), *args, vp(FAKE), None, None, None, vp(FAKE),
                          need, None)
    assert rc == 1
    # missing saved statistics
    a2 = list(args)
    a2[6] = None
    rc = so.hstu_attn_bwd(ctypes.byref(p), *a2, None, None, None, None, vp(FAKE), need, None)
    assert rc == 1
    rc = so.hstu_attn_bwd(ctypes.byref(p), *args, None, None, None, None, vp(FAKE), need - 256,
                          None)
    assert rc == 5


def test_check_and_selftest_reject_missing_workspace(lib):
    so = lib.load_library()
    assert so.hstu_attn_check(None, None) == 5
    assert so.hstu_selftest_wait_timeout(None, 1000, None) == 5
    assert so.hstu_selftest_wait_timeout(ctypes.c_void_p(FAKE), 0, None) == 1


def test_empty_problem_is_a_no_op(lib):
    p, _ = problem(lib, batch=0, total_tokens=0, max_seq_len=0, offsets=None)
    assert call_fwd(lib, p) == 0


def test_bwd_rejects_grids_beyond_32_bits(lib):
    """The backward launches one CTA per (head, sequence, 128-row tile) and the
    forward numbers (sequence, tile, head) slots in 32 bits with room for twice
    their count: problems past that bound are refused before anything is
    enqueued."""
    so = lib.load_library()
    vp = ctypes.c_void_p
    args = [vp(FAKE)] * 12
    # 8 heads x 2^20 sequences x 256 tiles = 2^31 CTAs
    p, _ = problem(lib, batch=1 << 20, total_tokens=1 << 20, max_seq_len=256 * 128,
                   num_heads=8)
    assert so.hstu_attn_bwd(ctypes.byref(p), *args, None, None, None, None, vp(FAKE), 1 << 40,
                            None) == 2
    assert call_fwd(lib, p) == 2
    # 8 x 2^20 x 128 = 2^30 slots: twice that passes the 2^31 - 256 bound no more
    p, _ = problem(lib, batch=1 << 20, total_tokens=1 << 20, max_seq_len=128 * 128,
                   num_heads=8)
    assert so.hstu_attn_bwd(ctypes.byref(p), *args, None, None, None, None, vp(FAKE), 0, None) == 2
    # 127 tiles per sequence fit: the call gets as far as the workspace check
    p, _ = problem(lib, batch=1 << 20, total_tokens=1 << 20, max_seq_len=127 * 128,
                   num_heads=8)
    assert so.hstu_attn_bwd(ctypes.byref(p), *args, None, None, None, None, vp(FAKE), 0, None) == 5


def test_noalloc_rejects_like_bwd_without_enqueueing(lib):
    """The workspace-free backward runs the backward's own argument checks
    first: same codes, nothing queued (these calls never reach the device)."""
    so = lib.load_library()
    vp = ctypes.c_void_p
    args = [vp(FAKE)] * 12
    # unsupported and larger than the built-in scratch: UNSUPPORTED, as hstu_attn_bwd says
    p, _ = problem(lib, d_qk=64, d_v=64, total_tokens=1 << 20, max_seq_len=4096)
    assert so.hstu_attn_bwd_noalloc(ctypes.byref(p), *args, None, None, None, None, None) == 2
    a2 = list(args)
    a2[8] = None                                    # dq missing
    p, _ = problem(lib)
    assert so.hstu_attn_bwd_noalloc(ctypes.byref(p), *a2, None, None, None, None, None) == 1
    p, _ = problem(lib, ln_eps=0.0)
    assert so.hstu_attn_bwd_noalloc(ctypes.byref(p), *args, None, None, None, None, None) == 1


def test_bwd_rejects_layernorm_gradients_without_tables(lib):
    """d_ln_weight / d_ln_bias need the matching table in the problem."""
    so = lib.load_library()
    vp = ctypes.c_void_p
    args = [vp(FAKE)] * 12
    p, _ = problem(lib)
    need = lib.hstu_attn_workspace_size(p, True)
    assert so.hstu_attn_bwd(ctypes.byref(p), *args, None, None, vp(FAKE), None, vp(FAKE), need,
                            None) == 1
    assert so.hstu_attn_bwd(ctypes.byref(p), *args, None, None, None, vp(FAKE), vp(FAKE), need,
                            None) == 1


def call_uvqk(lib, T=300, E=512, H=4, dqk=128, dv=128, act=0, x=FAKE, bias=None, u=FAKE,
              ws=FAKE, ws_bytes=256):
    so = lib.load_library()
    vp = ctypes.c_void_p
    return so.hstu_uvqk_fwd(T, E, H, dqk, dv, act, vp(x) if x else None, vp(FAKE),
                            vp(bias) if bias else None, vp(u) if u else None, vp(FAKE),
                            vp(FAKE), vp(FAKE), vp(ws) if ws else None, ws_bytes, None)


def call_out(lib, T=300, E=512, D=512, eps=1e-5, y=FAKE, ln_weight=None, mean=None, rstd=None,
             z=FAKE, ws=FAKE, ws_bytes=256):
    so = lib.load_library()
    vp = ctypes.c_void_p
    opt = lambda a: vp(a) if a else None
    return so.hstu_out_fwd(T, E, D, opt(y), vp(FAKE), vp(FAKE), None, opt(ln_weight), None,
                           eps, opt(z), opt(mean), opt(rstd), opt(ws), ws_bytes, None)


def test_uvqk_rejections(lib):
    assert call_uvqk(lib, T=-1) == 1
    assert call_uvqk(lib, act=2) == 1
    assert call_uvqk(lib, x=None) == 1
    assert call_uvqk(lib, u=FAKE + 8) == 1                  # not 16-byte aligned
    assert call_uvqk(lib, bias=FAKE + 4) == 1
    assert call_uvqk(lib, E=96) == 2                        # E not a multiple of 64
    assert call_uvqk(lib, H=1, dv=128) == 2                 # H*dv not a multiple of 256
    assert call_uvqk(lib, T=65536 * 128) == 2               # row tiles beyond the grid's y limit
    assert call_uvqk(lib, ws=None) == 5
    assert call_uvqk(lib, ws_bytes=255) == 5
    assert call_uvqk(lib, ws=FAKE + 16) == 5
    assert call_uvqk(lib, T=0) == 0                         # empty: nothing to do


def test_out_rejections(lib):
    assert call_out(lib, eps=0.0) == 1
    assert call_out(lib, eps=float("inf")) == 1
    assert call_out(lib, y=None) == 1
    assert call_out(lib, z=FAKE + 2) == 1
    assert call_out(lib, ln_weight=FAKE + 4) == 1
    assert call_out(lib, mean=FAKE) == 1                    # mean and rstd together or neither
    assert call_out(lib, E=384) == 2
    assert call_out(lib, D=100) == 2
    assert call_out(lib, ws=None) == 5
    assert call_out(lib, T=0) == 0


def call_cand(lib, p, C=300, maxc=200, cand_off=FAKE, cts=FAKE, q=FAKE, kh=FAKE, ws=FAKE,
              ws_bytes=1 << 24):
    so = lib.load_library()
    vp = ctypes.c_void_p
    opt = lambda a: vp(a) if a else None
    return so.hstu_cand_fwd(ctypes.byref(p), opt(kh), vp(FAKE), opt(cand_off), C, maxc, opt(cts),
                            opt(q), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), opt(ws), ws_bytes,
                            None)


def test_cand_rejections(lib):
    p, _ = problem(lib, rab_pos=FAKE, rab_pos_len=201)
    so = lib.load_library()
    need = so.hstu_cand_workspace_size(ctypes.byref(p), 300, 200)
    # status + 2 users x 2 micro-batch counters + O staging (300 x 512 fp32)
    assert need >= 256 + 300 * 4 * 128 * 4
    assert call_cand(lib, p, C=-1) == 1
    assert call_cand(lib, p, maxc=0) == 1                     # candidates but no per-user bound
    assert call_cand(lib, p, cand_off=None) == 1
    assert call_cand(lib, p, q=FAKE + 8) == 1
    assert call_cand(lib, p, kh=None) == 1
    p2, _ = problem(lib, rab_pos=FAKE, rab_pos_len=200)     # position n_b = 200 not in the table
    assert call_cand(lib, p2) == 1
    p3, _ = problem(lib, rab_time=FAKE, timestamps=FAKE, num_time_buckets=128)
    assert call_cand(lib, p3, cts=None) == 1                  # time table without request times
    p4, _ = problem(lib, d_qk=64, d_v=64)
    assert call_cand(lib, p4) == 2
    p5, _ = problem(lib, dtype=0)
    assert call_cand(lib, p5) == 2
    assert call_cand(lib, p, ws=None) == 5
    assert call_cand(lib, p, ws_bytes=need - 1) == 5
    assert call_cand(lib, p, C=0) == 0                        # nothing to score


def _al(x):
    return (x + 255) // 256 * 256


def test_workspace_sizes_with_a_time_table(lib):
    """With a time table the bf16 calls keep the time-plan words and the
    near-diagonal buckets in the workspace; the sizes follow the header's
    formulas."""
    so = lib.load_library()
    T, B, L, H = 1000, 3, 300, 4
    J = 4 * ((L + 127) // 128)
    kw = dict(total_tokens=T, batch=B, max_seq_len=L, num_heads=H, timestamps=FAKE,
              rab_time=FAKE, num_time_buckets=128)
    p, _ = problem(lib, **kw)
    q, _ = problem(lib, total_tokens=T, batch=B, max_seq_len=L, num_heads=H)
    fwd_t, fwd_0 = lib.hstu_attn_workspace_size(p, False), lib.hstu_attn_workspace_size(q, False)
    assert fwd_t - fwd_0 == _al(J * T * 4) + _al(T * 96)
    bwd_t, bwd_0 = lib.hstu_attn_workspace_size(p, True), lib.hstu_attn_workspace_size(q, True)
    assert bwd_t - bwd_0 == _al(2 * J * T * 4) + _al(T * 96)
    assert bwd_0 == 256 + _al(T * H * 128 * 2)
    C, M = 700, 300
    cand_t = so.hstu_cand_workspace_size(ctypes.byref(p), C, M)
    cand_0 = so.hstu_cand_workspace_size(ctypes.byref(q), C, M)
    assert cand_t - cand_0 == _al(J * C * 4)
