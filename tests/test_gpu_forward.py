"""GPU parity of the forward (CUDA path through the C ABI) against the fp64 oracle.

Small problems span several 128-row tiles and ragged tails and are compared
element by element on every output; the named workloads run at full size in
the launch configuration the benchmark times and are compared on every row.
"""
import numpy as np
import pytest
import torch

import hstu_inputs as hi
import oracle
import pointwise_attention_b200 as pa
from tests.gpu_util import assert_close, np64, run_fwd, to_dev

pytestmark = pytest.mark.gpu


def spec(lengths, H=4, d=128, dtype="bf16", pos=True, time=False, norm="own", norm_len=0,
         qk_std=1 / np.sqrt(128), rab_std=0.02, L=None, ts_sorted=True, affine=False):
    return hi.Spec("case", dtype, batch=len(lengths), heads=H, d_qk=d, d_v=d,
                   lengths=tuple(lengths), qk_std=qk_std, vu_std=1.0,
                   rab_pos_len=(L or max(max(lengths), 1)) if pos else 0, rab_time=time,
                   rab_std=rab_std, norm=norm, norm_len=norm_len, ts_sorted=ts_sorted,
                   ln_affine=affine)


def check_full(inp, dtype):
    y, saved, _ = run_fwd(inp)
    ref = oracle.fwd(inp)
    assert_close(np64(y), ref["y"], dtype, "y")
    assert_close(np64(saved[0]), ref["o"], dtype, "o_save")
    return y, saved, ref


def test_tiny_fp32_workload():
    inp = hi.make_inputs(hi.WORKLOADS["tiny"], seed=0)
    y, saved, ref = check_full(inp, "f32")
    np.testing.assert_allclose(np64(saved[1]), ref["mean"], rtol=0, atol=1e-5 * np.abs(ref["mean"]).max() + 1e-12)
    np.testing.assert_allclose(np64(saved[2]), ref["rstd"], rtol=1e-5)


@pytest.mark.parametrize("case", [
    dict(lengths=(128,), H=1),
    dict(lengths=(256,), H=2, pos=False),
    dict(lengths=(1, 127, 128, 129, 300), H=4),
    dict(lengths=(513, 77), H=8, time=True),
    dict(lengths=(200, 0, 385), H=4, time=True, norm="fixed", norm_len=500),
    dict(lengths=(640,), H=3, time=True, L=1000),
    dict(lengths=(260, 131), H=2, time=True, ts_sorted=False),
    dict(lengths=(300, 257), H=4, qk_std=1.0, rab_std=1.0, time=True),   # stress: large logits
    dict(lengths=(257, 100, 33), H=5, time=True),                          # odd head counts
    dict(lengths=(129, 129, 129), H=7),
    dict(lengths=(300, 70, 129), H=4, time=True, affine=True),             # LayerNorm affine
    dict(lengths=(200,), H=3, affine=True),
])
def test_bf16_small(case):
    inp = hi.make_inputs(spec(**case), seed=1)
    check_full(inp, "bf16")


@pytest.mark.parametrize("case", [
    dict(lengths=(5, 70, 130), H=2, d=32, dtype="f32", time=True),
    dict(lengths=(64, 1), H=4, d=100, dtype="f32", pos=False, norm="fixed", norm_len=64),
    dict(lengths=(40, 9), H=2, d=32, dtype="f32", time=True, affine=True),
])
def test_fp32_small(case):
    inp = hi.make_inputs(spec(**case, qk_std=0.5), seed=2)
    check_full(inp, "f32")


@pytest.mark.parametrize("how", ["wide", "jump"])
def test_time_span_past_2_31(how):
    """Time differences of 2^31 s and more take the 64-bit bucket search."""
    inp = hi.wide_time_span(hi.make_inputs(spec((300, 150), H=2, time=True), seed=5), how)
    check_full(inp, "bf16")


def test_neurarch_full():
    inp = hi.make_inputs(hi.WORKLOADS["neurarch"], seed=0)
    check_full(inp, "bf16")


def nan_outputs(inp):
    """Output buffers prefilled with NaN: a row the kernel never writes fails
    the comparison (every compared value must be finite)."""
    T, D = inp.u.shape
    y = torch.full((T, D), float("nan"), dtype=inp.q.dtype, device="cuda")
    saved = (torch.full((T, D), float("nan"), dtype=torch.float32, device="cuda"),
             torch.full((T,), float("nan"), dtype=torch.float32, device="cuda"),
             torch.full((T,), float("nan"), dtype=torch.float32, device="cuda"))
    return y, saved


def check_stats(saved, ref, what):
    """LayerNorm statistics of every row: the mean against the O tolerance
    (it is an average of O), rstd relative to itself."""
    o_scale = float(np.abs(ref["o"]).max())
    mean = np64(saved[1])
    assert np.all(np.isfinite(mean)), what
    err = np.abs(mean - ref["mean"])
    assert err.max() <= 1e-2 * o_scale and err.mean() <= 1e-3 * o_scale, (what, err.max())
    np.testing.assert_allclose(np64(saved[2]), ref["rstd"], rtol=1e-2, err_msg=what)


@pytest.mark.parametrize("name", ["jagged", "long", "train", "train_sl"])
def test_full_size_every_row(name):
    """The named workloads at full size, in the launch configuration the
    benchmark times, compared with the oracle on every element of Y, the saved
    O and the LayerNorm statistics."""
    inp = hi.make_inputs(hi.WORKLOADS[name], seed=0)
    dev = to_dev(inp)
    y, saved = nan_outputs(inp)
    pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"], inp.max_seq_len,
                     timestamps=dev["timestamps"], rab_pos=dev["rab_pos"],
                     rab_time=dev["rab_time"], norm_len=inp.norm_len, save_for_backward=True,
                     y=y, saved=saved)
    torch.cuda.synchronize()
    ref = oracle.fwd(inp)
    assert_close(np64(y), ref["y"], "bf16", "y[%s]" % name)
    assert_close(np64(saved[0]), ref["o"], "bf16", "o[%s]" % name)
    check_stats(saved, ref, name)
    # Y alone (no saved outputs) is the inference path the benchmark times
    y2 = torch.full_like(y, float("nan"))
    pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"], inp.max_seq_len,
                     timestamps=dev["timestamps"], rab_pos=dev["rab_pos"],
                     rab_time=dev["rab_time"], norm_len=inp.norm_len, y=y2)
    torch.cuda.synchronize()
    assert_close(np64(y2), ref["y"], "bf16", "y[%s] without saved outputs" % name)


def test_causality_on_gpu():
    inp = hi.make_inputs(spec((700,), H=4, time=True), seed=3)
    y0 = np64(run_fwd(inp, save=False)[0])
    cut = 333
    for name in ("q", "k", "v", "u"):
        pert = hi.make_inputs(spec((700,), H=4, time=True), seed=3)
        t = getattr(pert, name)
        t[cut + 1:] = -t[cut + 1:]
        y1 = np64(run_fwd(pert, save=False)[0])
        assert np.array_equal(y1[:cut + 1], y0[:cut + 1]), name
        assert not np.array_equal(y1[cut + 1:], y0[cut + 1:]), name


def test_deterministic():
    inp = hi.make_inputs(spec((900, 300), H=4, time=True), seed=4)
    a = np64(run_fwd(inp)[0])
    b = np64(run_fwd(inp)[0])
    assert np.array_equal(a, b)


def test_degenerate_shapes():
    # empty sequences, single tokens, max_seq_len above every length
    inp = hi.make_inputs(spec((0, 1, 0, 2, 129), H=2, time=True, L=400), seed=5)
    dev = to_dev(inp)
    y, saved = pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"], 400,
                                timestamps=dev["timestamps"], rab_pos=dev["rab_pos"],
                                rab_time=dev["rab_time"], save_for_backward=True)
    torch.cuda.synchronize()
    ref = oracle.fwd(inp)
    assert_close(np64(y), ref["y"], "bf16", "y")
    # a first token alone: O_0 = SiLU(q0.k0 + b)/1 * v0 exactly up to bf16 rounding of P
    # all-empty problem: nothing to do
    empty = hi.make_inputs(spec((0, 0), H=2), seed=6)
    dev = to_dev(empty)
    y, _ = pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"], 1,
                            rab_pos=dev["rab_pos"])
    torch.cuda.synchronize()
    assert y.numel() == 0


def test_work_counters_return_to_zero_and_calls_repeat():
    """The bf16 forward hands (sequence, query tile, head) items to its CTAs
    from a counter in the workspace head, and counts the heads done per
    (sequence, query tile) block; the last CTA to finish zeroes the first, the
    CTA that normalises a block zeroes its count.  So back-to-back calls on
    one workspace (first used with many empty slots: long and short sequences
    mixed) all see every item, and the counters are zero after every call."""
    inp = hi.make_inputs(spec((1500, 3, 700, 1, 0, 1200), H=4, time=True), seed=31)
    dev = to_dev(inp)
    p = pa.make_problem(dev["q"], dev["v"], dev["offsets"], inp.max_seq_len, dev["timestamps"],
                        dev["rab_pos"], dev["rab_time"], inp.norm_len)
    ws = pa.new_workspace(p, False, "cuda")
    n_cnt = len(inp.lengths) * ((inp.max_seq_len + 127) // 128)
    ref = oracle.fwd(inp)
    for call in range(3):
        y, _ = pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"],
                                inp.max_seq_len, timestamps=dev["timestamps"],
                                rab_pos=dev["rab_pos"], rab_time=dev["rab_time"],
                                workspace=ws)
        torch.cuda.synchronize()
        words = ws.view(torch.int32).cpu().numpy()
        assert words[16] == 0 and words[17] == 0, words[:20]
        assert not words[64:64 + n_cnt].any(), words[64:64 + n_cnt]
        assert pa.hstu_attn_check(ws) == 0
        assert_close(np64(y), ref["y"], "bf16", "y (call %d)" % call)


def test_sixteen_byte_aligned_buffers():
    """U, Y and the saved O at 16-byte (not 32-byte) aligned addresses take
    the 16-byte access path and give the same result."""
    inp = hi.make_inputs(spec((300, 170), H=2, time=True), seed=33)
    dev = to_dev(inp)
    T, D = inp.u.shape

    def shifted(shape, dtype, like=None):
        n = int(np.prod(shape))
        esz = torch.tensor([], dtype=dtype).element_size()
        big = torch.zeros(n + 64 // esz, dtype=dtype, device="cuda")
        t = big[16 // esz:16 // esz + n].view(*shape)
        assert t.data_ptr() % 32 == 16
        if like is not None:
            t.copy_(like)
        return t

    u = shifted((T, D), torch.bfloat16, dev["u"])
    y = shifted((T, D), torch.bfloat16)
    o_save = shifted((T, D), torch.float32)
    saved = (o_save, torch.zeros(T, device="cuda"), torch.zeros(T, device="cuda"))
    pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], u, dev["offsets"], inp.max_seq_len,
                     timestamps=dev["timestamps"], rab_pos=dev["rab_pos"],
                     rab_time=dev["rab_time"], save_for_backward=True, y=y, saved=saved)
    torch.cuda.synchronize()
    ref = oracle.fwd(inp)
    assert_close(np64(y), ref["y"], "bf16", "y")
    assert_close(np64(o_save), ref["o"], "bf16", "o_save")


def test_many_short_sequences():
    """Hundreds of sequences of 0 to 300 tokens: most work slots of the
    launch are empty and the clusters claim many small items."""
    rng = np.random.default_rng(41)
    lengths = tuple(int(x) for x in rng.integers(0, 301, size=180))
    inp = hi.make_inputs(spec(lengths, H=2, time=True, L=300), seed=42)
    check_full(inp, "bf16")


def test_bad_device_offsets_reported():
    """Offsets that contradict max_seq_len, given without a host copy, are found
    by the kernel: the sequence is skipped and the status word says so."""
    inp = hi.make_inputs(spec((300, 100), H=2), seed=7)
    dev = to_dev(inp)
    p = pa.make_problem(dev["q"], dev["v"], dev["offsets"], 200)
    ws = pa.new_workspace(p, False, "cuda")
    pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"], 200,
                     rab_pos=None, workspace=ws)
    assert pa.hstu_attn_check(ws) == 1
    assert pa.hstu_attn_check(ws) == 0          # re-armed


def test_bounded_wait_timeout_is_reported_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert pa.hstu_selftest_wait_timeout(ws, budget_ns=20_000_000) == 0
    assert pa.hstu_attn_check(ws) == 4
    assert pa.hstu_attn_check(ws) == 0
    inp = hi.make_inputs(spec((200,), H=2), seed=8)
    y, saved, _ = run_fwd(inp)
    assert_close(np64(y), oracle.fwd(inp)["y"], "bf16", "y after timeout")
