"""GPU parity of candidate scoring against cached histories (M-FALCON reading:
each candidate is the token after its user's history, attending to the
history and itself only) with the fp64 oracle, through the C ABI.

Small problems cover empty histories, users without candidates, micro-batches
with ragged tails and both bias tables; the full-size workload is compared on
sampled candidates (each candidate's row depends only on its own inputs and
its user's history, so the oracle takes the sampled candidates alone).  The
tolerance is the forward's for bf16 (max error <= 1e-2 max|ref|, mean error
<= 1e-3 max|ref|).
"""
import numpy as np
import pytest
import torch

import hstu_inputs as hi
import oracle
import pointwise_attention_b200 as pa
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run(ci, max_cands=None, workspace=None):
    import ctypes
    h = ci.hist
    d = lambda t: None if t is None else t.to(DEV)
    mc = max_cands if max_cands is not None else max(ci.counts + [0])
    if workspace is None:
        p = pa.make_problem(d(h.k), d(h.v), d(h.offsets), max(h.lengths + [0]),
                            d(h.timestamps), d(h.rab_pos), d(h.rab_time))
        n = pa.load_library().hstu_cand_workspace_size(ctypes.byref(p), ci.total_cands, mc)
        workspace = torch.zeros(max(n, 256), dtype=torch.uint8, device=DEV)
    y = pa.hstu_cand_fwd(d(h.k), d(h.v), d(h.offsets), max(h.lengths + [0]), d(ci.qc),
                         d(ci.kc), d(ci.vc), d(ci.uc), d(ci.cand_offsets), mc,
                         timestamps=d(h.timestamps), cand_timestamps=d(ci.cand_ts),
                         rab_pos=d(h.rab_pos), rab_time=d(h.rab_time), norm_len=h.norm_len,
                         ln_weight=d(h.ln_weight), ln_bias=d(h.ln_bias), workspace=workspace)
    assert pa.hstu_attn_check(workspace) == 0
    return y


def spec(lengths, H=4, pos=True, time=True, norm="own", norm_len=0, affine=False, L=None):
    return hi.Spec("cand", "bf16", batch=len(lengths), heads=H, d_qk=128, d_v=128,
                   lengths=tuple(lengths), qk_std=1 / np.sqrt(128), vu_std=1.0,
                   rab_pos_len=(L or max(lengths) + 1) if pos else 0, rab_time=time,
                   rab_std=0.02, norm=norm, norm_len=norm_len, ln_affine=affine)


@pytest.mark.parametrize("lengths,cands,kw", [
    ((300, 0, 129, 1), (5, 130, 3, 200), {}),                 # empty history, 2 micro-batches
    ((512, 77), (128, 129), dict(H=2)),
    ((256, 1000), (64, 0), dict(time=False)),                  # a user without candidates
    ((200, 45), (17, 300), dict(pos=False)),
    ((128, 384), (33, 40), dict(pos=False, time=False, norm="fixed", norm_len=700)),
    ((640,), (250,), dict(H=8, affine=True)),
    ((1, 2, 3), (1, 2, 3), dict(H=1)),
])
def test_small(lengths, cands, kw):
    sp = spec(lengths, **kw)
    # the seeded histories, then explicit per-user candidate counts
    ci = hi.make_cand_inputs(sp, 0, seed=len(lengths) + sum(cands))
    offs = np.concatenate([[0], np.cumsum(cands)]).astype(np.int32)
    g = torch.Generator().manual_seed(sum(cands))
    C = int(offs[-1])
    H = sp.heads
    ci.cand_offsets = torch.from_numpy(offs)
    ci.qc = (torch.randn(C, H, 128, generator=g) / np.sqrt(128)).to(torch.bfloat16)
    ci.kc = (torch.randn(C, H, 128, generator=g) / np.sqrt(128)).to(torch.bfloat16)
    ci.vc = torch.randn(C, H, 128, generator=g).to(torch.bfloat16)
    ci.uc = torch.randn(C, H * 128, generator=g).to(torch.bfloat16)
    if sp.rab_time:
        ho = ci.hist.offsets.tolist()
        ts = []
        for b, c in enumerate(cands):
            last = int(ci.hist.timestamps[ho[b + 1] - 1]) if ho[b + 1] > ho[b] else 1_700_000_000
            ts.append(last + torch.randint(1, 100_000, (c,), generator=g))
        ci.cand_ts = torch.cat(ts).to(torch.int64)
    else:
        ci.cand_ts = None
    y = run(ci)
    ref = oracle.mfalcon(ci)
    assert_close(y.double().cpu().numpy(), ref["y"], "bf16", "y")


def test_workspace_is_reusable_and_status_clean():
    sp = spec((300, 50), H=4)
    ci = hi.make_cand_inputs(sp, (100, 200), seed=9)
    h = ci.hist
    p = pa.make_problem(h.k.to(DEV), h.v.to(DEV), h.offsets.to(DEV), 300,
                        h.timestamps.to(DEV), h.rab_pos.to(DEV), h.rab_time.to(DEV))
    lib = pa.load_library()
    import ctypes
    n = lib.hstu_cand_workspace_size(ctypes.byref(p), ci.total_cands, max(ci.counts))
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    y1 = run(ci, workspace=ws)
    y2 = run(ci, workspace=ws)
    assert torch.equal(y1, y2)                       # counters returned to zero in between
    assert pa.hstu_attn_check(ws) == 0
    # per-micro-batch counters are back at zero
    cnt = ws[256:256 + 4 * 2 * 2].view(torch.int32)   # B = 2 users x 2 micro-batches
    assert int(cnt.abs().sum()) == 0


def test_full_size_sampled_candidates():
    sp, ncand = hi.CAND_WORKLOADS["mfalcon"]
    ci = hi.make_cand_inputs(sp, ncand, seed=0)
    y = run(ci)
    # the oracle on a sample: a few candidates of every user, first and last
    # of each micro-batch included
    g = torch.Generator().manual_seed(4)
    keep = []
    co = ci.cand_offsets.tolist()
    for b in range(sp.batch):
        picks = {co[b], co[b + 1] - 1, co[b] + 127, co[b] + 128}
        picks |= set(torch.randint(co[b], co[b + 1], (3,), generator=g).tolist())
        keep.extend(sorted(x for x in picks if co[b] <= x < co[b + 1]))
    keep_t = torch.tensor(keep)
    counts = [sum(1 for x in keep if co[b] <= x < co[b + 1]) for b in range(sp.batch)]
    sub = hi.CandInputs(ci.hist, torch.tensor(np.concatenate([[0], np.cumsum(counts)]),
                                              dtype=torch.int32),
                        ci.qc[keep_t], ci.kc[keep_t], ci.vc[keep_t], ci.uc[keep_t],
                        ci.cand_ts[keep_t])
    ref = oracle.mfalcon(sub)
    assert_close(y[keep_t.to(DEV)].double().cpu().numpy(), ref["y"], "bf16", "y")


@pytest.mark.parametrize("how", ["wide", "jump"])
def test_time_span_past_2_31(how):
    """History timestamps whose differences reach 2^31 s and more: the chunks
    that cross them take the 64-bit per-element search, the others the plans."""
    sp = spec((300, 150), H=2)
    ci = hi.make_cand_inputs(sp, (40, 130), seed=21)
    hi.wide_time_span(ci.hist, how)
    y = run(ci)
    ref = oracle.mfalcon(ci)
    assert_close(y.double().cpu().numpy(), ref["y"], "bf16", "y")
