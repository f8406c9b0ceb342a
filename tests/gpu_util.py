"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
call the library through its C ABI (the Python binding), compare with the
oracle under the stated tolerances.

Tolerances (per output tensor, relative to that tensor's max |reference|):
  bf16 inputs, fp32 accumulation:  max |err| <= 1e-2 * max|ref|,
                                   mean |err| <= 1e-3 * max|ref|
  fp32 inputs:                     max |err| <= 1e-5 * max|ref|
"""
import numpy as np
import torch

import pointwise_attention_b200 as pa

TOL = {"bf16": (1e-2, 1e-3), "f32": (1e-5, 1e-5)}


def to_dev(inp, device="cuda"):
    d = lambda x: None if x is None else x.to(device).contiguous()
    return dict(q=d(inp.q), k=d(inp.k), v=d(inp.v), u=d(inp.u), offsets=d(inp.offsets),
                timestamps=d(inp.timestamps), rab_pos=d(inp.rab_pos), rab_time=d(inp.rab_time),
                dy=d(inp.dy), ln_weight=d(inp.ln_weight), ln_bias=d(inp.ln_bias))


def max_len(inp):
    return max(inp.max_seq_len, 1)


def run_fwd(inp, save=True, dev=None, workspace=None, check=True):
    dev = dev or to_dev(inp)
    y, saved = pa.hstu_attn_fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"],
                                max_len(inp), timestamps=dev["timestamps"],
                                rab_pos=dev["rab_pos"], rab_time=dev["rab_time"],
                                norm_len=inp.norm_len, save_for_backward=save,
                                ln_weight=dev["ln_weight"], ln_bias=dev["ln_bias"],
                                offsets_host=inp.offsets, workspace=workspace)
    if check:
        ws = workspace
        if ws is not None:
            assert pa.hstu_attn_check(ws) == 0
    torch.cuda.synchronize()
    return y, saved, dev


def run_bwd(inp, dev, saved):
    g = pa.hstu_attn_bwd(dev["dy"], dev["q"], dev["k"], dev["v"], dev["u"], dev["offsets"],
                         max_len(inp), saved, timestamps=dev["timestamps"],
                         rab_pos=dev["rab_pos"], rab_time=dev["rab_time"],
                         norm_len=inp.norm_len, ln_weight=dev["ln_weight"],
                         ln_bias=dev["ln_bias"], offsets_host=inp.offsets)
    torch.cuda.synchronize()
    return g


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "%s: non-finite values" % what
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    if scale == 0.0:
        assert np.all(got == 0.0), what
        return
    err = np.abs(got - ref)
    tmax, tmean = TOL[dtype]
    assert err.max() <= tmax * scale, "%s: max err %.3e > %.1e * %.3e" % (
        what, err.max(), tmax, scale)
    assert err.mean() <= tmean * scale, "%s: mean err %.3e > %.1e * %.3e" % (
        what, err.mean(), tmean, scale)
