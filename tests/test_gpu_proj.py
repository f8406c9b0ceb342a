"""GPU parity of the two projection GEMMs (UVQK and output + residual +
LayerNorm; "HSTU (Generative Recommender)" model card, HSTUBlock) against the
fp64 oracle, through the C ABI.

Small problems span several 128-row tiles with a ragged tail and are compared
element by element; a large problem is compared on sampled rows (each output
row depends on its own input row only, so the oracle takes the sampled rows).

Tolerances: inputs are bf16 on both sides and the GPU accumulates in fp32
(relative error about K * 2^-24, negligible), so the error is the single bf16
rounding of each output (half an ulp: 2^-9 relative) plus, with SiLU, the
hardware tanh approximation (about 2^-11 relative); the LayerNorm statistics
are fp32.
"""
import numpy as np
import pytest
import torch

import hstu_inputs as hi
import oracle
import pointwise_attention_b200 as pa

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def close(got, ref, name, atol=1e-2, rtol=8e-3):
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert np.isfinite(got).all(), name + ": non-finite output"
    assert not bad.any(), "%s: %d of %d outside tolerance, max err %.3g at %s" % (
        name, int(bad.sum()), bad.size, err.max(), np.unravel_index(err.argmax(), err.shape))


def run_uvqk(p, act, bias=True):
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    out = pa.hstu_uvqk_fwd(p.x.to(DEV), p.w_uvqk.to(DEV), p.H, p.d_qk, p.d_v,
                           bias=p.b_uvqk.to(DEV) if bias else None, act=act, workspace=ws)
    assert pa.hstu_attn_check(ws) == 0
    return out


def ref_uvqk(p, act, bias=True, rows=None):
    x = p.x if rows is None else p.x[rows]
    return oracle.uvqk(x, p.w_uvqk, p.b_uvqk if bias else None, p.H, p.d_qk, p.d_v, act)


def compare_uvqk(p, out, ref, rows=None):
    T = p.T
    got = dict(u=out["u"], v=out["v"].reshape(T, -1), q=out["q"].reshape(T, -1),
               k=out["k"].reshape(T, -1))
    for n in ("u", "v", "q", "k"):
        g = np64(got[n])
        if rows is not None:
            g = g[rows]
        close(g, ref[n], n)


@pytest.mark.parametrize("T,E,H,act,bias", [
    (300, 512, 4, 0, True),      # 3 row tiles, ragged tail of 44
    (300, 512, 4, 1, True),      # with SiLU
    (129, 256, 2, 1, False),     # one row past a tile, no bias, Nu = 256
    (1, 64, 2, 0, True),         # a single row, one K step
    (128, 1024, 4, 1, True),     # exactly one tile, K = 1024
])
def test_uvqk_small(T, E, H, act, bias):
    p = hi.make_proj_inputs(T, E, H, seed=T + E + act)
    out = run_uvqk(p, act, bias)
    compare_uvqk(p, out, ref_uvqk(p, act, bias))


def test_uvqk_unequal_widths():
    # d_qk != d_v: the split points differ between (u, v) and (q, k)
    p = hi.make_proj_inputs(200, 256, 2, d_qk=256, d_v=128, seed=3)
    out = run_uvqk(p, 1)
    assert out["q"].shape == (200, 2, 256) and out["v"].shape == (200, 2, 128)
    compare_uvqk(p, out, ref_uvqk(p, 1))


def test_uvqk_large_sampled_rows():
    p = hi.make_proj_inputs(32768 + 77, 512, 4, seed=11)
    out = run_uvqk(p, 1)
    g = torch.Generator().manual_seed(0)
    rows = torch.cat([torch.randint(0, p.T, (200,), generator=g),
                      torch.arange(p.T - 77, p.T)]).numpy()
    compare_uvqk(p, out, ref_uvqk(p, 1, rows=rows), rows)


def run_out(p, bias=True, affine=True, stats=True):
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    z, st = pa.hstu_out_fwd(p.y.to(DEV), p.w_out.to(DEV), p.x.to(DEV),
                            bias=p.b_out.to(DEV) if bias else None,
                            ln_weight=p.ln_weight.to(DEV) if affine else None,
                            ln_bias=p.ln_bias.to(DEV) if affine else None,
                            save_stats=stats, workspace=ws)
    assert pa.hstu_attn_check(ws) == 0
    return z, st


def ref_out(p, bias=True, affine=True, rows=None):
    sel = (lambda t: t) if rows is None else (lambda t: t[rows])
    return oracle.out_proj(sel(p.y), sel(p.x), p.w_out, p.b_out if bias else None,
                           p.ln_weight if affine else None, p.ln_bias if affine else None)


def compare_out(z, st, ref, rows=None):
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])
    close(sel(np64(z)), ref["z"], "z", atol=2e-2, rtol=1e-2)
    if st is not None:
        np.testing.assert_allclose(sel(np64(st[0])), ref["mean"], rtol=1e-4, atol=1e-4)
        np.testing.assert_allclose(sel(np64(st[1])), ref["rstd"], rtol=1e-4)


@pytest.mark.parametrize("T,E,H,bias,affine", [
    (300, 512, 4, True, True),
    (300, 512, 4, False, False),
    (129, 256, 2, True, True),
    (1, 256, 1, True, False),    # D = 128
    (256, 512, 8, True, True),   # D = 1024
])
def test_out_small(T, E, H, bias, affine):
    p = hi.make_proj_inputs(T, E, H, seed=T + 7 * E + H)
    z, st = run_out(p, bias, affine)
    compare_out(z, st, ref_out(p, bias, affine))


def test_out_without_stats():
    p = hi.make_proj_inputs(140, 512, 4, seed=5)
    z, st = run_out(p, stats=False)
    assert st is None
    compare_out(z, None, ref_out(p))


def test_out_large_sampled_rows():
    p = hi.make_proj_inputs(32768 + 77, 512, 4, seed=12)
    z, st = run_out(p)
    g = torch.Generator().manual_seed(1)
    rows = torch.cat([torch.randint(0, p.T, (200,), generator=g),
                      torch.arange(p.T - 77, p.T)]).numpy()
    compare_out(z, st, ref_out(p, rows=rows), rows)


def test_layer_chain_feeds_attention():
    """UVQK -> attention -> output projection on one jagged batch, against the
    oracle's own chain from the same seeded inputs (each stage's result rounded
    to bf16, as the GPU stores it): the projection outputs land in the layouts
    the attention reads."""
    lengths = (300, 77, 512)
    T = sum(lengths)
    p = hi.make_proj_inputs(T, 512, 4, seed=21)
    offsets = torch.tensor([0, 300, 377, 889], dtype=torch.int32)
    out = run_uvqk(p, 1)
    y, _ = pa.hstu_attn_fwd(out["q"], out["k"], out["v"], out["u"], offsets.to(DEV), 512)
    z, _ = pa.hstu_out_fwd(y, p.w_out.to(DEV), p.x.to(DEV), bias=p.b_out.to(DEV),
                           ln_weight=p.ln_weight.to(DEV), ln_bias=p.ln_bias.to(DEV))
    torch.cuda.synchronize()

    r = ref_uvqk(p, 1)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    spec = hi.Spec("chain", "bf16", batch=3, heads=4, d_qk=128, d_v=128, lengths=lengths,
                   norm="own")
    inp = hi.Inputs(spec=spec, offsets=offsets, q=bf(r["q"]).reshape(T, 4, 128),
                    k=bf(r["k"]).reshape(T, 4, 128), v=bf(r["v"]).reshape(T, 4, 128),
                    u=bf(r["u"]), timestamps=None, rab_pos=None, rab_time=None, dy=None,
                    norm_len=0, rab_pos_len=0)
    y_ref = bf(oracle.fwd(inp)["y"])
    close(np64(y), y_ref.double().numpy(), "y", atol=2e-2, rtol=1e-2)
    z_ref = oracle.out_proj(y_ref, p.x, p.w_out, p.b_out, p.ln_weight, p.ln_bias)
    close(np64(z), z_ref["z"], "z", atol=3e-2, rtol=2e-2)
