"""GPU parity of the backward (through the C ABI) against the oracle's fp64
analytic gradients: dQ, dK, dV, dU, d(rab_pos) and d(rab_time)."""
import numpy as np
import pytest

import hstu_inputs as hi
import oracle
from tests.gpu_util import assert_close, np64, run_bwd, run_fwd

pytestmark = pytest.mark.gpu


def spec(lengths, H=4, d=128, dtype="bf16", pos=True, time=False, norm="own", norm_len=0,
         qk_std=1 / np.sqrt(128), L=None, ts_sorted=True, affine=False):
    return hi.Spec("case", dtype, batch=len(lengths), heads=H, d_qk=d, d_v=d,
                   lengths=tuple(lengths), qk_std=qk_std, vu_std=1.0,
                   rab_pos_len=(L or max(lengths)) if pos else 0, rab_time=time,
                   norm=norm, norm_len=norm_len, grad=True, ts_sorted=ts_sorted,
                   ln_affine=affine)


def check_bwd(inp, dtype, rows_of=None):
    y, saved, dev = run_fwd(inp)
    g = run_bwd(inp, dev, saved)
    ref = oracle.bwd(inp)
    for name in ("dq", "dk", "dv", "du"):
        assert_close(np64(g[name]), ref[name], dtype, name)
    if inp.rab_pos is not None:
        assert_close(np64(g["d_rab_pos"]), ref["d_rab_pos"], dtype, "d_rab_pos")
    if inp.rab_time is not None:
        assert_close(np64(g["d_rab_time"]), ref["d_rab_time"], dtype, "d_rab_time")
    if inp.ln_weight is not None:
        assert_close(np64(g["d_ln_weight"]), ref["d_ln_weight"], dtype, "d_ln_weight")
        assert_close(np64(g["d_ln_bias"]), ref["d_ln_bias"], dtype, "d_ln_bias")


@pytest.mark.parametrize("case", [
    dict(lengths=(40, 3), H=2, d=16, dtype="f32", time=True),
    dict(lengths=(130,), H=3, d=64, dtype="f32", norm="fixed", norm_len=200),
    dict(lengths=(33, 8), H=2, d=32, dtype="f32", time=True, affine=True),
])
def test_fp32_backward(case):
    check_bwd(hi.make_inputs(spec(**case, qk_std=0.5), seed=11), "f32")


@pytest.mark.parametrize("case", [
    dict(lengths=(128,), H=1),
    dict(lengths=(1, 200, 129), H=4, time=True),
    dict(lengths=(300, 0, 64), H=2, norm="fixed", norm_len=300),
    dict(lengths=(257, 129), H=8, time=True),
    # unsorted timestamps: both kernels take the per-element bucket search and
    # the dQ kernel accumulates d(rab_time) per element
    dict(lengths=(260, 131), H=2, time=True, ts_sorted=False),
    dict(lengths=(200,), H=4, pos=False, time=True, ts_sorted=False),
    # LayerNorm weight and bias, and their gradients (summed over every token)
    dict(lengths=(300, 1, 170), H=4, time=True, affine=True),
    dict(lengths=(257,), H=8, affine=True),
])
def test_bf16_backward_small(case):
    check_bwd(hi.make_inputs(spec(**case), seed=12), "bf16")


@pytest.mark.parametrize("how", ["wide", "jump"])
def test_time_span_past_2_31(how):
    """Time differences of 2^31 s and more: blocks that cross them take the
    64-bit per-element path, the others the 32-bit plans."""
    inp = hi.wide_time_span(hi.make_inputs(spec((300, 150), H=2, time=True), seed=13), how)
    check_bwd(inp, "bf16")


def test_train_reduced_batch():
    """The training workload's shapes and distributions with 2 sequences."""
    check_bwd(hi.make_inputs(hi.workload("train", batch=2), seed=0), "bf16")


def test_train_shapes_with_time_bias():
    """Training shapes (2 x 2048 tokens, H=4) with the time bias added: the
    backward of both relative biases at once, d(rab_time) included."""
    check_bwd(hi.make_inputs(hi.workload("train", batch=2, rab_time=True), seed=3), "bf16")


def test_train_full_size():
    """Full training workload on the GPU: every element of dQ, dK, dV, dU and
    d(rab_pos) compared with the oracle's gradients of the full problem."""
    inp = hi.make_inputs(hi.WORKLOADS["train"], seed=0)
    y, saved, dev = run_fwd(inp)
    g = run_bwd(inp, dev, saved)
    ref_full = oracle.bwd(inp)
    for name in ("dq", "dk", "dv", "du"):
        assert_close(np64(g[name]), ref_full[name], "bf16", name)
    assert_close(np64(g["d_rab_pos"]), ref_full["d_rab_pos"], "bf16", "d_rab_pos")


def test_train_time_full_size():
    """Full train_time workload (16 x 2048 tokens, H=4, position and time bias):
    every element of every gradient, d(rab_time) included, against the oracle."""
    inp = hi.make_inputs(hi.WORKLOADS["train_time"], seed=0)
    y, saved, dev = run_fwd(inp)
    g = run_bwd(inp, dev, saved)
    ref = oracle.bwd(inp)
    for name in ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time"):
        assert_close(np64(g[name]), ref[name], "bf16", name)


def test_train_sl_reduced_batch():
    """Training on histories shortened by Stochastic Length (lengths from the
    train_sl generator: jagged, some cut to 2048), with both biases."""
    inp = hi.make_inputs(hi.workload("train_sl", batch=5), seed=2)
    assert len(set(inp.lengths)) > 1
    check_bwd(inp, "bf16")


def test_train_with_layernorm_affine():
    """Training shapes (2 x 2048 tokens, H=4) with the LayerNorm weight and bias:
    the affine form of the LayerNorm/gate backward and its table gradients."""
    check_bwd(hi.make_inputs(hi.workload("train", batch=2, ln_affine=True), seed=4), "bf16")
