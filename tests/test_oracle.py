"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these tests needs a GPU.  Each pin is chosen so that a plausible slip in
the oracle (a dropped bias term, a wrong sign or index, a transposed operand, a
wrong normaliser, an off-by-one mask) fails at least one of them:

* dense torch restatement of the model card's HSTUBlock.forward (matrix form,
  library matmul / tril / layer_norm) -- forward to 1e-12;
* torch.autograd of that restatement -- every gradient to 1e-10;
* central finite differences of the oracle's own forward -- every gradient;
* the closed form of the first position, O_0 = SiLU(q_0.k_0 + b_00)/N * v_0;
* invariants: causality, linearity of O in V, zero output for K = 0 without
  bias, the A read-out with V = I, packing (jagged = each sequence alone),
  head permutation, LayerNorm row statistics;
* time buckets against exp thresholds and the special cases 0, +-1, the cap.
"""
import math

import numpy as np
import pytest
import torch

import hstu_inputs as hi
from tests.dense_torch import dense_forward


def small_inputs(lengths=(5, 9, 1, 12), H=3, dqk=6, dv=4, rab_pos=True, rab_time=True,
                 norm="own", norm_len=0, seed=0, qk_std=0.7, rab_std=0.5, grad=True,
                 ts_sorted=True, L=None, ln_affine=False):
    spec = hi.Spec("t", "f32", batch=len(lengths), heads=H, d_qk=dqk, d_v=dv,
                   lengths=tuple(lengths), qk_std=qk_std, vu_std=1.0,
                   rab_pos_len=(L or max(lengths)) if rab_pos else 0, rab_time=rab_time,
                   rab_std=rab_std, norm=norm, norm_len=norm_len, grad=grad,
                   ts_sorted=ts_sorted, ln_affine=ln_affine)
    inp = hi.make_inputs(spec, seed=seed)
    if rab_time:
        # Spread the timestamps so that many buckets are reached in small cases.
        g = torch.Generator().manual_seed(seed + 100)
        gaps = torch.randint(0, 4000, (inp.total_tokens,), generator=g).to(torch.int64)
        ts = []
        for b, n in enumerate(inp.lengths):
            s = int(inp.offsets[b])
            seq = 1_700_000_000 + torch.cumsum(gaps[s:s + n], 0)
            if not ts_sorted and n:
                seq = seq[torch.randperm(n, generator=g)]
            ts.append(seq)
        inp.timestamps = torch.cat(ts)
    return inp


def torch_args(inp, requires_grad=False):
    d = lambda x: None if x is None else x.to(torch.float64).clone().requires_grad_(requires_grad)
    return dict(offsets=inp.offsets.tolist(), q=d(inp.q), k=d(inp.k), v=d(inp.v), u=d(inp.u),
                ts=inp.timestamps, rab_pos=d(inp.rab_pos), rab_time=d(inp.rab_time),
                norm_len=inp.norm_len, ln_weight=d(inp.ln_weight), ln_bias=d(inp.ln_bias))


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    scale = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / scale)


@pytest.mark.parametrize("case", [
    dict(),
    dict(norm="fixed", norm_len=17),
    dict(rab_time=False),
    dict(rab_pos=False, rab_time=False),
    dict(ts_sorted=False),
    dict(lengths=(0, 7, 0, 3), H=2),
    dict(lengths=(16,), H=1, dqk=3, dv=5, qk_std=2.0, rab_std=2.0),
    dict(L=20),
    dict(ln_affine=True),
])
def test_forward_matches_dense_torch(oracle_lib, case):
    inp = small_inputs(**case)
    got = oracle_lib.fwd(inp)
    Y, O = dense_forward(**torch_args(inp), return_o=True)
    assert rel_err(got["o"], O.numpy()) < 1e-12
    assert rel_err(got["y"], Y.numpy()) < 1e-12


@pytest.mark.parametrize("case", [
    dict(),
    dict(norm="fixed", norm_len=11),
    dict(ts_sorted=False),
    dict(lengths=(0, 7, 0, 3), H=2),
    dict(rab_pos=False, rab_time=False, lengths=(13,), H=2, qk_std=1.5),
    dict(ln_affine=True),
])
def test_backward_matches_autograd(oracle_lib, case):
    inp = small_inputs(**case)
    ta = torch_args(inp, requires_grad=True)
    Y = dense_forward(**ta)
    Y.backward(inp.dy.to(torch.float64))
    got = oracle_lib.bwd(inp)
    assert rel_err(got["dq"], ta["q"].grad.numpy()) < 1e-10
    assert rel_err(got["dk"], ta["k"].grad.numpy()) < 1e-10
    assert rel_err(got["dv"], ta["v"].grad.numpy()) < 1e-10
    assert rel_err(got["du"], ta["u"].grad.numpy()) < 1e-10
    if inp.rab_pos is not None:
        assert rel_err(got["d_rab_pos"], ta["rab_pos"].grad.numpy()) < 1e-10
    if inp.rab_time is not None:
        assert rel_err(got["d_rab_time"], ta["rab_time"].grad.numpy()) < 1e-10
    if inp.ln_weight is not None:
        assert rel_err(got["d_ln_weight"], ta["ln_weight"].grad.numpy()) < 1e-10
        assert rel_err(got["d_ln_bias"], ta["ln_bias"].grad.numpy()) < 1e-10


def test_backward_finite_differences(oracle_lib):
    """<grad, R> from the oracle's backward equals the central difference of
    sum(Y * dY) along a random direction R, for every differentiable input
    (the LayerNorm weight and bias included)."""
    inp = small_inputs(lengths=(6, 4), H=2, dqk=3, dv=3, ln_affine=True)
    a = oracle_lib._args_from_inputs(inp)
    dy = inp.dy.to(torch.float64).numpy()
    grads = oracle_lib.bwd_raw(a, dy)
    rng = np.random.default_rng(1)
    h = 1e-6
    fields = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("u", "du"),
              ("rab_pos", "d_rab_pos"), ("rab_time", "d_rab_time"),
              ("ln_weight", "d_ln_weight"), ("ln_bias", "d_ln_bias")]
    for name, gname in fields:
        base = getattr(a, name).copy()
        R = rng.standard_normal(base.shape)
        vals = []
        for sgn in (+1, -1):
            getattr(a, name)[...] = base + sgn * h * R
            vals.append(float((oracle_lib.fwd_raw(a)["y"] * dy).sum()))
        getattr(a, name)[...] = base
        fd = (vals[0] - vals[1]) / (2 * h)
        an = float((grads[gname] * R).sum())
        assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-3), (name, fd, an)


def test_first_position_closed_form(oracle_lib):
    """O_0 = SiLU(q_0 . k_0 + rab_pos[L-1] + rab_time[0]) / N * v_0 per head."""
    inp = small_inputs(lengths=(8, 5), norm="fixed", norm_len=13)
    got = oracle_lib.fwd(inp)
    H, dv = inp.q.shape[1], inp.v.shape[2]
    L = inp.rab_pos_len
    for b in range(2):
        t = int(inp.offsets[b])
        for h in range(H):
            s = float((inp.q[t, h].double() * inp.k[t, h].double()).sum())
            s += float(inp.rab_pos[h, L - 1]) + float(inp.rab_time[h, 0])
            a = s / (1.0 + math.exp(-s)) / 13.0
            expect = a * inp.v[t, h].double().numpy()
            np.testing.assert_allclose(got["o"][t, h * dv:(h + 1) * dv], expect,
                                       rtol=1e-13, atol=1e-15)


def test_first_position_closed_form_own_length(oracle_lib):
    """With the normaliser taken as each sequence's own length (the jagged
    workload's reading of the model card's division by the length),
    O_0 = SiLU(q_0 . k_0 + rab_pos[L-1] + rab_time[0]) / n_b * v_0."""
    inp = small_inputs(lengths=(8, 5), norm="own")
    got = oracle_lib.fwd(inp)
    H, dv = inp.q.shape[1], inp.v.shape[2]
    L = inp.rab_pos_len
    for b, n in enumerate(inp.lengths):
        t = int(inp.offsets[b])
        for h in range(H):
            s = float((inp.q[t, h].double() * inp.k[t, h].double()).sum())
            s += float(inp.rab_pos[h, L - 1]) + float(inp.rab_time[h, 0])
            expect = s / (1.0 + math.exp(-s)) / n * inp.v[t, h].double().numpy()
            np.testing.assert_allclose(got["o"][t, h * dv:(h + 1) * dv], expect,
                                       rtol=1e-13, atol=1e-15)


def test_query_row_locality(oracle_lib):
    """q_i enters only row i's scores (S_ij = q_i . k_j), so changing it changes
    row i of Y and no other row, bit for bit."""
    base = small_inputs(lengths=(9,), H=2)
    y0 = oracle_lib.fwd(base)["y"]
    i = 4
    pert = small_inputs(lengths=(9,), H=2)
    pert.q[i] = pert.q[i] * -2.0 + 0.5
    y1 = oracle_lib.fwd(pert)["y"]
    rows = [r for r in range(9) if r != i]
    assert np.array_equal(y1[rows], y0[rows])
    assert not np.array_equal(y1[i], y0[i])


def test_gate_limits(oracle_lib):
    """SiLU(40) = 40 to within 1e-16 relative and SiLU(-40) is below 2e-16, so
    with U = +40 the output is 40 x_hat and with U = -40 it vanishes; x_hat is
    taken from the returned O, mean and rstd."""
    for uval in (40.0, -40.0):
        inp = small_inputs()
        inp.u = torch.full_like(inp.u, uval)
        got = oracle_lib.fwd(inp)
        xhat = (got["o"] - got["mean"][:, None]) * got["rstd"][:, None]
        if uval > 0:
            np.testing.assert_allclose(got["y"], 40.0 * xhat, rtol=1e-14, atol=1e-14)
        else:
            assert np.abs(got["y"]).max() <= 2e-16 * max(np.abs(xhat).max(), 1.0)


def test_causality(oracle_lib):
    inp = small_inputs(lengths=(12,), H=2)
    base = oracle_lib.fwd(inp)["y"]
    i = 5
    for name in ("q", "k", "v", "u"):
        pert = small_inputs(lengths=(12,), H=2)
        t = getattr(pert, name)
        t[i + 1:] = t[i + 1:] * -3.0 + 1.0
        if name == "v":
            pert.timestamps[i + 1:] += 10_000_000
        y = oracle_lib.fwd(pert)["y"]
        assert np.array_equal(y[:i + 1], base[:i + 1]), name
        assert not np.array_equal(y[i + 1:], base[i + 1:]), name


def test_linearity_in_v(oracle_lib):
    inp1 = small_inputs(seed=3)
    inp2 = small_inputs(seed=3)
    g = torch.Generator().manual_seed(9)
    inp2.v = torch.randn(inp1.v.shape, generator=g)
    comb = small_inputs(seed=3)
    comb.v = (2.5 * inp1.v.double() - 0.75 * inp2.v.double())
    o1, o2, oc = (oracle_lib.fwd(x)["o"] for x in (inp1, inp2, comb))
    assert rel_err(oc, 2.5 * o1 - 0.75 * o2) < 1e-12


def test_zero_keys_without_bias_give_zero(oracle_lib):
    inp = small_inputs(rab_pos=False, rab_time=False)
    inp.k = torch.zeros_like(inp.k)
    got = oracle_lib.fwd(inp)
    assert np.all(got["o"] == 0.0)
    assert np.all(got["y"] == 0.0)


def test_attention_readout_with_identity_values(oracle_lib):
    """K = 0 and v_j = e_j make O_i[h][:n] row i of A, so each bias index,
    bucket, mask and the normaliser are checked element by element."""
    n, H, L = 7, 2, 9
    inp = small_inputs(lengths=(n,), H=H, dqk=2, dv=n, L=L, norm="fixed", norm_len=5)
    inp.k = torch.zeros_like(inp.k)
    eye = torch.eye(n)
    inp.v = eye[:, None, :].repeat(1, H, 1)
    # distinct, recognisable table entries
    inp.rab_pos = (torch.arange(H * (2 * L - 1), dtype=torch.float32).reshape(H, 2 * L - 1)
                   * 0.01 - 0.3)
    inp.rab_time = (torch.arange(H * 128, dtype=torch.float32).reshape(H, 128) * -0.002 + 0.1)
    ts = inp.timestamps.tolist()
    got = oracle_lib.fwd(inp)["o"]
    for h in range(H):
        for i in range(n):
            for j in range(n):
                val = got[i, h * n + j]
                if j > i:
                    assert val == 0.0
                    continue
                dt = abs(ts[i] - ts[j])
                kb = min(127, int(math.floor(math.log(max(1, dt)) / 0.301)))
                bias = float(inp.rab_pos[h, i - j + L - 1]) + float(inp.rab_time[h, kb])
                expect = bias / (1 + math.exp(-bias)) / 5.0
                assert abs(val - expect) <= 1e-15 + 1e-13 * abs(expect)


def test_packing_invariance(oracle_lib):
    inp = small_inputs(lengths=(5, 9, 3), norm="own")
    full = oracle_lib.fwd(inp)
    for b, n in enumerate(inp.lengths):
        s = int(inp.offsets[b])
        one = oracle_lib._Args([0, n], inp.q[s:s + n], inp.k[s:s + n], inp.v[s:s + n],
                               inp.u[s:s + n], inp.timestamps[s:s + n].numpy(),
                               inp.rab_pos, inp.rab_time, 0, inp.rab_pos_len)
        alone = oracle_lib.fwd_raw(one)
        assert np.array_equal(alone["y"], full["y"][s:s + n])


def test_head_permutation(oracle_lib):
    inp = small_inputs(H=3)
    base = oracle_lib.fwd(inp)["y"]
    perm = [2, 0, 1]
    dv = inp.v.shape[2]
    T = inp.total_tokens
    p = small_inputs(H=3)
    p.q, p.k, p.v = inp.q[:, perm], inp.k[:, perm], inp.v[:, perm]
    p.u = inp.u.reshape(T, 3, dv)[:, perm].reshape(T, 3 * dv)
    p.rab_pos, p.rab_time = inp.rab_pos[perm], inp.rab_time[perm]
    y = oracle_lib.fwd(p)["y"].reshape(T, 3, dv)
    assert rel_err(y, base.reshape(T, 3, dv)[:, perm]) < 1e-12


def test_layernorm_rows(oracle_lib):
    inp = small_inputs()
    got = oracle_lib.fwd(inp)
    o = got["o"]
    xhat = (o - got["mean"][:, None]) * got["rstd"][:, None]
    var = o.var(axis=1)
    assert np.abs(xhat.mean(axis=1)).max() < 1e-12
    np.testing.assert_allclose(xhat.var(axis=1), var / (var + 1e-5), rtol=1e-10)


def test_time_bucket_thresholds(oracle_lib):
    """bucket(x) >= k exactly from ceil(exp(0.301 k)) on (integer |dt|)."""
    tb = oracle_lib.time_bucket
    assert tb(0) == 0 and tb(1) == 0 and tb(-1) == 0
    assert tb(2) == 2 and tb(-2) == 2      # ln 2 / 0.301 = 2.30
    assert tb(3) == 3                       # ln 3 / 0.301 = 3.65
    assert tb(300) == 18                    # ln 300 / 0.301 = 18.95
    assert tb(10 ** 17) == 127 and tb(-(2 ** 63)) == 127 and tb(2 ** 63 - 1) == 127
    for kk in range(1, 128):
        x = math.exp(0.301 * kk)
        lo = math.ceil(x)
        if lo > 2 ** 52 or abs(lo - x) < 1e-9 * x or abs(lo - 1 - x) < 1e-9 * x:
            continue
        assert tb(lo) >= kk and tb(lo - 1) < kk, kk
        assert tb(-lo) >= kk and tb(1 - lo) < kk
    # and on a sweep of small values the bucket is the count of thresholds passed
    for x in range(0, 5000, 7):
        assert tb(x) == sum(1 for kk in range(1, 128) if max(1, x) >= math.exp(0.301 * kk))
    assert tb(4, num_buckets=3) == 2


def test_workload_shapes_follow_model_card():
    """The Neurarch-shaped workload matches the model card's block:
    embed 512 = 4 heads x 128, attention width 128, 1024 input tokens."""
    import json, os
    fx = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "model_card_shapes.json")))
    w = hi.WORKLOADS["neurarch"]
    assert w.heads == fx["num_heads"] and w.d_v == fx["linear_dim"] and w.d_qk == fx["attn_dim"]
    assert w.heads * w.d_v == fx["embed_dim"] and w.seq_len == fx["input_tokens"]


def test_golden_regression(oracle_lib):
    """Values written by tests/golden/make_golden.py (which calls only the
    oracle) still come out of the oracle, so an unintended change shows."""
    import json, os
    fx = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")))
    inp = hi.make_inputs(hi.Spec(**fx["spec"]), seed=fx["seed"])
    got = oracle_lib.fwd(inp)
    np.testing.assert_allclose(got["y"][fx["rows"]], np.array(fx["y_rows"]), rtol=1e-12,
                               atol=1e-14)
    for dt, kb in fx["buckets"]:
        assert oracle_lib.time_bucket(dt) == kb


def test_layernorm_affine_closed_forms(oracle_lib):
    """With the LayerNorm weight at zero every output is bias * SiLU(U),
    whatever the attention computes; a constant weight c (no bias) scales the
    unit-affine output by c; and the bias gradient is sum_t dY * SiLU(U),
    which involves neither the attention nor the normalisation."""
    inp = small_inputs(lengths=(7, 3), H=2, dqk=4, dv=3, ln_affine=True)
    D = inp.u.shape[1]
    u = inp.u.to(torch.float64).numpy()
    silu_u = u / (1.0 + np.exp(-u))
    beta = inp.ln_bias.to(torch.float64).numpy()
    a = oracle_lib._args_from_inputs(inp, ln_weight=np.zeros(D))
    y0 = oracle_lib.fwd_raw(a)["y"]
    assert np.abs(y0 - beta[None, :] * silu_u).max() <= 1e-14 * max(1.0, np.abs(y0).max())
    unit = oracle_lib.fwd_raw(oracle_lib._args_from_inputs(inp, ln_weight=None, ln_bias=None))
    scaled = oracle_lib.fwd_raw(oracle_lib._args_from_inputs(inp, ln_weight=np.full(D, 2.5),
                                                             ln_bias=None))
    assert rel_err(scaled["y"], 2.5 * unit["y"]) < 1e-14
    g = oracle_lib.bwd(inp)
    dy = inp.dy.to(torch.float64).numpy()
    assert rel_err(g["d_ln_bias"], (dy * silu_u).sum(0)) < 1e-12


# ---------------------------------------------------------------- projections
def _proj_case(T=9, E=16, H=2, dqk=4, dv=3, seed=3):
    rng = np.random.default_rng(seed)
    N = H * (2 * dv + 2 * dqk)
    return dict(x=rng.standard_normal((T, E)), w=rng.standard_normal((N, E)) / 4,
                b=rng.standard_normal(N), H=H, dqk=dqk, dv=dv)


@pytest.mark.parametrize("act", [0, 1])
def test_uvqk_matches_torch(oracle_lib, act):
    """The model card's uvqk(x).split([h dv, h dv, h dqk, h dqk]) (nn.Linear:
    x W^T + b), with the reproduction note's SiLU when act = 1."""
    c = _proj_case()
    got = oracle_lib.uvqk(c["x"], c["w"], c["b"], c["H"], c["dqk"], c["dv"], act)
    P = torch.from_numpy(c["x"]) @ torch.from_numpy(c["w"]).T + torch.from_numpy(c["b"])
    if act:
        P = torch.nn.functional.silu(P)
    Nu, Nq = c["H"] * c["dv"], c["H"] * c["dqk"]
    parts = torch.split(P, [Nu, Nu, Nq, Nq], dim=-1)
    for name, ref in zip("uvqk", parts):
        assert rel_err(got[name], ref.numpy()) < 1e-12, name


def test_uvqk_closed_forms(oracle_lib):
    """Weight rows that are unit vectors copy input columns into the outputs,
    in the split order u, v, q, k; zero weights leave SiLU(bias) on every row."""
    c = _proj_case(T=4, E=32, H=2, dqk=4, dv=3)
    H, dqk, dv = c["H"], c["dqk"], c["dv"]
    N = H * (2 * dv + 2 * dqk)
    w = np.zeros((N, 32))
    for n in range(N):
        w[n, n] = 1.0
    got = oracle_lib.uvqk(c["x"], w, None, H, dqk, dv, 0)
    Nu, Nq = H * dv, H * dqk
    assert np.array_equal(got["u"], c["x"][:, :Nu])
    assert np.array_equal(got["v"], c["x"][:, Nu:2 * Nu])
    assert np.array_equal(got["q"], c["x"][:, 2 * Nu:2 * Nu + Nq])
    assert np.array_equal(got["k"], c["x"][:, 2 * Nu + Nq:N])
    b = c["b"]
    got = oracle_lib.uvqk(c["x"], np.zeros((N, 32)), b, H, dqk, dv, 1)
    silu_b = b / (1.0 + np.exp(-b))
    assert np.allclose(got["q"], np.broadcast_to(silu_b[2 * Nu:2 * Nu + Nq], got["q"].shape),
                       rtol=0, atol=1e-15)


@pytest.mark.parametrize("affine", [False, True])
def test_out_proj_matches_torch(oracle_lib, affine):
    """The model card's norm(x + out(o * silu(u))): nn.Linear then nn.LayerNorm
    over E (here the gated, normalised attention output is y)."""
    rng = np.random.default_rng(5)
    T, E, Dy = 7, 24, 12
    y, x = rng.standard_normal((T, Dy)), rng.standard_normal((T, E))
    w, b = rng.standard_normal((E, Dy)) / 3, rng.standard_normal(E)
    g = 1 + 0.2 * rng.standard_normal(E) if affine else None
    be = 0.3 * rng.standard_normal(E) if affine else None
    got = oracle_lib.out_proj(y, x, w, b, g, be)
    t = lambda a: None if a is None else torch.from_numpy(a)
    r = t(x) + t(y) @ t(w).T + t(b)
    ref = torch.nn.functional.layer_norm(r, (E,), weight=t(g), bias=t(be), eps=1e-5)
    assert rel_err(got["z"], ref.numpy()) < 1e-12
    assert rel_err(got["mean"], r.mean(-1).numpy()) < 1e-12


def test_out_proj_closed_forms(oracle_lib):
    """With no projection weight and no input, every row is the normalised
    bias; the residual alone gives LayerNorm rows of mean 0 and variance
    var/(var + eps)."""
    rng = np.random.default_rng(6)
    T, E, Dy = 5, 16, 8
    b = rng.standard_normal(E)
    got = oracle_lib.out_proj(np.zeros((T, Dy)), np.zeros((T, E)), np.zeros((E, Dy)), b)
    bn = (b - b.mean()) / np.sqrt(b.var() + 1e-5)
    assert np.abs(got["z"] - bn[None, :]).max() < 1e-13
    x = rng.standard_normal((T, E)) * 3
    got = oracle_lib.out_proj(rng.standard_normal((T, Dy)), x, np.zeros((E, Dy)))
    z = got["z"]
    var = x.var(axis=1)
    assert np.abs(z.mean(axis=1)).max() < 1e-13
    assert np.abs(z.var(axis=1) - var / (var + 1e-5)).max() < 1e-12


# ---------------------------------------------------------------- M-FALCON
def cand_case(lengths=(5, 0, 12), counts=(3, 2, 4), H=3, dqk=6, dv=4, rab_pos=True,
              rab_time=True, norm="own", norm_len=0, seed=0, ln_affine=False):
    """Histories from small_inputs (position table long enough for relative
    position n_b) and per-user candidates with request times after the history."""
    hist = small_inputs(lengths=lengths, H=H, dqk=dqk, dv=dv, rab_pos=rab_pos,
                        rab_time=rab_time, norm=norm, norm_len=norm_len, seed=seed,
                        L=max(lengths) + 1, ln_affine=ln_affine, grad=False)
    g = torch.Generator().manual_seed(seed + 50)
    C = sum(counts)
    offs = [0]
    for c in counts:
        offs.append(offs[-1] + c)
    qc = torch.randn(C, H, dqk, generator=g) * 0.7
    kc = torch.randn(C, H, dqk, generator=g) * 0.7
    vc = torch.randn(C, H, dv, generator=g)
    uc = torch.randn(C, H * dv, generator=g)
    cts = None
    if rab_time:
        ho = hist.offsets.tolist()
        cts = []
        for b, c in enumerate(counts):
            last = int(hist.timestamps[ho[b + 1] - 1]) if ho[b + 1] > ho[b] else 1_700_000_000
            cts.append(last + torch.randint(0, 5000, (c,), generator=g).to(torch.int64))
        cts = torch.cat(cts)
    return hi.CandInputs(hist, torch.tensor(offs, dtype=torch.int32), qc, kc, vc, uc, cts)


def history_plus(ci, c):
    """The problem (history of c's user, then c) as one sequence."""
    h = ci.hist
    b = int(np.searchsorted(ci.cand_offsets.numpy(), c, side="right")) - 1
    s, e = int(h.offsets[b]), int(h.offsets[b + 1])
    cat = lambda a, x: torch.cat([a[s:e], x[c:c + 1]])
    ts = None if h.timestamps is None else cat(h.timestamps, ci.cand_ts)
    return hi.Inputs(h.spec, torch.tensor([0, e - s + 1], dtype=torch.int32),
                     cat(h.q, ci.qc), cat(h.k, ci.kc), cat(h.v, ci.vc), cat(h.u, ci.uc), ts,
                     h.rab_pos, h.rab_time, None, h.norm_len, h.rab_pos_len, h.ln_weight,
                     h.ln_bias)


@pytest.mark.parametrize("case", [
    dict(), dict(norm="fixed", norm_len=9), dict(rab_time=False), dict(rab_pos=False),
    dict(ln_affine=True), dict(lengths=(1, 7), counts=(5, 0), H=1),
])
def test_mfalcon_is_the_token_after_the_history(oracle_lib, case):
    """Each candidate's output equals the last row of the causal forward on
    (its user's history, the candidate): position n_b, its own time, the
    normaliser of that sequence (the reading of M-FALCON scoring)."""
    ci = cand_case(**case)
    got = oracle_lib.mfalcon(ci)
    for c in range(ci.total_cands):
        ref = oracle_lib.fwd(history_plus(ci, c))
        assert rel_err(got["o"][c], ref["o"][-1]) < 1e-12
        assert rel_err(got["y"][c], ref["y"][-1]) < 1e-12
        assert abs(got["rstd"][c] - ref["rstd"][-1]) <= 1e-12 * ref["rstd"][-1]


def test_mfalcon_empty_history_closed_form(oracle_lib):
    """With no history a candidate attends to itself only:
    O = SiLU(q.k + rab_pos[L-1] + rab_time[bucket 0]) / N * v, N = 1 (own length)."""
    ci = cand_case(lengths=(0, 4), counts=(3, 1))
    got = oracle_lib.mfalcon(ci)
    h = ci.hist
    L = h.rab_pos_len
    for c in range(3):
        for hh in range(3):
            x = float(ci.qc[c, hh].double() @ ci.kc[c, hh].double())
            x += float(h.rab_pos[hh, L - 1]) + float(h.rab_time[hh, 0])
            silu = x / (1.0 + math.exp(-x))
            want = silu * ci.vc[c, hh].double().numpy()
            np.testing.assert_allclose(got["o"][c, hh * 4:(hh + 1) * 4], want, rtol=1e-13,
                                       atol=1e-15)


def test_mfalcon_candidates_do_not_see_each_other(oracle_lib):
    """Changing one candidate leaves every other candidate's output bitwise
    unchanged, and reordering a user's candidates reorders the outputs."""
    ci = cand_case()
    base = oracle_lib.mfalcon(ci)
    ci2 = cand_case()
    for t in (ci2.qc, ci2.kc, ci2.vc, ci2.uc):
        t[1] += 3.0
    if ci2.cand_ts is not None:
        ci2.cand_ts[1] += 10 ** 6
    pert = oracle_lib.mfalcon(ci2)
    keep = [c for c in range(ci.total_cands) if c != 1]
    assert np.array_equal(base["y"][keep], pert["y"][keep])
    assert not np.array_equal(base["y"][1], pert["y"][1])
    perm = torch.tensor([2, 0, 1, 3, 4, 8, 6, 5, 7])
    ci3 = cand_case()
    ci3.qc, ci3.kc, ci3.vc, ci3.uc = (t[perm] for t in (ci3.qc, ci3.kc, ci3.vc, ci3.uc))
    ci3.cand_ts = ci3.cand_ts[perm]
    got = oracle_lib.mfalcon(ci3)
    assert np.array_equal(got["y"], base["y"][perm.numpy()])
