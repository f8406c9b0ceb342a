"""The oracle's pins reject plausible mistakes.

Each case copies oracle/hstu_ref.c, plants one mistake in the copy (a dropped
term, a wrong sign or index, a transposed operand, a wrong normaliser, an
off-by-one mask or bucket, a missing term of the chain rule), compiles it and
runs the pins of test_oracle.py against it.  At least one pin that neither
restates the formula nor replays the oracle's own stored outputs has to fail:
the closed form of the first position, the invariants (causality, linearity
in V, zero keys, the A read-out, packing, head permutation, LayerNorm rows),
the time-bucket thresholds, or finite differences of the forward against the
backward.  The dense torch restatement, its autograd and the golden
regression values are left out on purpose, so that the oracle is shown to be
pinned by something other than a retyping of its formula or its own earlier
results.  A control compiles the unmodified source the same way and must pass
every pin.

A second set plants each mistake everywhere it can occur, forward and backward
alike, so that the two still agree under finite differences; those mistakes
must fail some other pin.

Nothing here needs a GPU; the planted mistakes live only in temporary copies.
"""
import os

import pytest

import oracle
from tests import test_oracle as T

SRC = os.path.join(os.path.dirname(oracle.__file__), "hstu_ref.c")

# (name, text in hstu_ref.c, replacement, which occurrence: 0 = the first)
MUTANTS = [
    # forward
    ("time bias dropped",
     "bias += p->rab_time[(int64_t)h * p->num_time_buckets + bk];", "(void)bk;", 0),
    ("position index sign",
     "bias += p->rab_pos[(int64_t)h * (2 * L - 1) + (i - j) + L - 1];",
     "bias += p->rab_pos[(int64_t)h * (2 * L - 1) + (j - i) + L - 1];", 0),
    ("diagonal masked out",
     "for (int j = 0; j <= i; ++j) {", "for (int j = 0; j < i; ++j) {", 0),
    ("sigmoid in place of SiLU",
     "double A = ref_silu(S) / Nn;", "double A = ref_sigmoid(S) / Nn;", 0),
    ("own length plus one",
     "double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)n;",
     "double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)(n + 1);", 0),
    ("unbiased LayerNorm variance", "var /= (double)D;", "var /= (double)(D - 1);", 0),
    ("eps outside the square root",
     "double rstd = 1.0 / sqrt(var + p->ln_eps);",
     "double rstd = 1.0 / (sqrt(var) + p->ln_eps);", 0),
    ("mean not subtracted",
     "y_row[c] = ((o_row[c] - mu) * rstd * w + bb) * ref_silu(ur[c]);",
     "y_row[c] = (o_row[c] * rstd * w + bb) * ref_silu(ur[c]);", 0),
    ("gate without SiLU",
     "y_row[c] = ((o_row[c] - mu) * rstd * w + bb) * ref_silu(ur[c]);",
     "y_row[c] = ((o_row[c] - mu) * rstd * w + bb) * ur[c];", 0),
    ("LayerNorm bias scaled by the weight",
     "y_row[c] = ((o_row[c] - mu) * rstd * w + bb) * ref_silu(ur[c]);",
     "y_row[c] = ((o_row[c] - mu) * rstd + bb) * w * ref_silu(ur[c]);", 0),
    ("decimal log in the bucket",
     "double b = floor(log(a) / 0.301);", "double b = floor(log10(a) / 0.301);", 0),
    ("query and key swapped",
     "double S = ref_dot(qi, kj, dqk) + ref_bias(p, h, s, i, j);",
     "double S = ref_dot(q + ((s + j) * H + h) * dqk, k + (t * H + h) * dqk, dqk)"
     " + ref_bias(p, h, s, i, j);", 0),
    # backward
    ("SiLU derivative reduced to sigmoid",
     "return s * (1.0 + x * (1.0 - s));", "return s;", 0),
    ("mean of dxhat dropped",
     "dOr[c] = rstd[t] * (dxh - m1 - xhat * m2);", "dOr[c] = rstd[t] * (dxh - xhat * m2);", 0),
    ("dU without xhat",
     "dur[c] = dyr[c] * (w * xhat + bb) * ref_silu_grad(ur[c]);",
     "dur[c] = dyr[c] * (w + bb) * ref_silu_grad(ur[c]);", 0),
    ("dxhat without the LayerNorm weight",
     "double dxh = dyr[c] * g * w;", "double dxh = dyr[c] * g;", 0),
    ("LayerNorm bias gradient times xhat",
     "if (d_ln_bias) d_ln_bias[c] += dyg;", "if (d_ln_bias) d_ln_bias[c] += dyg * xhat;", 0),
    ("LayerNorm weight gradient without xhat",
     "if (d_ln_weight) d_ln_weight[c] += dyg * xhat;", "if (d_ln_weight) d_ln_weight[c] += dyg;",
     0),
    # projections either side of the attention
    ("UVQK split with v before u",
     "if (n < Nu) u[t * Nu + n] = acc;\n            else if (n < 2 * Nu) v[t * Nu + (n - Nu)] = acc;",
     "if (n < Nu) v[t * Nu + n] = acc;\n            else if (n < 2 * Nu) u[t * Nu + (n - Nu)] = acc;",
     0),
    ("UVQK weight row read in reverse", "for (int c = 0; c < E; ++c) acc += xr[c] * wr[c];",
     "for (int c = 0; c < E; ++c) acc += xr[c] * wr[E - 1 - c];", 0),
    ("output residual dropped", "r[e] = xr[e] + acc + (b ? b[e] : 0.0);",
     "r[e] = acc + (b ? b[e] : 0.0);", 0),
    ("output bias dropped", "r[e] = xr[e] + acc + (b ? b[e] : 0.0);", "r[e] = xr[e] + acc;", 0),
    ("dS without 1/N",
     "double dS = dA * ref_silu_grad(S) / Nn;", "double dS = dA * ref_silu_grad(S);", 0),
    ("dV from dS instead of A",
     "for (int c = 0; c < dvv; ++c) dvj[c] += A * dOi[c];",
     "for (int c = 0; c < dvv; ++c) dvj[c] += dS * dOi[c];", 0),
    ("dK from k instead of q", "dkj[c] += dS * qi[c];", "dkj[c] += dS * kj[c];", 0),
    ("position gradient index sign",
     "if (pp) pp[(i - j) + L - 1] += dS;", "if (pp) pp[(j - i) + L - 1] += dS;", 0),
    ("time gradient one bucket low",
     "tp[bk] += dS;", "tp[bk > 0 ? bk - 1 : 0] += dS;", 0),
    # candidate scoring against a cached history
    ("candidate position one step short",
     "S += p->rab_pos[h * (2 * L - 1) + (n - j) + L - 1];",
     "S += p->rab_pos[h * (2 * L - 1) + (n - 1 - j) + L - 1];", 0),
    ("candidate normaliser without the candidate",
     "const double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)(n + 1);",
     "const double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)(n > 0 ? n : 1);", 0),
    ("candidate self term dropped",
     "for (int e = 0; e < dv; ++e) oh[e] += A * vs[e];", "(void)vs;", 0),
    ("candidate time measured from the first event",
     "cand_ts[c] - p->timestamps[s + j]", "cand_ts[c] - p->timestamps[s]", 0),
    ("candidate self term at relative position 1",
     "if (p->rab_pos) S += p->rab_pos[h * (2 * L - 1) + L - 1];",
     "if (p->rab_pos) S += p->rab_pos[h * (2 * L - 1) + L];", 0),
]

# The same mistake in the forward and the backward: (name, [(text, replacement)]),
# every occurrence of each text replaced.
CONSISTENT_MUTANTS = [
    ("own length plus one",
     [("double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)n;",
       "double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)(n + 1);")]),
    ("query and key swapped",
     [("double S = ref_dot(qi, kj, dqk) + ref_bias(p, h, s, i, j);",
       "double S = ref_dot(q + ((s + j) * H + h) * dqk, k + ((s + i) * H + h) * dqk, dqk)"
       " + ref_bias(p, h, s, i, j);")]),
    ("sigmoid as the SiLU", [("return x / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(-x));")]),
    ("gate without SiLU",
     [("y_row[c] = ((o_row[c] - mu) * rstd * w + bb) * ref_silu(ur[c]);",
       "y_row[c] = ((o_row[c] - mu) * rstd * w + bb) * ur[c];"),
      ("double g = ref_silu(ur[c]);", "double g = ur[c];"),
      ("dur[c] = dyr[c] * (w * xhat + bb) * ref_silu_grad(ur[c]);",
       "dur[c] = dyr[c] * (w * xhat + bb);"),
      ("double dxh = dyr[c] * ref_silu(ur[c]) * w;", "double dxh = dyr[c] * ur[c] * w;"),
      ("double dyg = dyr[c] * ref_silu(ur[c]);", "double dyg = dyr[c] * ur[c];")]),
    ("position index sign",
     [("+ (i - j) + L - 1];", "+ (j - i) + L - 1];"),
      ("if (pp) pp[(i - j) + L - 1] += dS;", "if (pp) pp[(j - i) + L - 1] += dS;")]),
]

# Pins that do not restate the formula (see the module docstring).
PINS = [
    T.test_first_position_closed_form,
    T.test_first_position_closed_form_own_length,
    T.test_query_row_locality,
    T.test_gate_limits,
    T.test_causality,
    T.test_linearity_in_v,
    T.test_zero_keys_without_bias_give_zero,
    T.test_attention_readout_with_identity_values,
    T.test_packing_invariance,
    T.test_head_permutation,
    T.test_layernorm_rows,
    T.test_time_bucket_thresholds,
    T.test_backward_finite_differences,
    T.test_layernorm_affine_closed_forms,
    T.test_uvqk_closed_forms,
    T.test_out_proj_closed_forms,
    T.test_mfalcon_empty_history_closed_form,
    T.test_mfalcon_candidates_do_not_see_each_other,
]


def _mfalcon_history_pin(o):
    for case in ({}, {"norm": "fixed", "norm_len": 9}, {"rab_pos": False}):
        T.test_mfalcon_is_the_token_after_the_history(o, case)


PINS.append(_mfalcon_history_pin)


def _plant(text, old, new, occurrence):
    at = -1
    for _ in range(occurrence + 1):
        at = text.find(old, at + 1)
        assert at >= 0, "hstu_ref.c no longer holds %r" % old
    return text[:at] + new + text[at + len(old):]


def _build(tmp_path, name, text):
    src = tmp_path / (name + ".c")
    src.write_text(text)
    return oracle.compile_source(str(src), str(tmp_path / ("lib" + name + ".so")))


def _failing_pins(lib_path):
    failed = []
    with oracle.library(lib_path):
        for pin in PINS:
            try:
                pin(oracle)
            except AssertionError:
                failed.append(pin.__name__)
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path):
    with open(SRC) as f:
        text = f.read()
    assert _failing_pins(_build(tmp_path, "control", text)) == []


@pytest.mark.parametrize("name,old,new,occurrence", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, name, old, new, occurrence):
    with open(SRC) as f:
        text = f.read()
    mutant = _plant(text, old, new, occurrence)
    assert mutant != text
    failed = _failing_pins(_build(tmp_path, "mutant", mutant))
    assert failed, "no pin rejects the planted mistake: %s" % name


@pytest.mark.parametrize("name,edits", CONSISTENT_MUTANTS, ids=[m[0] for m in CONSISTENT_MUTANTS])
def test_consistent_mistake_fails_a_pin_besides_finite_differences(tmp_path, name, edits):
    with open(SRC) as f:
        text = f.read()
    mutant = text
    for old, new in edits:
        assert old in mutant, "hstu_ref.c no longer holds %r" % old
        mutant = mutant.replace(old, new)
    failed = _failing_pins(_build(tmp_path, "mutant", mutant))
    others = [p for p in failed if p != "test_backward_finite_differences"]
    assert others, "only finite differences reject %s: %s" % (name, failed)
