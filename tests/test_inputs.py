"""The seeded input generator (CPU): determinism, draw order and the
Stochastic Length shortening of histories ("HSTU Hierarchical Sequential
Transduction Units", §6 Why it works)."""
import numpy as np
import pytest
import torch

import hstu_inputs as hi


def test_same_seed_same_problem():
    a = hi.make_inputs(hi.workload("train_sl", batch=6), seed=5)
    b = hi.make_inputs(hi.workload("train_sl", batch=6), seed=5)
    assert a.lengths == b.lengths
    for n in ("q", "k", "v", "u", "timestamps", "rab_pos", "rab_time", "dy"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n
    c = hi.make_inputs(hi.workload("train_sl", batch=6), seed=6)
    assert not torch.equal(a.q, c.q)


def test_stochastic_length_bounds_and_rate():
    g = torch.Generator().manual_seed(0)
    lengths = list(range(1, 4001))
    keep, prob = 1000, 0.3
    out = hi.stochastic_length(lengths, keep, prob, g)
    assert len(out) == len(lengths)
    for n, m in zip(lengths, out):
        if n <= keep:
            assert m == n                      # short histories are kept whole
        else:
            assert m in (n, keep)              # long ones are cut to keep_len or kept
    long_ = [(n, m) for n, m in zip(lengths, out) if n > keep]
    frac = sum(m == keep for _, m in long_) / len(long_)
    # 3000 Bernoulli(0.3) draws: 5 standard deviations is about 0.042
    assert abs(frac - prob) < 0.042


def test_stochastic_length_edge_probabilities():
    g = torch.Generator().manual_seed(1)
    lengths = [10, 500, 2049, 0, 4096]
    assert hi.stochastic_length(lengths, 2048, 0.0, g) == lengths
    assert hi.stochastic_length(lengths, 2048, 1.0, g) == [10, 500, 2048, 0, 2048]
    assert hi.stochastic_length(lengths, 0, 1.0, g) == [0, 0, 0, 0, 0]
    with pytest.raises(ValueError):
        hi.stochastic_length(lengths, 10, 1.5, g)


def test_stochastic_length_is_seeded():
    lengths = [3000] * 50
    a = hi.stochastic_length(lengths, 1024, 0.5, torch.Generator().manual_seed(7))
    b = hi.stochastic_length(lengths, 1024, 0.5, torch.Generator().manual_seed(7))
    c = hi.stochastic_length(lengths, 1024, 0.5, torch.Generator().manual_seed(8))
    assert a == b and a != c


def test_stochastic_length_rows_keep_the_latest_events():
    offsets = [0, 5, 5, 12, 15]
    new_offs, rows = hi.stochastic_length_rows(offsets, [2, 0, 7, 1])
    assert new_offs.tolist() == [0, 2, 2, 9, 10]
    assert rows.tolist() == [3, 4, 5, 6, 7, 8, 9, 10, 11, 14]
    # gathered timestamps stay increasing within each sequence
    ts = torch.arange(15, dtype=torch.int64) * 10
    kept = ts[rows]
    o = new_offs.tolist()
    for b in range(4):
        seg = kept[o[b]:o[b + 1]]
        assert torch.all(seg[1:] > seg[:-1])
    with pytest.raises(ValueError):
        hi.stochastic_length_rows(offsets, [6, 0, 7, 1])


def test_train_sl_workload_lengths():
    inp = hi.make_inputs(hi.WORKLOADS["train_sl"], seed=0)
    spec = inp.spec
    keep, _ = spec.stochastic_length
    lo, hi_ = spec.len_range
    ls = inp.lengths
    assert len(ls) == spec.batch and max(ls) <= spec.rab_pos_len
    # the lengths drawn before shortening, from the same seeded generator
    g = torch.Generator(device="cpu").manual_seed(0)
    drawn = torch.randint(lo, hi_ + 1, (spec.batch,), generator=g).tolist()
    for n, m in zip(drawn, ls):
        assert m == n or (n > keep and m == keep)
    assert any(n > keep and m == keep for n, m in zip(drawn, ls))
    assert inp.q.shape[0] == sum(ls) == inp.timestamps.shape[0]
    t = inp.timestamps.numpy()
    o = inp.offsets.numpy()
    for b in range(spec.batch):
        assert np.all(np.diff(t[o[b]:o[b + 1]]) > 0)


def test_candidate_inputs_follow_their_history():
    sp = hi.workload("jagged", batch=5, len_range=(0, 40), heads=2, rab_pos_len=41)
    a = hi.make_cand_inputs(sp, (0, 6), seed=3)
    b = hi.make_cand_inputs(sp, (0, 6), seed=3)
    assert a.counts == b.counts and torch.equal(a.qc, b.qc) and torch.equal(a.cand_ts, b.cand_ts)
    assert a.qc.shape == (a.total_cands, 2, 128) and a.uc.shape == (a.total_cands, 256)
    ho, co = a.hist.offsets.tolist(), a.cand_offsets.tolist()
    for u in range(5):
        last = int(a.hist.timestamps[ho[u + 1] - 1]) if ho[u + 1] > ho[u] else None
        for c in range(co[u], co[u + 1]):
            if last is not None:
                assert int(a.cand_ts[c]) > last       # requests come after the history
    # the history part is exactly the ordinary problem of the same seed
    h = hi.make_inputs(sp, seed=3)
    assert torch.equal(h.k, a.hist.k) and torch.equal(h.timestamps, a.hist.timestamps)
    spec, n = hi.CAND_WORKLOADS["mfalcon"]
    assert spec.rab_pos_len >= spec.len_range[1] + 1 and n == 512


def test_wide_time_span_keeps_order_and_crosses_2_31():
    sp = hi.Spec("case", "bf16", batch=3, heads=2, d_qk=128, d_v=128, lengths=(300, 1, 150),
                 rab_time=True)
    for how in ("wide", "jump"):
        inp = hi.wide_time_span(hi.make_inputs(sp, seed=2), how)
        off = inp.offsets.tolist()
        ts = inp.timestamps
        for b in range(len(off) - 1):
            seq = ts[off[b]:off[b + 1]]
            assert bool((seq[1:] >= seq[:-1]).all())
            if len(seq) > 1:
                assert int(seq[-1] - seq[0]) >= 2 ** 31
