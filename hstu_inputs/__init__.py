"""Seeded synthetic inputs for HSTU causal pointwise aggregated attention.

This module only draws random numbers and rounds them to the run's dtype.  It
holds none of the attention arithmetic, so both the fp64 oracle (``oracle/``)
and the CUDA path (``pointwise_attention_b200``) may use it without sharing
any of the method's code.

Shapes follow the HSTU model card ("HSTU (Generative Recommender)", Structure
table and Exported PyTorch: embed 512, 4 heads, d_qk = d_v = 128, 1024 tokens)
and the named workloads below.  Every draw comes from one CPU
``torch.Generator`` seeded per workload, in a fixed order:

    lengths [-> Stochastic Length draws] -> Q -> K -> V -> U -> timestamps
    -> rab_pos -> rab_time -> dY [-> LayerNorm weight -> LayerNorm bias]

Floating values are drawn in fp32 with ``randn`` and rounded (round to nearest
even) to bf16 for the bf16 workloads; the same rounded host tensors feed the
oracle (widened exactly to fp64) and the GPU.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import torch

__all__ = ["Spec", "Inputs", "WORKLOADS", "make_inputs", "workload", "causal_flops",
           "stochastic_length", "stochastic_length_rows", "ProjInputs", "make_proj_inputs",
           "CandInputs", "make_cand_inputs", "CAND_WORKLOADS"]

NUM_TIME_BUCKETS = 128
TIME_T0 = 1_700_000_000      # first timestamp of every sequence (seconds)
TIME_GAP_MEAN = 300.0        # mean of the exponential gaps between events (seconds)


@dataclasses.dataclass(frozen=True)
class Spec:
    """Shape and distribution of one synthetic workload."""
    name: str
    dtype: str                      # "f32" or "bf16"
    batch: int
    heads: int
    d_qk: int
    d_v: int
    seq_len: int = 0                # dense: every sequence has this length
    len_range: Optional[tuple] = None   # jagged: inclusive (lo, hi) uniform integer lengths
    lengths: Optional[tuple] = None     # explicit lengths (tests)
    qk_std: float = 1.0
    vu_std: float = 1.0
    rab_pos_len: int = 0            # L of the position table [H, 2L-1]; 0 = no position bias
    rab_time: bool = False          # per-head [H, 128] time-bucket table + int64 timestamps
    rab_std: float = 0.02
    norm: str = "fixed"             # "fixed": divide by norm_len; "own": each sequence's length
    norm_len: int = 0               # for "fixed"; 0 means the (dense) sequence length
    grad: bool = False              # also draw the upstream gradient dY
    ts_sorted: bool = True          # timestamps increasing within a sequence
    # Stochastic Length: (keep_len, prob).  Each drawn length above keep_len
    # is cut to keep_len with probability prob (see stochastic_length).
    stochastic_length: Optional[tuple] = None
    # LayerNorm affine over the D = H*d_v features: weight 1 + N(0, 0.1^2) and
    # bias N(0, 0.1^2), drawn last; False: no tables (unit affine).
    ln_affine: bool = False


def _spec_table() -> Dict[str, Spec]:
    s = 1.0 / math.sqrt(128.0)
    return {
        # Tiny fp32 forward: 2 x 64 tokens, 2 heads, d = 32, no relative bias.
        "tiny": Spec("tiny", "f32", batch=2, heads=2, d_qk=32, d_v=32, seq_len=64),
        # Shape of the model card's block: 8 x 1024 tokens, 4 heads, d = 128.
        "neurarch": Spec("neurarch", "bf16", batch=8, heads=4, d_qk=128, d_v=128,
                         seq_len=1024, qk_std=s, rab_pos_len=1024),
        # 64 jagged sequences of 256..4096 tokens with position and time bias.
        "jagged": Spec("jagged", "bf16", batch=64, heads=8, d_qk=128, d_v=128,
                       len_range=(256, 4096), qk_std=s, rab_pos_len=4096,
                       rab_time=True, norm="own"),
        # 4 x 8192 tokens with position and time bias; the position table must
        # reach i - j = 8191, so it holds 2 * 8192 - 1 entries.
        "long": Spec("long", "bf16", batch=4, heads=4, d_qk=128, d_v=128, seq_len=8192,
                     qk_std=s, rab_pos_len=8192, rab_time=True),
        # Training step: 16 x 2048 tokens, position bias, upstream gradient dY.
        "train": Spec("train", "bf16", batch=16, heads=4, d_qk=128, d_v=128, seq_len=2048,
                      qk_std=s, rab_pos_len=2048, grad=True),
        # The training step with the time bias as well: timestamps as in the
        # jagged and long workloads, and the backward of both bias tables.
        "train_time": Spec("train_time", "bf16", batch=16, heads=4, d_qk=128, d_v=128,
                           seq_len=2048, qk_std=s, rab_pos_len=2048, rab_time=True, grad=True),
        # Training step on jagged histories shortened by Stochastic Length:
        # lengths U{256..4096}, histories above 2048 events cut to their
        # latest 2048 with probability 1/2; position and time bias.
        "train_sl": Spec("train_sl", "bf16", batch=16, heads=4, d_qk=128, d_v=128,
                         len_range=(256, 4096), qk_std=s, rab_pos_len=4096, rab_time=True,
                         norm="own", grad=True, stochastic_length=(2048, 0.5)),
    }


WORKLOADS: Dict[str, Spec] = _spec_table()


def workload(name: str, **overrides) -> Spec:
    """Named workload, optionally with fields replaced (smaller batch, other lengths...)."""
    return dataclasses.replace(WORKLOADS[name], **overrides)


@dataclasses.dataclass
class Inputs:
    """Host (CPU) tensors of one problem, already rounded to the run dtype."""
    spec: Spec
    offsets: torch.Tensor           # int32 [B+1]
    q: torch.Tensor                 # [T, H, d_qk]
    k: torch.Tensor                 # [T, H, d_qk]
    v: torch.Tensor                 # [T, H, d_v]
    u: torch.Tensor                 # [T, H*d_v]
    timestamps: Optional[torch.Tensor]  # int64 [T]
    rab_pos: Optional[torch.Tensor]     # fp32 [H, 2L-1]
    rab_time: Optional[torch.Tensor]    # fp32 [H, 128]
    dy: Optional[torch.Tensor]          # [T, H*d_v]
    norm_len: int                   # >0: divide by it; 0: by each sequence's length
    rab_pos_len: int                # L (0 if no position table)
    ln_weight: Optional[torch.Tensor] = None   # fp32 [H*d_v] or None (unit affine)
    ln_bias: Optional[torch.Tensor] = None     # fp32 [H*d_v] or None

    @property
    def lengths(self) -> List[int]:
        o = self.offsets.tolist()
        return [o[i + 1] - o[i] for i in range(len(o) - 1)]

    @property
    def total_tokens(self) -> int:
        return int(self.offsets[-1])

    @property
    def max_seq_len(self) -> int:
        ls = self.lengths
        return max(ls) if ls else 0


def _torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def causal_flops(lengths: Sequence[int], heads: int, d_qk: int, d_v: int) -> int:
    """Algorithmic forward FLOPs: 2 * sum n(n+1)/2 * H * (d_qk + d_v)."""
    pairs = sum(n * (n + 1) // 2 for n in lengths)
    return 2 * pairs * heads * (d_qk + d_v)


def wide_time_span(inp: "Inputs", how: str) -> "Inputs":
    """Timestamps whose differences reach 2^31 s and beyond, for the kernels'
    64-bit time paths: "wide" scales every gap of each sequence by 2e7 (gaps of
    minutes become gaps of decades), "jump" adds 3e9 s to the second half of
    each sequence.  Sorted order is kept; inp is changed in place and returned."""
    ts = inp.timestamps.clone()
    off = inp.offsets.tolist()
    for b in range(len(off) - 1):
        s, e = off[b], off[b + 1]
        if e - s < 2:
            continue
        if how == "wide":
            ts[s:e] = TIME_T0 + (ts[s:e] - ts[s]) * 20_000_000
        elif how == "jump":
            ts[s + (e - s) // 2:e] += 3_000_000_000
        else:
            raise ValueError(how)
    inp.timestamps = ts
    return inp


def stochastic_length(lengths: Sequence[int], keep_len: int, prob: float,
                      generator: torch.Generator) -> List[int]:
    """Stochastic Length ("HSTU Hierarchical Sequential Transduction Units",
    §6 Why it works: long user histories are randomly shortened during
    training).  The page gives no formula; the reading taken here: every
    history longer than ``keep_len`` events is, with probability ``prob``,
    cut to its latest ``keep_len`` events (a contiguous suffix, so order and
    timestamps stay increasing); shorter histories are kept whole.  One
    uniform draw per sequence, in sequence order, from ``generator``."""
    if keep_len < 0 or not (0.0 <= prob <= 1.0):
        raise ValueError("keep_len must be >= 0 and prob in [0, 1]")
    draws = torch.rand(len(lengths), generator=generator, dtype=torch.float64).tolist()
    return [keep_len if (n > keep_len and r < prob) else int(n)
            for n, r in zip(lengths, draws)]


def stochastic_length_rows(offsets: Sequence[int], new_lengths: Sequence[int]):
    """Packed-token rows that a shortening keeps: for sequence b, its last
    new_lengths[b] tokens.  Returns (new int32 offsets [B+1], int64 rows),
    so that a packed tensor x becomes x[rows]."""
    offs = [int(o) for o in offsets]
    if len(offs) != len(new_lengths) + 1:
        raise ValueError("offsets must have one entry more than new_lengths")
    rows, new_offs = [], [0]
    for b, m in enumerate(new_lengths):
        s, e = offs[b], offs[b + 1]
        if not (0 <= m <= e - s):
            raise ValueError("sequence %d: kept length %d outside [0, %d]" % (b, m, e - s))
        rows.extend(range(e - m, e))
        new_offs.append(new_offs[-1] + m)
    return (torch.tensor(new_offs, dtype=torch.int32),
            torch.tensor(rows, dtype=torch.int64))


def make_inputs(spec: Spec, seed: int = 0) -> Inputs:
    """Draw one problem for ``spec`` from a CPU generator seeded with ``seed``."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    # lengths
    if spec.lengths is not None:
        lengths = [int(x) for x in spec.lengths]
    elif spec.len_range is not None:
        lo, hi = spec.len_range
        lengths = torch.randint(lo, hi + 1, (spec.batch,), generator=g).tolist()
    else:
        lengths = [spec.seq_len] * spec.batch
    if spec.stochastic_length is not None:
        keep_len, prob = spec.stochastic_length
        lengths = stochastic_length(lengths, int(keep_len), float(prob), g)
    offs = [0]
    for n in lengths:
        offs.append(offs[-1] + n)
    offsets = torch.tensor(offs, dtype=torch.int32)
    T, H = offs[-1], spec.heads
    dt = _torch_dtype(spec.dtype)

    def draw(shape, std):
        return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(dt)

    q = draw((T, H, spec.d_qk), spec.qk_std)
    k = draw((T, H, spec.d_qk), spec.qk_std)
    v = draw((T, H, spec.d_v), spec.vu_std)
    u = draw((T, H * spec.d_v), spec.vu_std)

    ts = None
    if spec.rab_time:
        parts = []
        for n in lengths:
            gaps = torch.empty(max(n - 1, 0), dtype=torch.float64).exponential_(
                1.0 / TIME_GAP_MEAN, generator=g)
            gaps = torch.clamp(torch.round(gaps), min=1.0).to(torch.int64)
            seq = torch.empty(n, dtype=torch.int64)
            if n:
                seq[0] = TIME_T0
                seq[1:] = TIME_T0 + torch.cumsum(gaps, 0)
            if not spec.ts_sorted and n:
                seq = seq[torch.randperm(n, generator=g)]
            parts.append(seq)
        ts = torch.cat(parts) if parts else torch.empty(0, dtype=torch.int64)

    L = spec.rab_pos_len
    rab_pos = None
    if L > 0:
        rab_pos = torch.randn((H, 2 * L - 1), generator=g, dtype=torch.float32) * spec.rab_std
    rab_time = None
    if spec.rab_time:
        rab_time = torch.randn((H, NUM_TIME_BUCKETS), generator=g,
                               dtype=torch.float32) * spec.rab_std
    dy = draw((T, H * spec.d_v), 1.0) if spec.grad else None
    ln_weight = ln_bias = None
    if spec.ln_affine:
        D = H * spec.d_v
        ln_weight = 1.0 + 0.1 * torch.randn(D, generator=g, dtype=torch.float32)
        ln_bias = 0.1 * torch.randn(D, generator=g, dtype=torch.float32)

    if spec.norm == "own":
        norm_len = 0
    else:
        norm_len = spec.norm_len if spec.norm_len > 0 else (spec.seq_len or max(lengths or [1]))
    return Inputs(spec, offsets, q, k, v, u, ts, rab_pos, rab_time, dy, norm_len, L,
                  ln_weight, ln_bias)


@dataclasses.dataclass
class ProjInputs:
    """Host tensors of the two projections around one HSTU layer's attention.

    x [T, E] layer input (already normalised; bf16), w_uvqk [H(2dv+2dqk), E]
    and b_uvqk [N]; y [T, H dv] an attention output (bf16), w_out [E, H dv],
    b_out [E], ln_weight, ln_bias [E] (fp32)."""
    T: int
    E: int
    H: int
    d_qk: int
    d_v: int
    x: torch.Tensor
    w_uvqk: torch.Tensor
    b_uvqk: torch.Tensor
    y: torch.Tensor
    w_out: torch.Tensor
    b_out: torch.Tensor
    ln_weight: torch.Tensor
    ln_bias: torch.Tensor


def make_proj_inputs(T: int, E: int = 512, H: int = 4, d_qk: int = 128, d_v: int = 128,
                     seed: int = 0) -> ProjInputs:
    """Seeded projection inputs, drawn in the order x, w_uvqk, b_uvqk, y, w_out,
    b_out, ln_weight, ln_bias.  Weights are randn / sqrt(fan_in) (the scale of a
    default-initialised linear layer), biases 0.1 randn, the LayerNorm weight
    1 + 0.1 randn; matrices are rounded to bf16."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    bf = torch.bfloat16
    N = 2 * H * d_v + 2 * H * d_qk
    D = H * d_v
    x = torch.randn(T, E, generator=g).to(bf)
    w_uvqk = (torch.randn(N, E, generator=g) / math.sqrt(E)).to(bf)
    b_uvqk = 0.1 * torch.randn(N, generator=g)
    y = torch.randn(T, D, generator=g).to(bf)
    w_out = (torch.randn(E, D, generator=g) / math.sqrt(D)).to(bf)
    b_out = 0.1 * torch.randn(E, generator=g)
    ln_weight = 1.0 + 0.1 * torch.randn(E, generator=g)
    ln_bias = 0.1 * torch.randn(E, generator=g)
    return ProjInputs(T, E, H, d_qk, d_v, x, w_uvqk, b_uvqk, y, w_out, b_out, ln_weight,
                      ln_bias)


@dataclasses.dataclass
class CandInputs:
    """Candidate scoring against cached histories (M-FALCON).

    ``hist`` holds the users' histories as an ordinary problem (its k, v and
    timestamps are the cached keys, values and event times; its q and u are
    drawn but unused).  Candidates of user b are rows cand_offsets[b] ..
    cand_offsets[b+1]-1 of qc, kc [C, H, d_qk], vc [C, H, d_v], uc [C, H*d_v],
    with request timestamps cand_ts [C] (None without a time table)."""
    hist: Inputs
    cand_offsets: torch.Tensor      # int32 [B+1]
    qc: torch.Tensor
    kc: torch.Tensor
    vc: torch.Tensor
    uc: torch.Tensor
    cand_ts: Optional[torch.Tensor]

    @property
    def counts(self) -> List[int]:
        o = self.cand_offsets.tolist()
        return [o[i + 1] - o[i] for i in range(len(o) - 1)]

    @property
    def total_cands(self) -> int:
        return int(self.cand_offsets[-1])


def make_cand_inputs(spec: Spec, cands, seed: int = 0) -> CandInputs:
    """History from ``make_inputs(spec, seed)``; then, from a second generator
    seeded with seed + 7919, per user a candidate count (``cands`` an int, or
    an inclusive (lo, hi) range drawn uniformly), qc, kc, vc, uc with the
    spec's distributions, and request times: each candidate of user b at
    (last history time) + max(1, round(Exp(mean 300 s))), the history's
    first time when it is empty."""
    hist = make_inputs(spec, seed)
    g = torch.Generator(device="cpu").manual_seed(seed + 7919)
    B, H = spec.batch, spec.heads
    if isinstance(cands, int):
        counts = [cands] * B
    else:
        lo, hi = cands
        counts = torch.randint(lo, hi + 1, (B,), generator=g).tolist()
    offs = [0]
    for c in counts:
        offs.append(offs[-1] + c)
    C = offs[-1]
    dt = _torch_dtype(spec.dtype)

    def draw(shape, std):
        return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(dt)

    qc = draw((C, H, spec.d_qk), spec.qk_std)
    kc = draw((C, H, spec.d_qk), spec.qk_std)
    vc = draw((C, H, spec.d_v), spec.vu_std)
    uc = draw((C, H * spec.d_v), spec.vu_std)
    cand_ts = None
    if spec.rab_time:
        parts = []
        ho = hist.offsets.tolist()
        for b, c in enumerate(counts):
            last = int(hist.timestamps[ho[b + 1] - 1]) if ho[b + 1] > ho[b] else TIME_T0
            gaps = torch.empty(c, dtype=torch.float64).exponential_(1.0 / TIME_GAP_MEAN,
                                                                    generator=g)
            parts.append(last + torch.clamp(torch.round(gaps), min=1.0).to(torch.int64))
        cand_ts = torch.cat(parts) if parts else torch.empty(0, dtype=torch.int64)
    return CandInputs(hist, torch.tensor(offs, dtype=torch.int32), qc, kc, vc, uc, cand_ts)


# Candidate-scoring workloads: (history spec, candidates per user).
#   mfalcon: 32 users with histories of U{256..4096} events (as the jagged
#   workload: 8 heads, position and time bias, own-length normaliser), 512
#   candidates each; the position table reaches relative position 4096.
CAND_WORKLOADS = {
    "mfalcon": (Spec("mfalcon", "bf16", batch=32, heads=8, d_qk=128, d_v=128,
                     len_range=(256, 4096), qk_std=1.0 / math.sqrt(128.0), rab_pos_len=4097,
                     rab_time=True, norm="own"), 512),
}
