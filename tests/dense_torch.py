"""Dense torch fp64 restatement of the attention, used only to pin the oracle.

It follows the model card's HSTUBlock.forward ("HSTU (Generative Recommender)",
Exported PyTorch): per head, ``tril(silu(q @ k^T + bias) / N) @ v`` as whole
matrices, then ``F.layer_norm`` over the concatenated heads (with its weight
and bias when given) and the ``* F.silu(u)`` gate.  It is built from library primitives (matmul, tril,
layer_norm, autograd) rather than the oracle's scalar loops, so agreement
between the two checks each against the other.
"""
import math

import torch
import torch.nn.functional as F


def bucket_matrix(ts_seq: torch.Tensor, num_buckets: int) -> torch.Tensor:
    """Time buckets of all pairs of one sequence, written with exp thresholds.

    bucket(dt) = k  iff  exp(0.301 k) <= max(1,|dt|) < exp(0.301 (k+1))  (capped);
    counted here as the number of k in 1..NB-1 whose threshold is <= |dt|.
    """
    dt = (ts_seq[:, None] - ts_seq[None, :]).abs().to(torch.float64).clamp(min=1.0)
    thr = torch.exp(0.301 * torch.arange(1, num_buckets, dtype=torch.float64))
    # ln(x)/0.301 >= k  <=>  x >= exp(0.301 k); count thresholds passed.
    return (dt[..., None] >= thr).sum(-1)


def dense_forward(offsets, q, k, v, u, ts=None, rab_pos=None, rab_time=None,
                  norm_len=0, eps=1e-5, return_o=False, ln_weight=None, ln_bias=None):
    """All inputs fp64 torch tensors (may require grad). Returns Y [T, D] (and O)."""
    T, H, dqk = q.shape
    dv = v.shape[-1]
    outs = []
    offs = [int(x) for x in offsets]
    L = (rab_pos.shape[-1] + 1) // 2 if rab_pos is not None else 0
    for b in range(len(offs) - 1):
        s, e = offs[b], offs[b + 1]
        n = e - s
        if n == 0:
            continue
        Nn = float(norm_len) if norm_len > 0 else float(n)
        qb = q[s:e].transpose(0, 1)            # [H, n, d]
        kb = k[s:e].transpose(0, 1)
        vb = v[s:e].transpose(0, 1)
        S = qb @ kb.transpose(-1, -2)          # [H, n, n]
        ii = torch.arange(n)[:, None]
        jj = torch.arange(n)[None, :]
        if rab_pos is not None:
            idx = (ii - jj + L - 1).clamp(0, 2 * L - 2)
            S = S + rab_pos[:, idx]
        if rab_time is not None:
            bk = bucket_matrix(ts[s:e], rab_time.shape[-1])
            S = S + rab_time[:, bk]
        A = torch.tril(F.silu(S) / Nn)
        outs.append((A @ vb).transpose(0, 1).reshape(n, H * dv))
    O = torch.cat(outs, 0) if outs else torch.zeros(0, H * dv, dtype=q.dtype)
    Y = F.layer_norm(O, (H * dv,), weight=ln_weight, bias=ln_bias, eps=eps) * F.silu(u)
    return (Y, O) if return_o else Y
