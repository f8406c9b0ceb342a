"""ctypes binding of libhstu (include/hstu.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
only checks tensor placement, builds the ``hstu_problem_t`` struct, allocates
outputs and workspace with torch (device memory is plumbing) and forwards
raw pointers.  There is no fallback: if libhstu.so is missing, or a tensor is
not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# HSTU_DEBUG_BOUNDS=1 in the environment selects the build with device-side
# index checks (python -m pointwise_attention_b200.build --debug-bounds).
LIB_PATH = os.path.join(_HERE, "libhstu_debug.so" if os.environ.get("HSTU_DEBUG_BOUNDS") == "1"
                        else "libhstu.so")

HSTU_OK, HSTU_ERR_INVALID_ARG, HSTU_ERR_UNSUPPORTED = 0, 1, 2
HSTU_ERR_CUDA, HSTU_ERR_TIMEOUT, HSTU_ERR_WORKSPACE, HSTU_ERR_BOUNDS = 3, 4, 5, 6
HSTU_F32, HSTU_BF16 = 0, 1

EXPORTED = ("hstu_attn_workspace_size", "hstu_attn_fwd", "hstu_attn_bwd", "hstu_attn_check",
            "hstu_status_string", "hstu_time_bucket_thresholds", "hstu_selftest_wait_timeout",
            "hstu_attn_bwd_noalloc", "hstu_uvqk_fwd", "hstu_out_fwd", "hstu_cand_workspace_size",
            "hstu_cand_fwd")


class HSTUError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__("%s: %s" % (what, status_string(code)))


class hstu_problem_t(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("batch", ctypes.c_int32),
        ("total_tokens", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("d_qk", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("offsets", ctypes.c_void_p),
        ("offsets_host", ctypes.c_void_p),
        ("timestamps", ctypes.c_void_p),
        ("rab_pos", ctypes.c_void_p),
        ("rab_pos_len", ctypes.c_int32),
        ("rab_time", ctypes.c_void_p),
        ("num_time_buckets", ctypes.c_int32),
        ("norm_len", ctypes.c_int32),
        ("ln_eps", ctypes.c_float),
        ("ln_weight", ctypes.c_void_p),
        ("ln_bias", ctypes.c_void_p),
    ]


_lib = None


def load_library():
    """Loads libhstu.so from the package directory (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libhstu.so is not built (%s); run `python -m "
                           "pointwise_attention_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(hstu_problem_t)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.hstu_attn_workspace_size.argtypes = [P, ctypes.c_int]
    lib.hstu_attn_workspace_size.restype = sz
    lib.hstu_attn_fwd.argtypes = [P] + [vp] * 5 + [vp] * 3 + [vp, sz, vp]
    lib.hstu_attn_fwd.restype = ctypes.c_int
    lib.hstu_attn_bwd.argtypes = [P] + [vp] * 5 + [vp] * 3 + [vp] * 4 + [vp] * 4 + [vp, sz, vp]
    lib.hstu_attn_bwd.restype = ctypes.c_int
    lib.hstu_attn_check.argtypes = [vp, vp]
    lib.hstu_attn_check.restype = ctypes.c_int
    lib.hstu_status_string.argtypes = [ctypes.c_int]
    lib.hstu_status_string.restype = ctypes.c_char_p
    lib.hstu_time_bucket_thresholds.argtypes = [vp, ctypes.c_int32]
    lib.hstu_time_bucket_thresholds.restype = ctypes.c_int32
    lib.hstu_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint64, vp]
    lib.hstu_selftest_wait_timeout.restype = ctypes.c_int
    lib.hstu_attn_bwd_noalloc.argtypes = [P] + [vp] * 5 + [vp] * 3 + [vp] * 4 + [vp] * 4 + [vp]
    lib.hstu_attn_bwd_noalloc.restype = ctypes.c_int
    i32 = ctypes.c_int32
    lib.hstu_uvqk_fwd.argtypes = [i32] * 6 + [vp] * 7 + [vp, sz, vp]
    lib.hstu_uvqk_fwd.restype = ctypes.c_int
    lib.hstu_out_fwd.argtypes = [i32] * 3 + [vp] * 6 + [ctypes.c_float] + [vp] * 3 + [vp, sz, vp]
    lib.hstu_out_fwd.restype = ctypes.c_int
    lib.hstu_cand_workspace_size.argtypes = [P, i32, i32]
    lib.hstu_cand_workspace_size.restype = sz
    lib.hstu_cand_fwd.argtypes = [P, vp, vp, vp, i32, i32] + [vp] * 6 + [vp, sz, vp]
    lib.hstu_cand_fwd.restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load_library().hstu_status_string(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError("%s must be a CUDA tensor (the library runs on the GPU only)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must have dtype %s, got %s" % (name, dtype, t.dtype))
    return t


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_problem(q, v, offsets, max_seq_len, timestamps=None, rab_pos=None, rab_time=None,
                 norm_len=0, eps=1e-5, offsets_host=None, ln_weight=None, ln_bias=None):
    """hstu_problem_t for tensors q [T,H,dqk], v [T,H,dv] and int32 offsets [B+1];
    ln_weight, ln_bias: fp32 [H*dv] LayerNorm affine, or None (ones, zeros)."""
    if q.dtype == torch.bfloat16:
        dt = HSTU_BF16
    elif q.dtype == torch.float32:
        dt = HSTU_F32
    else:
        raise ValueError("q must be bf16 or fp32")
    T, H, dqk = q.shape
    p = hstu_problem_t()
    p.dtype = dt
    p.batch = offsets.numel() - 1
    p.total_tokens = T
    p.max_seq_len = int(max_seq_len)
    p.num_heads = H
    p.d_qk = dqk
    p.d_v = v.shape[-1]
    p.offsets = offsets.data_ptr()
    p.offsets_host = None if offsets_host is None else offsets_host.data_ptr()
    p.timestamps = None if timestamps is None else timestamps.data_ptr()
    p.rab_pos = None if rab_pos is None else rab_pos.data_ptr()
    p.rab_pos_len = 0 if rab_pos is None else (rab_pos.shape[-1] + 1) // 2
    p.rab_time = None if rab_time is None else rab_time.data_ptr()
    p.num_time_buckets = 0 if rab_time is None else rab_time.shape[-1]
    p.norm_len = int(norm_len)
    p.ln_eps = float(eps)
    p.ln_weight = None if ln_weight is None else ln_weight.data_ptr()
    p.ln_bias = None if ln_bias is None else ln_bias.data_ptr()
    return p


def hstu_attn_workspace_size(problem: hstu_problem_t, is_bwd: bool = False) -> int:
    return int(load_library().hstu_attn_workspace_size(ctypes.byref(problem), int(bool(is_bwd))))


def new_workspace(problem: hstu_problem_t, is_bwd: bool, device) -> torch.Tensor:
    n = hstu_attn_workspace_size(problem, is_bwd)
    if n == 0:
        raise HSTUError(HSTU_ERR_INVALID_ARG, "hstu_attn_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def hstu_attn_fwd(q, k, v, u, offsets, max_seq_len, *, timestamps=None, rab_pos=None,
                  rab_time=None, norm_len=0, eps=1e-5, ln_weight=None, ln_bias=None,
                  save_for_backward=False, offsets_host=None, y=None, saved=None,
                  workspace=None, stream=None):
    """Forward.  Returns (y, saved) with saved = (o_save, ln_mean, ln_rstd) or None."""
    lib = load_library()
    for name, t in (("q", q), ("k", k), ("v", v), ("u", u)):
        _dev(t, name, q.dtype)
    _dev(offsets, "offsets", torch.int32)
    _dev(timestamps, "timestamps", torch.int64)
    _dev(rab_pos, "rab_pos", torch.float32)
    _dev(rab_time, "rab_time", torch.float32)
    _dev(ln_weight, "ln_weight", torch.float32)
    _dev(ln_bias, "ln_bias", torch.float32)
    T, H, _ = q.shape
    D = H * v.shape[-1]
    p = make_problem(q, v, offsets, max_seq_len, timestamps, rab_pos, rab_time, norm_len, eps,
                     offsets_host, ln_weight, ln_bias)
    if y is None:
        y = torch.empty((T, D), dtype=q.dtype, device=q.device)
    _dev(y, "y", q.dtype)
    if save_for_backward and saved is None:
        saved = (torch.empty((T, D), dtype=torch.float32, device=q.device),
                 torch.empty((T,), dtype=torch.float32, device=q.device),
                 torch.empty((T,), dtype=torch.float32, device=q.device))
    if not save_for_backward:
        saved = None
    if workspace is None:
        workspace = new_workspace(p, False, q.device)
    o_save, mean, rstd = saved if saved is not None else (None, None, None)
    rc = lib.hstu_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(y),
                           _ptr(o_save), _ptr(mean), _ptr(rstd), _ptr(workspace),
                           workspace.numel(), _stream_ptr(stream))
    if rc != HSTU_OK:
        raise HSTUError(rc, "hstu_attn_fwd")
    return y, saved


def hstu_attn_bwd(dy, q, k, v, u, offsets, max_seq_len, saved, *, timestamps=None,
                  rab_pos=None, rab_time=None, norm_len=0, eps=1e-5, ln_weight=None,
                  ln_bias=None, offsets_host=None, need_rab_grads=True, grads=None,
                  workspace=None, stream=None):
    """Backward.  Returns dict dq, dk, dv, du, d_rab_pos, d_rab_time, d_ln_weight,
    d_ln_bias (the table gradients None where the table is absent)."""
    lib = load_library()
    for name, t in (("dy", dy), ("q", q), ("k", k), ("v", v), ("u", u)):
        _dev(t, name, q.dtype)
    _dev(offsets, "offsets", torch.int32)
    o_save, mean, rstd = saved
    for name, t in (("o_save", o_save), ("ln_mean", mean), ("ln_rstd", rstd)):
        _dev(t, name, torch.float32)
    _dev(ln_weight, "ln_weight", torch.float32)
    _dev(ln_bias, "ln_bias", torch.float32)
    p = make_problem(q, v, offsets, max_seq_len, timestamps, rab_pos, rab_time, norm_len, eps,
                     offsets_host, ln_weight, ln_bias)
    if grads is None:
        grads = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                     du=torch.empty_like(u),
                     d_rab_pos=(torch.empty_like(rab_pos)
                                if (rab_pos is not None and need_rab_grads) else None),
                     d_rab_time=(torch.empty_like(rab_time)
                                 if (rab_time is not None and need_rab_grads) else None),
                     d_ln_weight=(torch.empty_like(ln_weight)
                                  if (ln_weight is not None and need_rab_grads) else None),
                     d_ln_bias=(torch.empty_like(ln_bias)
                                if (ln_bias is not None and need_rab_grads) else None))
    grads.setdefault("d_ln_weight", None)
    grads.setdefault("d_ln_bias", None)
    if workspace is None:
        workspace = new_workspace(p, True, q.device)
    rc = lib.hstu_attn_bwd(ctypes.byref(p), _ptr(dy), _ptr(q), _ptr(k), _ptr(v), _ptr(u),
                           _ptr(o_save), _ptr(mean), _ptr(rstd), _ptr(grads["dq"]),
                           _ptr(grads["dk"]), _ptr(grads["dv"]), _ptr(grads["du"]),
                           _ptr(grads["d_rab_pos"]), _ptr(grads["d_rab_time"]),
                           _ptr(grads["d_ln_weight"]), _ptr(grads["d_ln_bias"]),
                           _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if rc != HSTU_OK:
        raise HSTUError(rc, "hstu_attn_bwd")
    return grads


def hstu_attn_check(workspace, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status word."""
    return int(load_library().hstu_attn_check(_ptr(workspace), _stream_ptr(stream)))


def hstu_time_bucket_thresholds(num_buckets: int = 128):
    import numpy as np
    out = np.zeros(max(num_buckets - 1, 1), dtype=np.int64)
    n = load_library().hstu_time_bucket_thresholds(out.ctypes.data_as(ctypes.c_void_p),
                                                   int(num_buckets))
    if n < 0:
        raise HSTUError(HSTU_ERR_INVALID_ARG, "hstu_time_bucket_thresholds")
    return out[:n]


def hstu_selftest_wait_timeout(workspace, budget_ns: int = 50_000_000, stream=None) -> int:
    """Runs the bounded-wait self-test kernel; returns the launch status."""
    return int(load_library().hstu_selftest_wait_timeout(_ptr(workspace), int(budget_ns),
                                                         _stream_ptr(stream)))


def _status_workspace(device):
    return torch.zeros(256, dtype=torch.uint8, device=device)


def hstu_uvqk_fwd(x, w, num_heads: int, d_qk: int, d_v: int, *, bias=None, act: int = 0,
                  out=None, workspace=None, stream=None):
    """UVQK projection act(x w^T + bias) of x [T, E] by w [H(2dv+2dqk), E] (bf16).

    Returns dict u [T, H*dv], v [T, H, dv], q [T, H, dqk], k [T, H, dqk] (bf16)."""
    lib = load_library()
    _dev(x, "x", torch.bfloat16)
    _dev(w, "w", torch.bfloat16)
    _dev(bias, "bias", torch.float32)
    T, E = x.shape
    H = int(num_heads)
    if out is None:
        out = dict(u=torch.empty((T, H * d_v), dtype=x.dtype, device=x.device),
                   v=torch.empty((T, H, d_v), dtype=x.dtype, device=x.device),
                   q=torch.empty((T, H, d_qk), dtype=x.dtype, device=x.device),
                   k=torch.empty((T, H, d_qk), dtype=x.dtype, device=x.device))
    for n in ("u", "v", "q", "k"):
        _dev(out[n], n, x.dtype)
    if workspace is None:
        workspace = _status_workspace(x.device)
    rc = lib.hstu_uvqk_fwd(int(T), int(E), H, int(d_qk), int(d_v), int(act), _ptr(x), _ptr(w),
                           _ptr(bias), _ptr(out["u"]), _ptr(out["v"]), _ptr(out["q"]),
                           _ptr(out["k"]), _ptr(workspace), workspace.numel(),
                           _stream_ptr(stream))
    if rc != HSTU_OK:
        raise HSTUError(rc, "hstu_uvqk_fwd")
    return out


def hstu_out_fwd(y, w, x, *, bias=None, ln_weight=None, ln_bias=None, eps: float = 1e-5,
                 save_stats: bool = False, z=None, workspace=None, stream=None):
    """Z = LayerNorm(x + y w^T + bias) * ln_weight + ln_bias for y [T, D], w [E, D],
    x [T, E] (bf16).  Returns (z, (mean, rstd) or None)."""
    lib = load_library()
    _dev(y, "y", torch.bfloat16)
    _dev(w, "w", torch.bfloat16)
    _dev(x, "x", torch.bfloat16)
    for n, t in (("bias", bias), ("ln_weight", ln_weight), ("ln_bias", ln_bias)):
        _dev(t, n, torch.float32)
    T, D = y.shape
    E = x.shape[1]
    if z is None:
        z = torch.empty((T, E), dtype=x.dtype, device=x.device)
    _dev(z, "z", x.dtype)
    stats = None
    if save_stats:
        stats = (torch.empty(T, dtype=torch.float32, device=x.device),
                 torch.empty(T, dtype=torch.float32, device=x.device))
    if workspace is None:
        workspace = _status_workspace(x.device)
    mean, rstd = stats if stats is not None else (None, None)
    rc = lib.hstu_out_fwd(int(T), int(E), int(D), _ptr(y), _ptr(w), _ptr(x), _ptr(bias),
                          _ptr(ln_weight), _ptr(ln_bias), float(eps), _ptr(z), _ptr(mean),
                          _ptr(rstd), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if rc != HSTU_OK:
        raise HSTUError(rc, "hstu_out_fwd")
    return z, stats


def hstu_cand_fwd(k_hist, v_hist, offsets, max_seq_len, q, k, v, u, cand_offsets,
                  max_cands: int, *, timestamps=None, cand_timestamps=None, rab_pos=None,
                  rab_time=None, norm_len=0, eps=1e-5, ln_weight=None, ln_bias=None,
                  offsets_host=None, y=None, workspace=None, stream=None):
    """Candidate scoring against cached histories (M-FALCON): every candidate
    of user b attends to b's history (k_hist, v_hist [T_h, H, 128], offsets)
    and to itself.  q, k, v [C, H, 128], u [C, H*128] (bf16); cand_offsets
    int32 [B+1].  Returns y [C, H*128]."""
    lib = load_library()
    for name, t in (("k_hist", k_hist), ("v_hist", v_hist), ("q", q), ("k", k), ("v", v),
                    ("u", u)):
        _dev(t, name, torch.bfloat16)
    _dev(offsets, "offsets", torch.int32)
    _dev(cand_offsets, "cand_offsets", torch.int32)
    _dev(timestamps, "timestamps", torch.int64)
    _dev(cand_timestamps, "cand_timestamps", torch.int64)
    for name, t in (("rab_pos", rab_pos), ("rab_time", rab_time), ("ln_weight", ln_weight),
                    ("ln_bias", ln_bias)):
        _dev(t, name, torch.float32)
    p = make_problem(k_hist, v_hist, offsets, max_seq_len, timestamps, rab_pos, rab_time,
                     norm_len, eps, offsets_host, ln_weight, ln_bias)
    C, H, _ = q.shape
    if y is None:
        y = torch.empty((C, H * v.shape[-1]), dtype=q.dtype, device=q.device)
    _dev(y, "y", q.dtype)
    if workspace is None:
        n = int(lib.hstu_cand_workspace_size(ctypes.byref(p), int(C), int(max_cands)))
        if n == 0:
            raise HSTUError(HSTU_ERR_INVALID_ARG, "hstu_cand_workspace_size")
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device)
    rc = lib.hstu_cand_fwd(ctypes.byref(p), _ptr(k_hist), _ptr(v_hist), _ptr(cand_offsets),
                           int(C), int(max_cands), _ptr(cand_timestamps), _ptr(q), _ptr(k),
                           _ptr(v), _ptr(u), _ptr(y), _ptr(workspace), workspace.numel(),
                           _stream_ptr(stream))
    if rc != HSTU_OK:
        raise HSTUError(rc, "hstu_cand_fwd")
    return y
