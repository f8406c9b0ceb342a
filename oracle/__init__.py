"""fp64 CPU oracle for HSTU causal pointwise aggregated attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It wraps the plain C
oracle ``hstu_ref.c`` (fp64, fixed summation order, OpenMP over rows) through
ctypes and shares no code with the CUDA library.

Inputs are the rounded host tensors from ``hstu_inputs``; they are widened
exactly to fp64 before the call, so input rounding is not counted as error.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_ref.c")
_LIB = os.path.join(_HERE, "libhstu_ref.so")
_lib = None

LN_EPS = 1e-5
NUM_TIME_BUCKETS = 128


def compile_source(src: str, out: str) -> str:
    """Compile one C source of the oracle (hstu_ref.h found beside this file)."""
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC",
                           "-shared", "-Wall", "-I", _HERE, "-o", out, src, "-lm"])
    return out


def build(force: bool = False) -> str:
    """Compile hstu_ref.c into libhstu_ref.so beside it (gcc, OpenMP)."""
    hdr = os.path.join(_HERE, "hstu_ref.h")
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(hdr))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + ".tmp%d" % os.getpid()
        compile_source(_SRC, tmp)
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("d_qk", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("offsets", ctypes.c_void_p),
        ("timestamps", ctypes.c_void_p),
        ("rab_pos", ctypes.c_void_p),
        ("rab_pos_len", ctypes.c_int32),
        ("rab_time", ctypes.c_void_p),
        ("num_time_buckets", ctypes.c_int32),
        ("norm_len", ctypes.c_int32),
        ("ln_eps", ctypes.c_double),
        ("ln_weight", ctypes.c_void_p),
        ("ln_bias", ctypes.c_void_p),
    ]


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(_Problem)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.hstu_ref_time_bucket.argtypes = [ctypes.c_int64, ctypes.c_int32]
    lib.hstu_ref_time_bucket.restype = ctypes.c_int32
    lib.hstu_ref_fwd.argtypes = [P] + [vp] * 8 + [i32]
    lib.hstu_ref_fwd.restype = ctypes.c_int
    lib.hstu_ref_fwd_rows.argtypes = [P] + [vp] * 5 + [i64] + [vp] * 4 + [i32]
    lib.hstu_ref_fwd_rows.restype = ctypes.c_int
    lib.hstu_ref_bwd.argtypes = [P] + [vp] * 13 + [i32]
    lib.hstu_ref_bwd.restype = ctypes.c_int
    lib.hstu_ref_uvqk.argtypes = [i64] + [ctypes.c_int32] * 5 + [vp] * 7
    lib.hstu_ref_uvqk.restype = ctypes.c_int
    lib.hstu_ref_out.argtypes = [i64, ctypes.c_int32, ctypes.c_int32] + [vp] * 6 + [
        ctypes.c_double] + [vp] * 3
    lib.hstu_ref_out.restype = ctypes.c_int
    lib.hstu_ref_mfalcon.argtypes = [P] + [vp] * 12 + [i32]
    lib.hstu_ref_mfalcon.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


@contextlib.contextmanager
def library(path: str):
    """Route every call of this module to another build of the oracle (for the
    tests that plant a mistake in a copy of hstu_ref.c and check that the pins
    reject it); the regular library is restored on exit."""
    global _lib
    prev = _load()
    _lib = _bind(path)
    try:
        yield
    finally:
        _lib = prev


def _f64(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class _Args:
    """Keeps the fp64 copies alive while the C call runs."""

    def __init__(self, offsets, q, k, v, u, timestamps=None, rab_pos=None, rab_time=None,
                 norm_len=0, rab_pos_len=0, ln_eps=LN_EPS, ln_weight=None, ln_bias=None):
        self.offsets = np.ascontiguousarray(np.asarray(offsets), dtype=np.int32)
        self.q, self.k, self.v, self.u = _f64(q), _f64(k), _f64(v), _f64(u)
        T = int(self.offsets[-1])
        self.H = self.q.shape[1] if self.q.ndim == 3 else 1
        self.dqk = self.q.shape[-1]
        self.dv = self.v.shape[-1]
        self.T = T
        self.D = self.H * self.dv
        self.ts = None if timestamps is None else np.ascontiguousarray(
            np.asarray(timestamps), dtype=np.int64)
        self.rab_pos = _f64(rab_pos)
        self.rab_time = _f64(rab_time)
        self.ln_weight = _f64(ln_weight)
        self.ln_bias = _f64(ln_bias)
        if self.rab_pos is not None and rab_pos_len <= 0:
            rab_pos_len = (self.rab_pos.shape[-1] + 1) // 2
        self.prob = _Problem(
            batch=len(self.offsets) - 1, num_heads=self.H, d_qk=self.dqk, d_v=self.dv,
            offsets=_ptr(self.offsets), timestamps=_ptr(self.ts), rab_pos=_ptr(self.rab_pos),
            rab_pos_len=int(rab_pos_len), rab_time=_ptr(self.rab_time),
            num_time_buckets=(self.rab_time.shape[-1] if self.rab_time is not None
                              else NUM_TIME_BUCKETS),
            norm_len=int(norm_len), ln_eps=float(ln_eps), ln_weight=_ptr(self.ln_weight),
            ln_bias=_ptr(self.ln_bias))


def _args_from_inputs(inp, **kw):
    kw.setdefault("ln_weight", getattr(inp, "ln_weight", None))
    kw.setdefault("ln_bias", getattr(inp, "ln_bias", None))
    return _Args(inp.offsets.numpy(), inp.q, inp.k, inp.v, inp.u,
                 None if inp.timestamps is None else inp.timestamps.numpy(),
                 inp.rab_pos, inp.rab_time, inp.norm_len, inp.rab_pos_len, **kw)


def time_bucket(dt: int, num_buckets: int = NUM_TIME_BUCKETS) -> int:
    return int(_load().hstu_ref_time_bucket(int(dt), int(num_buckets)))


def fwd_raw(a: _Args, threads: int = 0):
    """Full forward: returns dict y, o [T,D], mean, rstd [T] (fp64)."""
    lib = _load()
    y = np.zeros((a.T, a.D)); o = np.zeros((a.T, a.D))
    mean = np.zeros(a.T); rstd = np.zeros(a.T)
    rc = lib.hstu_ref_fwd(ctypes.byref(a.prob), _ptr(a.q), _ptr(a.k), _ptr(a.v), _ptr(a.u),
                          _ptr(y), _ptr(o), _ptr(mean), _ptr(rstd), int(threads))
    if rc != 0:
        raise ValueError("hstu_ref_fwd rejected the problem (code %d)" % rc)
    return dict(y=y, o=o, mean=mean, rstd=rstd)


def fwd_rows_raw(a: _Args, rows: Sequence[int], threads: int = 0):
    """Forward on selected global token rows; outputs are compact [len(rows), ...]."""
    lib = _load()
    r = np.ascontiguousarray(np.asarray(rows), dtype=np.int64)
    n = len(r)
    y = np.zeros((n, a.D)); o = np.zeros((n, a.D)); mean = np.zeros(n); rstd = np.zeros(n)
    rc = lib.hstu_ref_fwd_rows(ctypes.byref(a.prob), _ptr(a.q), _ptr(a.k), _ptr(a.v),
                               _ptr(a.u), _ptr(r), n, _ptr(y), _ptr(o), _ptr(mean),
                               _ptr(rstd), int(threads))
    if rc != 0:
        raise ValueError("hstu_ref_fwd_rows rejected the problem (code %d)" % rc)
    return dict(y=y, o=o, mean=mean, rstd=rstd)


def bwd_raw(a: _Args, dy, threads: int = 0):
    """Backward: returns dict dq, dk [T,H,dqk], dv [T,H,dv], du [T,D], d_rab_pos,
    d_rab_time, and d_ln_weight, d_ln_bias [D] (those of the unit affine when
    the problem has no LayerNorm tables)."""
    lib = _load()
    dyd = _f64(dy)
    dq = np.zeros((a.T, a.H, a.dqk)); dk = np.zeros((a.T, a.H, a.dqk))
    dv = np.zeros((a.T, a.H, a.dv)); du = np.zeros((a.T, a.D))
    drp = None if a.rab_pos is None else np.zeros_like(a.rab_pos)
    drt = None if a.rab_time is None else np.zeros_like(a.rab_time)
    dlw = np.zeros(a.D); dlb = np.zeros(a.D)
    rc = lib.hstu_ref_bwd(ctypes.byref(a.prob), _ptr(a.q), _ptr(a.k), _ptr(a.v), _ptr(a.u),
                          _ptr(dyd), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(du), _ptr(drp),
                          _ptr(drt), _ptr(dlw), _ptr(dlb), int(threads))
    if rc != 0:
        raise ValueError("hstu_ref_bwd rejected the problem (code %d)" % rc)
    return dict(dq=dq, dk=dk, dv=dv, du=du, d_rab_pos=drp, d_rab_time=drt, d_ln_weight=dlw,
                d_ln_bias=dlb)


def fwd(inp, threads: int = 0):
    """Forward of an ``hstu_inputs.Inputs`` problem."""
    return fwd_raw(_args_from_inputs(inp), threads)


def fwd_rows(inp, rows, threads: int = 0):
    return fwd_rows_raw(_args_from_inputs(inp), rows, threads)


def bwd(inp, threads: int = 0):
    """Backward of an ``hstu_inputs.Inputs`` problem (uses ``inp.dy``)."""
    return bwd_raw(_args_from_inputs(inp), inp.dy, threads)


def uvqk(x, w, b, H: int, dqk: int, dv: int, act: int = 0):
    """UVQK projection of x [T, E] by w [H(2dv+2dqk), E] (+ b): dict u, v, q, k
    ([T, H*dv] twice, [T, H*dqk] twice, fp64)."""
    lib = _load()
    xd, wd, bd = _f64(x), _f64(w), _f64(b)
    T, E = xd.shape
    Nu, Nq = H * dv, H * dqk
    out = dict(u=np.zeros((T, Nu)), v=np.zeros((T, Nu)), q=np.zeros((T, Nq)),
               k=np.zeros((T, Nq)))
    rc = lib.hstu_ref_uvqk(int(T), int(E), int(H), int(dqk), int(dv), int(act), _ptr(xd),
                           _ptr(wd), _ptr(bd), _ptr(out["u"]), _ptr(out["v"]), _ptr(out["q"]),
                           _ptr(out["k"]))
    if rc != 0:
        raise ValueError("hstu_ref_uvqk rejected the sizes (code %d)" % rc)
    return out


def out_proj(y, x, w, b=None, gamma=None, beta=None, eps: float = LN_EPS):
    """Z = LayerNorm_E(x + y w^T + b) (gamma, beta): dict z [T, E], mean, rstd [T]."""
    lib = _load()
    yd, xd, wd = _f64(y), _f64(x), _f64(w)
    bd, gd, btd = _f64(b), _f64(gamma), _f64(beta)
    T, E = xd.shape
    Dy = yd.shape[1]
    z = np.zeros((T, E)); mean = np.zeros(T); rstd = np.zeros(T)
    rc = lib.hstu_ref_out(int(T), int(E), int(Dy), _ptr(yd), _ptr(xd), _ptr(wd), _ptr(bd),
                          _ptr(gd), _ptr(btd), float(eps), _ptr(z), _ptr(mean), _ptr(rstd))
    if rc != 0:
        raise ValueError("hstu_ref_out rejected the sizes (code %d)" % rc)
    return dict(z=z, mean=mean, rstd=rstd)


def mfalcon(ci, threads: int = 0):
    """Candidate scoring (M-FALCON reading: each candidate is the token after
    its user's history, attending to the history and itself only) of an
    ``hstu_inputs.CandInputs``: dict y, o [C, D], mean, rstd [C] (fp64)."""
    lib = _load()
    h = ci.hist
    a = _Args(h.offsets.numpy(), h.k, h.k, h.v, h.u,
              None if h.timestamps is None else h.timestamps.numpy(), h.rab_pos, h.rab_time,
              h.norm_len, h.rab_pos_len, ln_weight=h.ln_weight, ln_bias=h.ln_bias)
    co = np.ascontiguousarray(ci.cand_offsets.numpy(), dtype=np.int32)
    cts = None if ci.cand_ts is None else np.ascontiguousarray(ci.cand_ts.numpy(),
                                                                dtype=np.int64)
    qc, kc, vc, uc = _f64(ci.qc), _f64(ci.kc), _f64(ci.vc), _f64(ci.uc)
    C = int(co[-1])
    y = np.zeros((C, a.D)); o = np.zeros((C, a.D)); mean = np.zeros(C); rstd = np.zeros(C)
    rc = lib.hstu_ref_mfalcon(ctypes.byref(a.prob), _ptr(a.k), _ptr(a.v), _ptr(co), _ptr(cts),
                              _ptr(qc), _ptr(kc), _ptr(vc), _ptr(uc), _ptr(y), _ptr(o),
                              _ptr(mean), _ptr(rstd), int(threads))
    if rc != 0:
        raise ValueError("hstu_ref_mfalcon rejected the problem (code %d)" % rc)
    return dict(y=y, o=o, mean=mean, rstd=rstd)
