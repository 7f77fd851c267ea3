"""fp64 CPU oracle for padding-aware sigmoid attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline (and its ``--impl reference`` arm) may import this package.  The
product path (``padding_aware_sigmoid_b200``) never imports it, and this
package imports nothing from the product path.

The arithmetic lives in ``sigattn_oracle.c`` (plain loops, double precision,
OpenMP over independent rows).  This module only compiles it with gcc and
marshals numpy arrays.  Every function follows the definitions cited there:

* forward: gist.science summary, section 2.A (sigmoid attention formula) and
  paper.rainbus.top summary, method steps (1)-(3) (padding semantics);
* backward: paper.rainbus.top summary, method step (4) (dS, dQ and the
  transposed dK/dV view).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force, library special cases, finite differences,
invariants and the hand-worked golden example under ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "sigattn_oracle.c")
_LIB = os.path.join(_HERE, "_sigattn_oracle.so")
_lock = threading.Lock()
_default = None

DTYPE_BF16 = 0
DTYPE_FP32 = 1


def build(force: bool = False, src: str = SOURCE, out: str = _LIB) -> str:
    """Compile the oracle shared library (gcc, -O2, OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
               "-ffp-contract=off", src, "-o", out, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def _as_raw(t) -> tuple[np.ndarray, int]:
    """Return a contiguous numpy view of the stored bits and the dtype code.

    Accepts numpy float32 arrays, numpy uint16 arrays holding bf16 bits, or CPU
    torch tensors (bf16 / fp32); bf16 stays bf16 so the oracle widens the exact
    stored values itself.
    """
    if hasattr(t, "detach"):  # torch tensor
        import torch
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), DTYPE_BF16
        if t.dtype == torch.float32:
            return t.numpy(), DTYPE_FP32
        raise TypeError(f"oracle takes bf16 or fp32 tensors, got {t.dtype}")
    a = np.ascontiguousarray(t)
    if a.dtype == np.uint16:
        return a, DTYPE_BF16
    if a.dtype == np.float32:
        return a, DTYPE_FP32
    raise TypeError(f"oracle takes float32 or bf16-bit (uint16) arrays, got {a.dtype}")


def _common(q, k, v, dout, seqlens_q, seqlens_k):
    qa, dt = _as_raw(q)
    ka, dt_k = _as_raw(k)
    va, dt_v = _as_raw(v)
    if not (dt == dt_k == dt_v):
        raise TypeError("q, k, v must share one dtype")
    da = None
    if dout is not None:
        da, dt_o = _as_raw(dout)
        if dt_o != dt:
            raise TypeError("dout must share the dtype of q")
    # q (and dout) are [Z, Lq, H, D]; k and v are [Z, Lk, H, D]
    if qa.ndim != 4 or ka.ndim != 4 or ka.shape != va.shape:
        raise ValueError("q, k, v must be [Z, L, H, D]; k and v of one shape")
    if qa.shape[0] != ka.shape[0] or qa.shape[2:] != ka.shape[2:]:
        raise ValueError("q and k must agree in Z, H and D")
    if da is not None and da.shape != qa.shape:
        raise ValueError("dout must match q's shape")
    Z, Lq, H, D = (int(s) for s in qa.shape)
    Lk = int(ka.shape[1])
    nq = np.ascontiguousarray(np.asarray(seqlens_q, dtype=np.int32).reshape(-1))
    nk = np.ascontiguousarray(np.asarray(seqlens_k, dtype=np.int32).reshape(-1))
    if nq.shape[0] != Z or nk.shape[0] != Z:
        raise ValueError("seqlens must have Z entries")
    return qa, ka, va, da, dt, (Z, Lq, Lk, H, D), nq, nk


def _items(items) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(items, dtype=np.int64).reshape(-1, 3))


def _vp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _p(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _bias(bias, Z: int) -> np.ndarray:
    """The bias as one float64 per sample: a scalar is broadcast to every sample."""
    b = np.asarray(bias, dtype=np.float64)
    if b.ndim == 0:
        return np.full(Z, float(b), dtype=np.float64)
    b = np.ascontiguousarray(b.reshape(-1))
    if b.shape[0] != Z:
        raise ValueError(f"bias has {b.shape[0]} entries, expected {Z}")
    return b


class OracleLib:
    """One loaded build of the oracle.  The module-level functions use the
    default build; tests may load a deliberately altered copy to show that the
    pins reject it."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        vp, i32p, i64p, f64p = (ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32),
                                ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double))
        ci, cd, c64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.oracle_sigmoid.argtypes = [cd]
        lib.oracle_sigmoid.restype = cd
        lib.oracle_sigmoid_grad.argtypes = [cd]
        lib.oracle_sigmoid_grad.restype = cd
        lib.oracle_fwd_rows.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, i32p, i32p, cd, f64p,
                                        i64p, c64, f64p]
        lib.oracle_dq_rows.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, i32p, i32p, cd, f64p,
                                       i64p, c64, f64p]
        lib.oracle_dkdv_rows.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, i32p, i32p, cd,
                                         f64p, i64p, c64, f64p, f64p]
        lib.oracle_dbias.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, i32p, i32p, cd, f64p,
                                     f64p, f64p]
        lib.oracle_num_threads.restype = ci
        self.lib = lib
        self.path = path

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def sigmoid(self, x: float) -> float:
        """Exact logistic function sigma(x) = 1 / (1 + e^-x) in double."""
        return float(self.lib.oracle_sigmoid(float(x)))

    def sigmoid_grad(self, x: float) -> float:
        """sigma'(x) = sigma(x) (1 - sigma(x))."""
        return float(self.lib.oracle_sigmoid_grad(float(x)))

    def fwd_rows(self, q, k, v, seqlens_q, seqlens_k, alpha, bias, items) -> np.ndarray:
        """O rows for the (z, h, i) triples in ``items``; returns float64 [n, D]."""
        qa, ka, va, _, dt, (Z, Lq, Lk, H, D), nq, nk = _common(q, k, v, None, seqlens_q, seqlens_k)
        it = _items(items)
        out = np.zeros((it.shape[0], D), dtype=np.float64)
        bz = _bias(bias, Z)
        self.lib.oracle_fwd_rows(_vp(qa), _vp(ka), _vp(va), dt, Z, Lq, Lk, H, D,
                                 _p(nq, ctypes.c_int32), _p(nk, ctypes.c_int32),
                                 float(alpha), _p(bz, ctypes.c_double), _p(it, ctypes.c_int64),
                                 it.shape[0], _p(out, ctypes.c_double))
        return out

    def dq_rows(self, q, k, v, dout, seqlens_q, seqlens_k, alpha, bias, items) -> np.ndarray:
        """dQ rows for the (z, h, i) triples in ``items``; float64 [n, D]."""
        qa, ka, va, da, dt, (Z, Lq, Lk, H, D), nq, nk = _common(q, k, v, dout, seqlens_q, seqlens_k)
        it = _items(items)
        out = np.zeros((it.shape[0], D), dtype=np.float64)
        bz = _bias(bias, Z)
        self.lib.oracle_dq_rows(_vp(qa), _vp(ka), _vp(va), _vp(da), dt, Z, Lq, Lk, H, D,
                                _p(nq, ctypes.c_int32), _p(nk, ctypes.c_int32),
                                float(alpha), _p(bz, ctypes.c_double), _p(it, ctypes.c_int64),
                                it.shape[0], _p(out, ctypes.c_double))
        return out

    def dkdv_rows(self, q, k, v, dout, seqlens_q, seqlens_k, alpha, bias, items):
        """(dK rows, dV rows) for the (z, h, j) key triples in ``items``; float64 [n, D] each."""
        qa, ka, va, da, dt, (Z, Lq, Lk, H, D), nq, nk = _common(q, k, v, dout, seqlens_q, seqlens_k)
        it = _items(items)
        dk = np.zeros((it.shape[0], D), dtype=np.float64)
        dv = np.zeros((it.shape[0], D), dtype=np.float64)
        bz = _bias(bias, Z)
        self.lib.oracle_dkdv_rows(_vp(qa), _vp(ka), _vp(va), _vp(da), dt, Z, Lq, Lk, H, D,
                                  _p(nq, ctypes.c_int32), _p(nk, ctypes.c_int32),
                                  float(alpha), _p(bz, ctypes.c_double), _p(it, ctypes.c_int64),
                                  it.shape[0], _p(dk, ctypes.c_double), _p(dv, ctypes.c_double))
        return dk, dv

    def fwd(self, q, k, v, seqlens_q, seqlens_k, alpha, bias) -> np.ndarray:
        """Full forward O as float64 [Z, Lq, H, D]."""
        Z, Lq, H, D = (int(s) for s in q.shape)
        rows = self.fwd_rows(q, k, v, seqlens_q, seqlens_k, alpha, bias, all_rows(Z, Lq, H))
        return rows.reshape(Z, Lq, H, D)

    def dbias(self, q, k, v, dout, seqlens_q, seqlens_k, alpha, bias) -> np.ndarray:
        """Bias gradient per sample, float64 [Z]: db_z = sum over heads and valid
        (i, j) of dS_ij (paperlayer.ai summary, section 3; gist.science summary,
        section 2.A: x = alpha q.k + b, so dx/db = 1)."""
        qa, ka, va, da, dt, (Z, Lq, Lk, H, D), nq, nk = _common(q, k, v, dout, seqlens_q, seqlens_k)
        bz = _bias(bias, Z)
        rowsum = np.zeros(Z * H * Lq, dtype=np.float64)
        out = np.zeros(Z, dtype=np.float64)
        self.lib.oracle_dbias(_vp(qa), _vp(ka), _vp(va), _vp(da), dt, Z, Lq, Lk, H, D,
                              _p(nq, ctypes.c_int32), _p(nk, ctypes.c_int32), float(alpha),
                              _p(bz, ctypes.c_double), _p(rowsum, ctypes.c_double),
                              _p(out, ctypes.c_double))
        return out

    def bwd(self, q, k, v, dout, seqlens_q, seqlens_k, alpha, bias):
        """Full backward: dQ as float64 [Z, Lq, H, D], dK and dV as [Z, Lk, H, D]."""
        Z, Lq, H, D = (int(s) for s in q.shape)
        Lk = int(k.shape[1])
        dq = self.dq_rows(q, k, v, dout, seqlens_q, seqlens_k, alpha, bias, all_rows(Z, Lq, H))
        dk, dv = self.dkdv_rows(q, k, v, dout, seqlens_q, seqlens_k, alpha, bias,
                                all_rows(Z, Lk, H))
        return (dq.reshape(Z, Lq, H, D), dk.reshape(Z, Lk, H, D), dv.reshape(Z, Lk, H, D))


def default() -> OracleLib:
    """The oracle built from ``sigattn_oracle.c`` in this directory."""
    global _default
    with _lock:
        if _default is None:
            _default = OracleLib(build())
    return _default


def all_rows(Z: int, L: int, H: int) -> np.ndarray:
    """Every (z, h, row) triple, in [Z][L][H] order (matches the tensor layout)."""
    z, l, h = np.meshgrid(np.arange(Z), np.arange(L), np.arange(H), indexing="ij")
    return np.stack([z.ravel(), h.ravel(), l.ravel()], axis=1).astype(np.int64)


def num_threads() -> int:
    return default().num_threads()


def sigmoid(x: float) -> float:
    return default().sigmoid(x)


def sigmoid_grad(x: float) -> float:
    return default().sigmoid_grad(x)


def fwd_rows(*a, **kw):
    return default().fwd_rows(*a, **kw)


def dq_rows(*a, **kw):
    return default().dq_rows(*a, **kw)


def dkdv_rows(*a, **kw):
    return default().dkdv_rows(*a, **kw)


def dbias(*a, **kw):
    return default().dbias(*a, **kw)


def fwd(*a, **kw):
    return default().fwd(*a, **kw)


def bwd(*a, **kw):
    return default().bwd(*a, **kw)
