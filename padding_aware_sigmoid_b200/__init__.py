"""Padding-aware bidirectional sigmoid self-attention for NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libsigattn.so`` (C ABI in ``include/sigattn.h``).
PyTorch supplies device memory and the current CUDA stream; every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback:
calling any op without the built library or without a CUDA device raises.

    O = sigma(alpha Q K^T + b) V   (keys >= n_k masked, query rows >= n_q zero)

Tensors are [Z, L, H, D] (batch, padded length, heads, head dim), contiguous,
bf16 (tensor-core path) or fp32 (accuracy path); ``seqlens_q`` / ``seqlens_k``
are int32 [Z] on the same device.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "SigattnError", "fwd", "bwd", "sigmoid_eval", "set_sigmoid_mode", "get_sigmoid_mode",
    "last_device_status", "set_wait_timeout_ns", "selftest_wait_timeout", "status_string",
    "version", "library_path", "load_library", "SIGMOID_TANH", "SIGMOID_EXP", "EXPORTS",
    "SigmoidAttention", "bwd_dq", "bwd_dkdv", "last_cuda_error", "fwd_noalloc", "NOALLOC_MAX_Z",
    "fwd_bias", "bwd_bias", "dbias_workspace_bytes", "fwd_rect", "bwd_rect", "fwd_bwd_host",
    "fwd_bwd_host_workspace_bytes", "launch_order", "log_length_bias",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsigattn.so")
_lock = threading.Lock()
_lib = None

SIGMOID_TANH = 0
SIGMOID_EXP = 1
_BF16, _FP32 = 0, 1

STATUS_NAMES = {
    0: "SIGATTN_OK", 1: "SIGATTN_ERR_INVALID_ARG", 2: "SIGATTN_ERR_UNSUPPORTED_HEADDIM",
    3: "SIGATTN_ERR_UNSUPPORTED_DTYPE", 4: "SIGATTN_ERR_UNSUPPORTED_DEVICE",
    5: "SIGATTN_ERR_MISALIGNED", 6: "SIGATTN_ERR_CUDA", 7: "SIGATTN_ERR_TIMEOUT",
    8: "SIGATTN_ERR_SEQLEN_RANGE", 9: "SIGATTN_ERR_TOO_LARGE",
}

NOALLOC_MAX_Z = 8192   # SIGATTN_NOALLOC_MAX_Z

# every symbol include/sigattn.h declares
EXPORTS = (
    "sigattn_fwd", "sigattn_bwd", "sigattn_bwd_dq", "sigattn_bwd_dkdv",
    "sigattn_set_sigmoid_mode", "sigattn_get_sigmoid_mode", "sigattn_sigmoid_eval",
    "sigattn_last_device_status", "sigattn_set_wait_timeout_ns", "sigattn_selftest_wait_timeout",
    "sigattn_last_cuda_error", "sigattn_status_string", "sigattn_version",
    "sigattn_fwd_noalloc", "sigattn_fwd_bias", "sigattn_bwd_bias", "sigattn_dbias_workspace_bytes",
    "sigattn_fwd_rect", "sigattn_bwd_rect", "sigattn_fwd_bwd_host",
    "sigattn_fwd_bwd_host_workspace_bytes", "sigattn_launch_order", "sigattn_log_length_bias",
)


class SigattnError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str = ""):
        self.code = int(code)
        msg = f"{where}: {STATUS_NAMES.get(self.code, self.code)}"
        super().__init__(msg + (f" ({detail})" if detail else ""))


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Loads libsigattn.so (built in-tree by ``padding_aware_sigmoid_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libsigattn.so is not built ({_LIB_PATH}); run "
                              "`python -m padding_aware_sigmoid_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, ci, cf, i64, u64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64,
                                ctypes.c_uint64)
        lib.sigattn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, cf, ci, vp]
        lib.sigattn_fwd.restype = ci
        lib.sigattn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, cf,
                                    ci, vp]
        lib.sigattn_bwd.restype = ci
        lib.sigattn_bwd_dq.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, cf, ci, vp]
        lib.sigattn_bwd_dq.restype = ci
        lib.sigattn_bwd_dkdv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, cf,
                                         ci, vp]
        lib.sigattn_bwd_dkdv.restype = ci
        lib.sigattn_fwd_bwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                             cf, cf, ci, vp, ctypes.c_size_t, vp]
        lib.sigattn_fwd_bwd_host.restype = ci
        lib.sigattn_fwd_bwd_host_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
        lib.sigattn_fwd_bwd_host_workspace_bytes.restype = ctypes.c_size_t
        lib.sigattn_fwd_rect.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, cf, ci, vp]
        lib.sigattn_fwd_rect.restype = ci
        lib.sigattn_bwd_rect.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf,
                                         cf, ci, vp]
        lib.sigattn_bwd_rect.restype = ci
        lib.sigattn_fwd_bias.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, vp, ci, vp]
        lib.sigattn_fwd_bias.restype = ci
        lib.sigattn_bwd_bias.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, cf,
                                         vp, vp, vp, ctypes.c_size_t, ci, vp]
        lib.sigattn_bwd_bias.restype = ci
        lib.sigattn_dbias_workspace_bytes.argtypes = [ci, ci, ci, ci]
        lib.sigattn_dbias_workspace_bytes.restype = ctypes.c_size_t
        lib.sigattn_last_cuda_error.restype = ctypes.c_char_p
        lib.sigattn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, cf, ci, vp]
        lib.sigattn_fwd_noalloc.restype = ci
        lib.sigattn_set_sigmoid_mode.argtypes = [ci]
        lib.sigattn_set_sigmoid_mode.restype = ci
        lib.sigattn_get_sigmoid_mode.restype = ci
        lib.sigattn_sigmoid_eval.argtypes = [vp, vp, vp, i64, ci, vp]
        lib.sigattn_sigmoid_eval.restype = ci
        lib.sigattn_last_device_status.argtypes = [vp]
        lib.sigattn_last_device_status.restype = ci
        lib.sigattn_set_wait_timeout_ns.argtypes = [u64]
        lib.sigattn_set_wait_timeout_ns.restype = ci
        lib.sigattn_selftest_wait_timeout.argtypes = [u64, vp]
        lib.sigattn_selftest_wait_timeout.restype = ci
        lib.sigattn_status_string.argtypes = [ci]
        lib.sigattn_status_string.restype = ctypes.c_char_p
        lib.sigattn_version.restype = ci
        lib.sigattn_log_length_bias.argtypes = [vp, ci, vp, vp]
        lib.sigattn_log_length_bias.restype = ci
        lib.sigattn_launch_order.argtypes = [vp, ci, vp]
        lib.sigattn_launch_order.restype = ci
        _lib = lib
        return lib


def _check(code: int, where: str):
    if code != 0:
        detail = last_cuda_error() if code == 6 else ""
        raise SigattnError(code, where, detail)


def _stream_ptr(t) -> int:
    """Raw handle of the current stream on t's device (what torch.cuda.current_stream
    returns, without building a Stream object on every call)."""
    import torch
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:
        return raw(t.get_device())
    return torch.cuda.current_stream(t.device).cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return _BF16
    if t.dtype == torch.float32:
        return _FP32
    raise TypeError(f"sigattn takes bf16 or fp32 tensors, got {t.dtype}")


def _check_inputs(tensors, seqlens):
    import torch
    ref = tensors[0]
    shape, dtype, device = ref.shape, ref.dtype, ref.device
    if len(shape) != 4:
        raise ValueError("tensors must be [Z, L, H, D]")
    if not ref.is_cuda:
        raise ValueError("sigattn tensors must live on a CUDA device (no CPU fallback)")
    for t in tensors:
        if t is not ref and (t.shape != shape or t.dtype != dtype or t.device != device):
            raise ValueError("all tensors must share shape, dtype and device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [Z, L, H, D]")
    for s in seqlens:
        if not (s.device == device and s.dtype == torch.int32 and s.dim() == 1
                and s.shape[0] == shape[0] and s.is_contiguous()):
            raise ValueError("seqlens must be contiguous int32 [Z] tensors on the tensors' device")


def fwd(q, k, v, seqlens_q, seqlens_k, alpha: float, bias: float, out=None):
    """O = [i < n_q] sum_{j < n_k} sigma(alpha q_i . k_j + bias) v_j, [Z, L, H, D]."""
    import torch
    _check_inputs([q, k, v], [seqlens_q, seqlens_k])
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_inputs([q, out], [])
    Z, L, H, D = (int(s) for s in q.shape)
    lib = load_library()
    _check(lib.sigattn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           seqlens_q.data_ptr(), seqlens_k.data_ptr(), Z, L, H, D, float(alpha),
                           float(bias), _dtype_code(q), _stream_ptr(q)), "sigattn_fwd")
    return out


def bwd(q, k, v, dout, seqlens_q, seqlens_k, alpha: float, bias: float, dq=None, dk=None,
        dv=None):
    """(dQ, dK, dV) given dout = dLoss/dO; P is recomputed, O is not needed."""
    import torch
    _check_inputs([q, k, v, dout], [seqlens_q, seqlens_k])
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_inputs([q, dq, dk, dv], [])
    Z, L, H, D = (int(s) for s in q.shape)
    lib = load_library()
    _check(lib.sigattn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), seqlens_q.data_ptr(),
                           seqlens_k.data_ptr(), Z, L, H, D, float(alpha), float(bias),
                           _dtype_code(q), _stream_ptr(q)), "sigattn_bwd")
    return dq, dk, dv


def bwd_dq(q, k, v, dout, seqlens_q, seqlens_k, alpha: float, bias: float, dq=None):
    """dQ only (the dQ kernel of the backward)."""
    import torch
    _check_inputs([q, k, v, dout], [seqlens_q, seqlens_k])
    dq = torch.empty_like(q) if dq is None else dq
    _check_inputs([q, dq], [])
    Z, L, H, D = (int(s) for s in q.shape)
    _check(load_library().sigattn_bwd_dq(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dq.data_ptr(),
        seqlens_q.data_ptr(), seqlens_k.data_ptr(), Z, L, H, D, float(alpha), float(bias),
        _dtype_code(q), _stream_ptr(q)), "sigattn_bwd_dq")
    return dq


def bwd_dkdv(q, k, v, dout, seqlens_q, seqlens_k, alpha: float, bias: float, dk=None, dv=None):
    """(dK, dV) only (the dK/dV kernel of the backward)."""
    import torch
    _check_inputs([q, k, v, dout], [seqlens_q, seqlens_k])
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_inputs([q, dk, dv], [])
    Z, L, H, D = (int(s) for s in q.shape)
    _check(load_library().sigattn_bwd_dkdv(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dk.data_ptr(), dv.data_ptr(),
        seqlens_q.data_ptr(), seqlens_k.data_ptr(), Z, L, H, D, float(alpha), float(bias),
        _dtype_code(q), _stream_ptr(q)), "sigattn_bwd_dkdv")
    return dk, dv


def _check_rect(queries, keys, seqlens):
    """Shapes of the rectangular calls: query-side tensors [Z, Lq, H, D] share one
    shape, key-side tensors [Z, Lk, H, D] another, with the same Z, H, D, dtype
    and device."""
    _check_inputs(queries, seqlens)
    _check_inputs(keys, [])
    a, b = queries[0], keys[0]
    if a.shape[0] != b.shape[0] or a.shape[2:] != b.shape[2:] or a.dtype != b.dtype \
            or a.device != b.device:
        raise ValueError("queries and keys must share Z, H, D, dtype and device")


def fwd_rect(q, k, v, seqlens_q, seqlens_k, alpha: float, bias: float, out=None):
    """Forward with q [Z, Lq, H, D] against k, v [Z, Lk, H, D]; O is [Z, Lq, H, D]."""
    import torch
    out = torch.empty_like(q) if out is None else out
    _check_rect([q, out], [k, v], [seqlens_q, seqlens_k])
    Z, Lq, H, D = (int(x) for x in q.shape)
    Lk = int(k.shape[1])
    _check(load_library().sigattn_fwd_rect(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), seqlens_q.data_ptr(),
        seqlens_k.data_ptr(), Z, Lq, Lk, H, D, float(alpha), float(bias), _dtype_code(q),
        _stream_ptr(q)), "sigattn_fwd_rect")
    return out


def bwd_rect(q, k, v, dout, seqlens_q, seqlens_k, alpha: float, bias: float, dq=None, dk=None,
             dv=None):
    """Backward of ``fwd_rect``: dQ [Z, Lq, H, D]; dK, dV [Z, Lk, H, D]."""
    import torch
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_rect([q, dout, dq], [k, v, dk, dv], [seqlens_q, seqlens_k])
    Z, Lq, H, D = (int(x) for x in q.shape)
    Lk = int(k.shape[1])
    _check(load_library().sigattn_bwd_rect(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), seqlens_q.data_ptr(), seqlens_k.data_ptr(), Z, Lq, Lk, H, D, float(alpha),
        float(bias), _dtype_code(q), _stream_ptr(q)), "sigattn_bwd_rect")
    return dq, dk, dv


def fwd_bwd_host_workspace_bytes(Z: int, L: int, H: int, D: int, dtype) -> int:
    import torch
    code = _FP32 if dtype == torch.float32 else _BF16
    return int(load_library().sigattn_fwd_bwd_host_workspace_bytes(int(Z), int(L), int(H),
                                                                    int(D), code))


def fwd_bwd_host(q, k, v, dout, seqlens_q, seqlens_k, alpha: float, bias: float, outs=None,
                 workspace=None, device=None):
    """Forward and backward of a batch held in host memory (CPU tensors, pinned
    for the copies to overlap the compute): returns host (O, dQ, dK, dV).  Lengths
    are host int32 [Z] arrays or CPU tensors.  ``workspace``: a device uint8 tensor
    of at least fwd_bwd_host_workspace_bytes(...) bytes (allocated here when
    omitted).  The work runs on ``device``'s current stream (default: the current
    device) and is complete once that stream has passed it."""
    import numpy as np
    import torch
    tensors = [q, k, v, dout]
    ref = q
    for t in tensors:
        if t.is_cuda or t.shape != ref.shape or t.dtype != ref.dtype or not t.is_contiguous():
            raise ValueError("fwd_bwd_host takes contiguous CPU tensors of one shape and dtype")
    if outs is None:
        outs = [torch.empty_like(ref, pin_memory=ref.is_pinned()) for _ in range(4)]
    nq = np.ascontiguousarray(np.asarray(seqlens_q, dtype=np.int32).reshape(-1))
    nk = np.ascontiguousarray(np.asarray(seqlens_k, dtype=np.int32).reshape(-1))
    Z, L, H, D = (int(x) for x in ref.shape)
    if nq.shape[0] != Z or nk.shape[0] != Z:
        raise ValueError("seqlens must have Z entries")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    need = fwd_bwd_host_workspace_bytes(Z, L, H, D, ref.dtype)
    if workspace is None:
        # kept for later calls: the library's copy streams may still use it after
        # this call returns, so it is never handed back to the allocator
        key = (dev.index, need)
        workspace = _host_workspaces.get(key)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
            _host_workspaces[key] = workspace
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev).cuda_stream
        _check(load_library().sigattn_fwd_bwd_host(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), outs[0].data_ptr(),
            outs[1].data_ptr(), outs[2].data_ptr(), outs[3].data_ptr(),
            nq.ctypes.data, nk.ctypes.data, Z, L, H, D, float(alpha), float(bias),
            _dtype_code(ref), workspace.data_ptr(), workspace.numel(), stream),
            "sigattn_fwd_bwd_host")
    return tuple(outs)


_host_workspaces = {}


def _check_bias(bias, ref):
    import torch
    if not (bias.is_cuda and bias.dtype == torch.float32 and bias.dim() == 1 and
            bias.shape[0] == ref.shape[0] and bias.is_contiguous() and bias.device == ref.device):
        raise ValueError("bias must be a contiguous float32 [Z] tensor on the tensors' device")


def fwd_bias(q, k, v, seqlens_q, seqlens_k, alpha: float, bias, out=None):
    """Forward with one bias per sample: ``bias`` is a float32 [Z] CUDA tensor
    (for example -log(n_z)); otherwise as ``fwd``."""
    import torch
    _check_inputs([q, k, v], [seqlens_q, seqlens_k])
    _check_bias(bias, q)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_inputs([q, out], [])
    Z, L, H, D = (int(s) for s in q.shape)
    _check(load_library().sigattn_fwd_bias(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), seqlens_q.data_ptr(),
        seqlens_k.data_ptr(), Z, L, H, D, float(alpha), bias.data_ptr(), _dtype_code(q),
        _stream_ptr(q)), "sigattn_fwd_bias")
    return out


def log_length_bias(seqlens):
    """b_z = -ln n_z (0 where n_z <= 1) as a float32 [Z] tensor on the lengths'
    device, computed by the library: the pages' per-sample bias for ``fwd_bias``
    and ``bwd_bias``.  ``seqlens``: int32 [Z] CUDA tensor."""
    import torch
    if not (seqlens.is_cuda and seqlens.dtype == torch.int32 and seqlens.is_contiguous()
            and seqlens.dim() == 1):
        raise ValueError("seqlens must be a contiguous int32 [Z] CUDA tensor")
    out = torch.empty(seqlens.shape, dtype=torch.float32, device=seqlens.device)
    _check(load_library().sigattn_log_length_bias(seqlens.data_ptr(), int(seqlens.numel()),
                                                  out.data_ptr(), _stream_ptr(seqlens)),
           "sigattn_log_length_bias")
    return out


def dbias_workspace_bytes(Z: int, L: int, H: int, dtype) -> int:
    """Device workspace bytes ``bwd_bias`` needs to return the bias gradient."""
    import torch
    code = _FP32 if dtype == torch.float32 else _BF16
    return int(load_library().sigattn_dbias_workspace_bytes(int(Z), int(L), int(H), code))


def bwd_bias(q, k, v, dout, seqlens_q, seqlens_k, alpha: float, bias, want_dbias: bool = True,
             dq=None, dk=None, dv=None, workspace=None):
    """(dQ, dK, dV, db) with one bias per sample (``bias``: float32 [Z] CUDA
    tensor); db[z] = sum over heads and valid (i, j) of dS (None when
    ``want_dbias`` is false).  The db workspace is allocated here unless given."""
    import torch
    _check_inputs([q, k, v, dout], [seqlens_q, seqlens_k])
    _check_bias(bias, q)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_inputs([q, dq, dk, dv], [])
    Z, L, H, D = (int(s) for s in q.shape)
    db = None
    ws_ptr, ws_bytes = None, 0
    if want_dbias:
        db = torch.empty(Z, dtype=torch.float32, device=q.device)
        need = dbias_workspace_bytes(Z, L, H, q.dtype)
        if workspace is None:
            workspace = torch.empty(max(need // 4, 1), dtype=torch.float32, device=q.device)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check(load_library().sigattn_bwd_bias(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), seqlens_q.data_ptr(), seqlens_k.data_ptr(), Z, L, H, D, float(alpha),
        bias.data_ptr(), None if db is None else db.data_ptr(), ws_ptr, ws_bytes,
        _dtype_code(q), _stream_ptr(q)), "sigattn_bwd_bias")
    return dq, dk, dv, db


def fwd_noalloc(q, k, v, seqlens_q, seqlens_k, alpha: float, bias: float, out=None):
    """Forward for callers that cannot allocate device memory: the same result as
    ``fwd``, with the lengths given on the host (numpy int32 arrays or CPU
    tensors) and staged in the library's fixed device array instead of any
    allocation (see sigattn_fwd_noalloc in include/sigattn.h).  ``out`` should be
    preallocated by such callers; Z is limited to NOALLOC_MAX_Z."""
    import numpy as np
    import torch
    _check_inputs([q, k, v], [])
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_inputs([q, out], [])
    # private copies: the call reads them on the host before it returns
    nq = np.array(seqlens_q.cpu() if hasattr(seqlens_q, "cpu") else seqlens_q,
                  dtype=np.int32, copy=True).reshape(-1)
    nk = np.array(seqlens_k.cpu() if hasattr(seqlens_k, "cpu") else seqlens_k,
                  dtype=np.int32, copy=True).reshape(-1)
    Z, L, H, D = (int(s) for s in q.shape)
    if nq.shape[0] != Z or nk.shape[0] != Z:
        raise ValueError("seqlens must have Z entries")
    _check(load_library().sigattn_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
        nq.ctypes.data_as(ctypes.c_void_p), nk.ctypes.data_as(ctypes.c_void_p), Z, L, H, D,
        float(alpha), float(bias), _dtype_code(q), _stream_ptr(q)), "sigattn_fwd_noalloc")
    return out


def last_cuda_error() -> str:
    return load_library().sigattn_last_cuda_error().decode()


def sigmoid_eval(x, mode: int):
    """(sigma(x), sigma'(x)) as evaluated in the bf16 kernels' registers (fp32 CUDA x)."""
    import torch
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    dy = torch.empty_like(x)
    _check(load_library().sigattn_sigmoid_eval(x.data_ptr(), y.data_ptr(), dy.data_ptr(),
                                               x.numel(), int(mode), _stream_ptr(x)),
           "sigattn_sigmoid_eval")
    return y, dy


def set_sigmoid_mode(mode: int):
    _check(load_library().sigattn_set_sigmoid_mode(int(mode)), "sigattn_set_sigmoid_mode")


def get_sigmoid_mode() -> int:
    return int(load_library().sigattn_get_sigmoid_mode())


def last_device_status(device=None) -> int:
    """Reads and clears the device status word (synchronises the current stream)."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return int(load_library().sigattn_last_device_status(
            torch.cuda.current_stream(dev).cuda_stream))


def set_wait_timeout_ns(ns: int):
    _check(load_library().sigattn_set_wait_timeout_ns(int(ns)), "sigattn_set_wait_timeout_ns")


def selftest_wait_timeout(ns: int):
    import torch
    _check(load_library().sigattn_selftest_wait_timeout(
        int(ns), torch.cuda.current_stream().cuda_stream), "sigattn_selftest_wait_timeout")


def status_string(code: int) -> str:
    return load_library().sigattn_status_string(int(code)).decode()


def version() -> int:
    return int(load_library().sigattn_version())


def launch_order(work) -> list:
    """Sample index for each launch rank: decreasing work, ties by index (the
    rule the bf16 kernels use to start long samples first)."""
    import numpy as np
    w = np.ascontiguousarray(np.asarray(work, dtype=np.int32))
    order = np.empty(w.shape[0], dtype=np.int32)
    _check(load_library().sigattn_launch_order(w.ctypes.data, int(w.shape[0]),
                                               order.ctypes.data), "sigattn_launch_order")
    return order.tolist()


from .autograd import SigmoidAttention  # noqa: E402  (needs the functions above)
