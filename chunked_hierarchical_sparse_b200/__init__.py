"""Hierarchical Sparse Attention (HSA) for B200 (sm_100a): thin Python binding.

Every function here only marshals arguments to the C ABI of ``libhsa.so``
(declared in ``include/hsa.h``): it checks dtypes and layouts, allocates the
output and workspace tensors with PyTorch (device memory and streams are all
PyTorch is used for), and passes raw device pointers plus the current CUDA
stream.  All arithmetic runs in the library's CUDA kernels; there is no CPU
or PyTorch fallback -- if the library is missing, importing the binding
functions raises.

Layouts (see include/hsa.h): q, o, dO [B, L, h_q, d]; q_slc [B, L, h_kv, d];
k, v [B, h_kv, L, d]; kbar [B, h_kv, L//S, d] fp32; idx/w [B, L, h_kv, K];
lse [B, L, h_q, K].
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["hsa_set_wait_limit_ns", "hsa_timing_enable", "hsa_timing_read", "KERNELS", "hsa_workspace_size", "hsa_pool", "hsa_select", "hsa_fwd", "hsa_attend", "hsa_decode", "hsa_decode_multi", "hsa_bwd",
           "hsa_device_status", "HsaError", "lib_path", "load_library", "OP_POOL", "OP_SELECT",
           "OP_FWD", "OP_DECODE", "OP_BWD"]

_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "libhsa.so")

OP_POOL, OP_SELECT, OP_FWD, OP_DECODE, OP_BWD = range(5)
_F32, _BF16 = 0, 1
# kernel kinds of hsa_timing_read (hsa_kernel_t)
KERNELS = {"pool": 1, "select": 2, "attend_simt": 3, "decode": 4, "bwd1": 5, "invert": 6, "bwd2": 7,
           "attend_tc": 8, "plan": 9,
           "bwd_tc": 10, "bwd_sel": 11}
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace too small",
           4: "CUDA launch or API error", 5: "device wait timed out",
           6: "device-side input check failed"}


class HsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_STATUS.get(code, 'unknown status')} (code {code})")


class HsaShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "L", "h_q", "h_kv", "d", "S", "K", "dtype")]


_lib = None


def load_library():
    """Load ``libhsa.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError(f"{lib_path} is missing: build it with "
                              "`python -m chunked_hierarchical_sparse_b200.build`")
        L = ctypes.CDLL(lib_path)
        P, Z, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        sp = ctypes.POINTER(HsaShape)
        L.hsa_workspace_size.argtypes = [sp, I]
        L.hsa_workspace_size.restype = Z
        L.hsa_pool.argtypes = [sp, P, P, P, Z, P]
        L.hsa_select.argtypes = [sp, P, P, P, P, P, P, Z, P]
        L.hsa_fwd.argtypes = [sp, P, P, P, P, P, P, P, P, P, P, Z, P]
        L.hsa_attend.argtypes = [sp, P, P, P, P, P, P, P, P, Z, P]
        L.hsa_decode.argtypes = [sp, P, P, P, P, P, P, P, P, P, Z, P]
        L.hsa_decode_multi.argtypes = [sp, ctypes.c_int32, P, P, P, P, P, P, P, P, P, Z, P]
        L.hsa_bwd.argtypes = [sp, P, P, P, P, P, P, P, P, P, P, P, P, P, P, Z, P]
        L.hsa_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32), P]
        L.hsa_timing_enable.argtypes = [I]
        L.hsa_timing_read.argtypes = [I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
        L.hsa_timing_enable.restype = ctypes.c_int
        L.hsa_timing_read.restype = ctypes.c_int
        L.hsa_status_string.argtypes = [ctypes.c_int32]
        L.hsa_status_string.restype = ctypes.c_char_p
        L.hsa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.hsa_set_wait_limit_ns.restype = ctypes.c_int
        for f in ("hsa_pool", "hsa_select", "hsa_fwd", "hsa_attend", "hsa_decode", "hsa_decode_multi", "hsa_bwd", "hsa_device_status"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


# ------------------------------------------------------------------ helpers
def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return _F32
    if t.dtype == torch.bfloat16:
        return _BF16
    raise TypeError(f"token tensors must be float32 or bfloat16, got {t.dtype}")


def _need(t: torch.Tensor, name: str, shape, dtype=None, device=None, host_ok=False):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if host_ok and not t.is_cuda:  # an offloaded cache: page-locked host memory the GPU reads directly
        if not t.is_pinned():
            raise ValueError(f"{name}: a host tensor must be page-locked (pin_memory())")
        return
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _run(name: str, dev, stream, *args):
    """Call a C entry point with the tensors' device current, on the given stream or
    else that device's current stream (the library launches on the current device)."""
    if stream is not None and stream.device != dev:
        raise ValueError(f"{name}: the stream is on {stream.device}, the tensors on {dev}")
    fn = getattr(load_library(), name)
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev) if stream is None else stream
        _check(fn(*args, ctypes.c_void_p(s.cuda_stream)), name)


def _check(code: int, where: str):
    if code != 0:
        raise HsaError(code, where)


def hsa_workspace_size(B, L, h_q, h_kv, d, S, K, dtype, op) -> int:
    sh = HsaShape(B, L, h_q, h_kv, d, S, K, _BF16 if dtype == torch.bfloat16 else _F32)
    n = int(load_library().hsa_workspace_size(ctypes.byref(sh), op))
    if n == 0:
        raise HsaError(2, "hsa_workspace_size")
    return n


def _workspace(sh: HsaShape, op: int, device, ws):
    n = int(load_library().hsa_workspace_size(ctypes.byref(sh), op))
    if n == 0:
        raise HsaError(1, "hsa_workspace_size")
    if ws is not None:
        if not isinstance(ws, torch.Tensor) or ws.device != device or not ws.is_contiguous():
            raise ValueError(f"workspace: a contiguous tensor on {device} is required")
        if ws.numel() * ws.element_size() < n:
            raise HsaError(3, "workspace")
        return ws, ws.numel() * ws.element_size()
    buf = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 256
    return buf[off:off + n], n


# ------------------------------------------------------------------ entry points
def hsa_pool(k: torch.Tensor, S: int = 64, kbar=None, ws=None, stream=None) -> torch.Tensor:
    B, h_kv, L, d = k.shape
    _need(k, "k", k.shape)
    sh = HsaShape(B, L, h_kv, h_kv, d, S, 1, _dtype_code(k))
    if kbar is None:
        kbar = torch.empty(B, h_kv, L // S, d, dtype=torch.float32, device=k.device)
    _need(kbar, "kbar", (B, h_kv, L // S, d), torch.float32, k.device)
    w_, n = _workspace(sh, OP_POOL, k.device, ws)
    _run("hsa_pool", k.device, stream, ctypes.byref(sh), _p(k), _p(kbar), _p(w_), n)
    return kbar


def hsa_select(q_slc: torch.Tensor, k: torch.Tensor, K: int, S: int = 64, ws=None, stream=None):
    """Returns (kbar, idx, w)."""
    B, L, h_kv, d = q_slc.shape
    dt = _dtype_code(q_slc)
    _need(q_slc, "q_slc", q_slc.shape, q_slc.dtype)
    _need(k, "k", (B, h_kv, L, d), q_slc.dtype, q_slc.device)
    dev = q_slc.device
    kbar = torch.empty(B, h_kv, L // S, d, dtype=torch.float32, device=dev)
    idx = torch.empty(B, L, h_kv, K, dtype=torch.int32, device=dev)
    w = torch.empty(B, L, h_kv, K, dtype=torch.float32, device=dev)
    sh = HsaShape(B, L, h_kv, h_kv, d, S, K, dt)
    w_, n = _workspace(sh, OP_SELECT, dev, ws)
    _run("hsa_select", dev, stream, ctypes.byref(sh), _p(q_slc), _p(k), _p(kbar), _p(idx), _p(w),
         _p(w_), n)
    return kbar, idx, w


def hsa_fwd(q, k, v, q_slc, K: int, S: int = 64, want_lse: bool = True, want_sel: bool = True,
            o=None, ws=None, stream=None):
    """Forward pass.  Returns (o, lse, idx, w, kbar); lse / idx, w, kbar are None
    when not requested (they then stay in the workspace)."""
    B, L, h_q, d = q.shape
    h_kv = k.shape[1]
    dt, dev = _dtype_code(q), q.device
    _need(q, "q", q.shape, q.dtype)
    _need(k, "k", (B, h_kv, L, d), q.dtype, dev)
    _need(v, "v", (B, h_kv, L, d), q.dtype, dev)
    _need(q_slc, "q_slc", (B, L, h_kv, d), q.dtype, dev)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype, dev)
    lse = torch.empty(B, L, h_q, K, dtype=torch.float32, device=dev) if want_lse else None
    idx = torch.empty(B, L, h_kv, K, dtype=torch.int32, device=dev) if want_sel else None
    w = torch.empty(B, L, h_kv, K, dtype=torch.float32, device=dev) if want_sel else None
    kbar = torch.empty(B, h_kv, L // S, d, dtype=torch.float32, device=dev) if want_sel else None
    sh = HsaShape(B, L, h_q, h_kv, d, S, K, dt)
    w_, n = _workspace(sh, OP_FWD, dev, ws)
    _run("hsa_fwd", dev, stream, ctypes.byref(sh), _p(q), _p(k), _p(v), _p(q_slc), _p(o), _p(lse),
         _p(idx), _p(w), _p(kbar), _p(w_), n)
    return o, lse, idx, w, kbar


def hsa_attend(q, k, v, idx, w, S: int = 64, want_lse: bool = True, o=None, ws=None, stream=None):
    """Attention and fusion for a given selection (idx, w from hsa_select or
    hsa_fwd), e.g. one selection shared by several layers.  Returns (o, lse)."""
    B, L, h_q, d = q.shape
    h_kv, K = k.shape[1], idx.shape[-1]
    dt, dev = _dtype_code(q), q.device
    _need(q, "q", q.shape, q.dtype)
    _need(k, "k", (B, h_kv, L, d), q.dtype, dev)
    _need(v, "v", (B, h_kv, L, d), q.dtype, dev)
    _need(idx, "idx", (B, L, h_kv, K), torch.int32, dev)
    _need(w, "w", (B, L, h_kv, K), torch.float32, dev)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype, dev)
    lse = torch.empty(B, L, h_q, K, dtype=torch.float32, device=dev) if want_lse else None
    sh = HsaShape(B, L, h_q, h_kv, d, S, K, dt)
    w_, n = _workspace(sh, OP_FWD, dev, ws)
    _run("hsa_attend", dev, stream, ctypes.byref(sh), _p(q), _p(k), _p(v), _p(idx), _p(w), _p(o),
         _p(lse), _p(w_), n)
    return o, lse


def hsa_decode(q, q_slc, k_cache, v_cache, kbar, K: int, S: int = 64, o=None, want_sel=True,
               ws=None, stream=None):
    """One decode step.  q [B,h_q,d], q_slc [B,h_kv,d], caches [B,h_kv,P,d],
    kbar [B,h_kv,P//S,d].  Returns (o, idx, w)."""
    B, h_q, d = q.shape
    h_kv, P = k_cache.shape[1], k_cache.shape[2]
    dt, dev = _dtype_code(q), q.device
    _need(q, "q", q.shape, q.dtype)
    _need(q_slc, "q_slc", (B, h_kv, d), q.dtype, dev)
    _need(k_cache, "k_cache", (B, h_kv, P, d), q.dtype, dev, host_ok=True)
    _need(v_cache, "v_cache", (B, h_kv, P, d), q.dtype, dev, host_ok=True)
    _need(kbar, "kbar", (B, h_kv, P // S, d), torch.float32, dev)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype, dev)
    idx = torch.empty(B, h_kv, K, dtype=torch.int32, device=dev) if want_sel else None
    w = torch.empty(B, h_kv, K, dtype=torch.float32, device=dev) if want_sel else None
    sh = HsaShape(B, P, h_q, h_kv, d, S, K, dt)
    w_, n = _workspace(sh, OP_DECODE, dev, ws)
    _run("hsa_decode", dev, stream, ctypes.byref(sh), _p(q), _p(q_slc), _p(k_cache), _p(v_cache),
         _p(kbar), _p(o), _p(idx), _p(w), _p(w_), n)
    return o, idx, w


def hsa_decode_multi(q, q_slc, k_cache, v_cache, kbar, K: int, S: int = 64, o=None, want_sel=True,
                     ws=None, stream=None):
    """One decode step for several HSA layers sharing the selection and the KV
    cache.  q [n_layers,B,h_q,d]; the rest as in hsa_decode (the caches may be
    page-locked host tensors).  Returns (o [n_layers,B,h_q,d], idx, w)."""
    NL, B, h_q, d = q.shape
    h_kv, P = k_cache.shape[1], k_cache.shape[2]
    dt, dev = _dtype_code(q), q.device
    _need(q, "q", q.shape, q.dtype)
    _need(q_slc, "q_slc", (B, h_kv, d), q.dtype, dev)
    _need(k_cache, "k_cache", (B, h_kv, P, d), q.dtype, dev, host_ok=True)
    _need(v_cache, "v_cache", (B, h_kv, P, d), q.dtype, dev, host_ok=True)
    _need(kbar, "kbar", (B, h_kv, P // S, d), torch.float32, dev)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype, dev)
    idx = torch.empty(B, h_kv, K, dtype=torch.int32, device=dev) if want_sel else None
    w = torch.empty(B, h_kv, K, dtype=torch.float32, device=dev) if want_sel else None
    sh = HsaShape(B, P, h_q, h_kv, d, S, K, dt)
    w_, n = _workspace(sh, OP_DECODE, dev, ws)
    _run("hsa_decode_multi", dev, stream, ctypes.byref(sh), NL, _p(q), _p(q_slc), _p(k_cache),
         _p(v_cache), _p(kbar), _p(o), _p(idx), _p(w), _p(w_), n)
    return o, idx, w


def hsa_bwd(q, k, v, q_slc, dO, lse, idx, w, kbar, K: int, S: int = 64, ws=None, stream=None):
    """Backward of hsa_fwd.  Returns (dq, dk, dv, dq_slc)."""
    B, L, h_q, d = q.shape
    h_kv = k.shape[1]
    dt, dev = _dtype_code(q), q.device
    _need(q, "q", q.shape, q.dtype)
    for name, t, shp in (("k", k, (B, h_kv, L, d)), ("v", v, (B, h_kv, L, d)),
                         ("q_slc", q_slc, (B, L, h_kv, d)), ("dO", dO, (B, L, h_q, d))):
        _need(t, name, shp, q.dtype, dev)
    _need(lse, "lse", (B, L, h_q, K), torch.float32, dev)
    _need(idx, "idx", (B, L, h_kv, K), torch.int32, dev)
    _need(w, "w", (B, L, h_kv, K), torch.float32, dev)
    _need(kbar, "kbar", (B, h_kv, L // S, d), torch.float32, dev)
    dq, dk, dv, dqs = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                       torch.empty_like(q_slc))
    sh = HsaShape(B, L, h_q, h_kv, d, S, K, dt)
    w_, n = _workspace(sh, OP_BWD, dev, ws)
    _run("hsa_bwd", dev, stream, ctypes.byref(sh), _p(q), _p(k), _p(v), _p(q_slc), _p(dO), _p(lse),
         _p(idx), _p(w), _p(kbar), _p(dq), _p(dk), _p(dv), _p(dqs), _p(w_), n)
    return dq, dk, dv, dqs


def hsa_device_status(ws: torch.Tensor, stream=None) -> int:
    code = ctypes.c_int32(0)
    _run("hsa_device_status", ws.device, stream, _p(ws), ctypes.byref(code))
    return int(code.value)


def hsa_set_wait_limit_ns(ns: int) -> None:
    """Bound every wait inside the persistent kernels at `ns` nanoseconds (0: the
    default of 2 s) -- a testing aid that makes a wait run out on purpose."""
    _check(load_library().hsa_set_wait_limit_ns(int(ns)), "hsa_set_wait_limit_ns")


def hsa_timing_enable(on: bool = True) -> None:
    """Start (and clear) or stop CUDA-event timing of the library's launches."""
    _check(load_library().hsa_timing_enable(1 if on else 0), "hsa_timing_enable")


def hsa_timing_read(kind) -> tuple[float, int]:
    """(total milliseconds, kernel launches) recorded for a kernel kind."""
    k = KERNELS[kind] if isinstance(kind, str) else int(kind)
    ms, n = ctypes.c_double(0.0), ctypes.c_int64(0)
    _check(load_library().hsa_timing_read(k, ctypes.byref(ms), ctypes.byref(n)), "hsa_timing_read")
    return float(ms.value), int(n.value)
