"""Python binding of the C ABI in include/fa.h (argument marshalling only).

Every step of the attention runs in the sm_100a kernels of
``libfa_sm100.so``; this module only checks tensors, allocates outputs with
PyTorch (device memory is PyTorch's job here) and passes raw pointers and the
current CUDA stream.  There is no fallback: if the library is missing or the
device is not a B200 the calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_sm100.so")
HEADER_PATH = os.path.join(os.path.dirname(HERE), "include", "fa.h")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_TOO_LARGE = range(6)
NOALLOC_SCRATCH_BYTES = 32 << 20  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


class FaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("N", ctypes.c_int),
                ("D", ctypes.c_int), ("scale", ctypes.c_float), ("causal", ctypes.c_int)]


class FaKvShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("Nq", ctypes.c_int),
                ("Nk", ctypes.c_int), ("D", ctypes.c_int), ("scale", ctypes.c_float), ("causal", ctypes.c_int)]


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (built in-tree by ``tiled_attention_16_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run `python -m tiled_attention_16_b200.build`)")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        shp = ctypes.POINTER(FaShape)
        L.fa_fwd.argtypes = [shp, vp, vp, vp, vp, vp, vp]
        f32 = ctypes.c_float
        L.fa_fwd_fp8.argtypes = [shp, vp, vp, vp, f32, f32, f32, vp, vp, vp]
        L.fa_fwd_fp8.restype = ctypes.c_int
        kshp = ctypes.POINTER(FaKvShape)
        L.fa_decode_workspace_bytes.argtypes = [kshp]
        L.fa_decode_workspace_bytes.restype = ctypes.c_size_t
        L.fa_decode.argtypes = [kshp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.fa_decode.restype = ctypes.c_int
        L.fa_fwd.restype = ctypes.c_int
        L.fa_bwd_workspace_bytes.argtypes = [shp]
        L.fa_bwd_workspace_bytes.restype = sz
        L.fa_bwd.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.fa_bwd.restype = ctypes.c_int
        L.fa_get_device_status.argtypes = [vp]
        L.fa_get_device_status.restype = ctypes.c_int
        L.fa_status_str.argtypes = [ctypes.c_int]
        L.fa_status_str.restype = ctypes.c_char_p
        L.fa_debug_timeout_sites.argtypes = []
        L.fa_debug_timeout_sites.restype = ctypes.c_uint
        L.fa_bwd_noalloc.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.fa_bwd_noalloc.restype = ctypes.c_int
        ll = ctypes.c_longlong
        L.fa_lse_merge.argtypes = [ll, ctypes.c_int, vp, vp, vp, vp, vp, ctypes.c_int, vp]
        L.fa_lse_merge.restype = ctypes.c_int
        L.fa_accumulate.argtypes = [ll, vp, vp, vp, ctypes.c_int, vp]
        L.fa_accumulate.restype = ctypes.c_int
        L.fa_fwd_merge.argtypes = [shp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp]
        L.fa_fwd_merge.restype = ctypes.c_int
        L.fa_bwd_stats.argtypes = [shp, vp, vp, vp, vp, sz, vp]
        L.fa_bwd_stats.restype = ctypes.c_int
        L.fa_bwd_accumulate.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, sz, vp]
        L.fa_bwd_accumulate.restype = ctypes.c_int
        L.fa_selftest_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_int, vp]
        L.fa_selftest_wait_timeout.restype = ctypes.c_int
        L.fa_profile_begin.argtypes = []
        L.fa_profile_begin.restype = ctypes.c_int
        L.fa_profile_end.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]
        L.fa_profile_end.restype = ctypes.c_int
        L.fa_set_bwd_mode.argtypes = [ctypes.c_int]
        L.fa_set_bwd_mode.restype = ctypes.c_int
        L.fa_get_bwd_mode.argtypes = []
        L.fa_get_bwd_mode.restype = ctypes.c_int
        _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Entry points declared in include/fa.h (FA_API functions)."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def status_str(status: int) -> str:
    return lib().fa_status_str(int(status)).decode()


def make_shape(B, Hq, Hkv, N, D, scale, causal) -> FaShape:
    return FaShape(int(B), int(Hq), int(Hkv), int(N), int(D), float(scale), 1 if causal else 0)


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(t: torch.Tensor, name: str, shape, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _same_device(*tensors):
    """The device every given tensor (None entries skipped) lives on.  The
    library builds its tensor maps and looks up its static tables on the
    current CUDA device, so all tensors of one call must share a device and
    the call runs with that device made current."""
    ts = [t for t in tensors if t is not None]
    dev = ts[0].device
    for t in ts[1:]:
        if t.device != dev:
            raise ValueError(f"all tensors must be on one device: got {dev} and {t.device}")
    return dev


def _dims(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, H, N, D]")
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    return B, Hq, Hkv, N, D


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, scale: float | None = None,
        out: torch.Tensor | None = None, lse: torch.Tensor | None = None):
    """Attention forward.  Returns (o [B,Hq,N,D] bf16, lse [B,Hq,N] fp32)."""
    B, Hq, Hkv, N, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check(q, "q", (B, Hq, N, D))
    _check(k, "k", (B, Hkv, N, D))
    _check(v, "v", (B, Hkv, N, D))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    _check(out, "out", (B, Hq, N, D))
    _check(lse, "lse", (B, Hq, N), torch.float32)
    dev = _same_device(q, k, v, out, lse)
    shp = make_shape(B, Hq, Hkv, N, D, scale, causal)
    with torch.cuda.device(dev):
        st = lib().fa_fwd(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          lse.data_ptr(), _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_fwd")
    return out, lse


def fwd_fp8(q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, q_scale: float = 1.0, k_scale: float = 1.0,
            v_scale: float = 1.0, causal: bool = False, scale: float | None = None,
            out: torch.Tensor | None = None, lse: torch.Tensor | None = None):
    """FP8 attention forward over e4m3 tensors (torch.float8_e4m3fn), each
    element standing for element * its tensor's descale.  Returns (o bf16,
    lse fp32) as fwd() does.  Head dimension 128 only."""
    B, Hq, Hkv, N, D = _dims(q8, k8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check(q8, "q8", (B, Hq, N, D), torch.float8_e4m3fn)
    _check(k8, "k8", (B, Hkv, N, D), torch.float8_e4m3fn)
    _check(v8, "v8", (B, Hkv, N, D), torch.float8_e4m3fn)
    if out is None:
        out = torch.empty((B, Hq, N, D), device=q8.device, dtype=torch.bfloat16)
    if lse is None:
        lse = torch.empty((B, Hq, N), device=q8.device, dtype=torch.float32)
    _check(out, "out", (B, Hq, N, D))
    _check(lse, "lse", (B, Hq, N), torch.float32)
    dev = _same_device(q8, k8, v8, out, lse)
    shp = make_shape(B, Hq, Hkv, N, D, scale, causal)
    with torch.cuda.device(dev):
        st = lib().fa_fwd_fp8(ctypes.byref(shp), q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), float(q_scale),
                              float(k_scale), float(v_scale), out.data_ptr(), lse.data_ptr(), _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_fp8")
    return out, lse


def make_kv_shape(B, Hq, Hkv, Nq, Nk, D, scale, causal) -> FaKvShape:
    return FaKvShape(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(D), float(scale), 1 if causal else 0)


def decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, D, causal=True, scale=None) -> int:
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    return int(lib().fa_decode_workspace_bytes(ctypes.byref(make_kv_shape(B, Hq, Hkv, Nq, Nk, D, scale, causal))))


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, scale: float | None = None,
           out: torch.Tensor | None = None, lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Attention of Nq new queries q [B,Hq,Nq,D] over an Nk-long K/V history
    k, v [B,Hkv,Nk,D] (bf16); query i stands at position Nk - Nq + i.
    Returns (o [B,Hq,Nq,D] bf16, lse [B,Hq,Nq] fp32)."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, H, N, D]")
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check(q, "q", (B, Hq, Nq, D))
    _check(k, "k", (B, Hkv, Nk, D))
    _check(v, "v", (B, Hkv, Nk, D))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32)
    _check(out, "out", (B, Hq, Nq, D))
    _check(lse, "lse", (B, Hq, Nq), torch.float32)
    shp = make_kv_shape(B, Hq, Hkv, Nq, Nk, D, scale, causal)
    nbytes = int(lib().fa_decode_workspace_bytes(ctypes.byref(shp)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), device=q.device, dtype=torch.uint8)
    if workspace.device.type != "cuda" or workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace must be a CUDA buffer of at least {nbytes} bytes")
    dev = _same_device(q, k, v, out, lse, workspace)
    with torch.cuda.device(dev):
        st = lib().fa_decode(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_decode")
    return out, lse


BWD_MODES = {"auto": 0, "deterministic": 1, "fused": 2}   # FA_BWD_AUTO, _DETERMINISTIC, _FUSED


def set_bwd_mode(mode: str) -> None:
    """Process-wide dQ strategy of bwd(): "fused" (one kernel, dQ summed by fp32
    reductions in varying order), "deterministic" (separate dQ pass; repeated
    calls bitwise equal) or "auto" (the measured choice: fused for D = 128).
    The environment variable FA_DQ_MODE, if set, overrides it."""
    st = lib().fa_set_bwd_mode(BWD_MODES[mode])
    if st != FA_OK:
        raise FAError(st, "fa_set_bwd_mode")


def get_bwd_mode() -> str:
    m = lib().fa_get_bwd_mode()
    return next(k for k, v in BWD_MODES.items() if v == m)


@contextlib.contextmanager
def bwd_mode(mode: str):
    """Run the enclosed calls under backward mode `mode`, then restore the previous one."""
    old = get_bwd_mode()
    set_bwd_mode(mode)
    try:
        yield
    finally:
        set_bwd_mode(old)


def workspace_bytes(B, Hq, Hkv, N, D, causal=False, scale=None) -> int:
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    shp = make_shape(B, Hq, Hkv, N, D, scale, causal)
    return int(lib().fa_bwd_workspace_bytes(ctypes.byref(shp)))


def bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None,
        dq=None, dk=None, dv=None, workspace: torch.Tensor | None = None):
    """Attention backward.  Returns (dq, dk, dv), bf16, shaped like q, k, v."""
    B, Hq, Hkv, N, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    for t, name, shape in ((q, "q", (B, Hq, N, D)), (k, "k", (B, Hkv, N, D)), (v, "v", (B, Hkv, N, D)),
                           (o, "o", (B, Hq, N, D)), (do, "do", (B, Hq, N, D))):
        _check(t, name, shape)
    _check(lse, "lse", (B, Hq, N), torch.float32)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", (B, Hq, N, D))
    _check(dk, "dk", (B, Hkv, N, D))
    _check(dv, "dv", (B, Hkv, N, D))
    shp = make_shape(B, Hq, Hkv, N, D, scale, causal)
    nbytes = int(lib().fa_bwd_workspace_bytes(ctypes.byref(shp)))
    if workspace is None:
        workspace = torch.empty(nbytes, device=q.device, dtype=torch.uint8)
    if workspace.device.type != "cuda" or workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace must be a CUDA buffer of at least {nbytes} bytes")
    dev = _same_device(q, k, v, o, do, lse, dq, dk, dv, workspace)
    with torch.cuda.device(dev):
        st = lib().fa_bwd(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                          lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                          workspace.numel() * workspace.element_size(), _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_bwd")
    return dq, dk, dv


def bwd_noalloc(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, dq=None, dk=None, dv=None):
    """Backward through fa_bwd_noalloc: no workspace argument, the library's
    static scratch is used (for callers that must not allocate device memory
    on this path).  Output tensors may be passed in to avoid allocating them
    here too.  Calls on one device share the scratch, so they must not overlap."""
    B, Hq, Hkv, N, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    for t, name, shape in ((q, "q", (B, Hq, N, D)), (k, "k", (B, Hkv, N, D)), (v, "v", (B, Hkv, N, D)),
                           (o, "o", (B, Hq, N, D)), (do, "do", (B, Hq, N, D))):
        _check(t, name, shape)
    _check(lse, "lse", (B, Hq, N), torch.float32)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", (B, Hq, N, D))
    _check(dk, "dk", (B, Hkv, N, D))
    _check(dv, "dv", (B, Hkv, N, D))
    dev = _same_device(q, k, v, o, do, lse, dq, dk, dv)
    shp = make_shape(B, Hq, Hkv, N, D, scale, causal)
    with torch.cuda.device(dev):
        st = lib().fa_bwd_noalloc(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_noalloc")
    return dq, dk, dv


FA_ACC_DQ_FIRST, FA_ACC_DKV_FIRST = 1, 2


def fwd_merge(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o_acc: torch.Tensor, lse_acc: torch.Tensor,
              causal: bool = False, scale: float | None = None, first: bool = False,
              out: torch.Tensor | None = None) -> None:
    """Attention of q over (k, v), folded into the running fp32 result
    (o_acc [B,Hq,N,D], lse_acc [B,Hq,N]) in place by the log-sum-exp rule
    inside the forward kernel (fa_fwd_merge); first=True sets it from this
    call; `out` (bf16) also receives the merged result."""
    B, Hq, Hkv, N, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check(q, "q", (B, Hq, N, D))
    _check(k, "k", (B, Hkv, N, D))
    _check(v, "v", (B, Hkv, N, D))
    _check(o_acc, "o_acc", (B, Hq, N, D), torch.float32)
    _check(lse_acc, "lse_acc", (B, Hq, N), torch.float32)
    if out is not None:
        _check(out, "out", (B, Hq, N, D))
    dev = _same_device(q, k, v, o_acc, lse_acc, out)
    shp = make_shape(B, Hq, Hkv, N, D, scale, causal)
    with torch.cuda.device(dev):
        st = lib().fa_fwd_merge(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), o_acc.data_ptr(),
                                lse_acc.data_ptr(), None if out is None else out.data_ptr(), 1 if first else 0,
                                _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_merge")


def bwd_stats(o: torch.Tensor, do: torch.Tensor, lse: torch.Tensor, causal: bool = False, scale: float | None = None,
              workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Row statistics of the backward for (o, do, lse) written into a
    workspace (fa_bwd_stats); returns the workspace for bwd_accumulate."""
    B, Hq, N, D = o.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check(o, "o", (B, Hq, N, D))
    _check(do, "do", (B, Hq, N, D))
    _check(lse, "lse", (B, Hq, N), torch.float32)
    shp = make_shape(B, Hq, Hq, N, D, scale, causal)
    nbytes = int(lib().fa_bwd_workspace_bytes(ctypes.byref(shp)))
    if workspace is None:
        workspace = torch.empty(nbytes, device=o.device, dtype=torch.uint8)
    if workspace.device.type != "cuda" or workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace must be a CUDA buffer of at least {nbytes} bytes")
    dev = _same_device(o, do, lse, workspace)
    with torch.cuda.device(dev):
        st = lib().fa_bwd_stats(ctypes.byref(shp), o.data_ptr(), do.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_stats")
    return workspace


def bwd_accumulate(q, k, v, do, workspace: torch.Tensor, dq_acc: torch.Tensor, dk_acc: torch.Tensor,
                   dv_acc: torch.Tensor, causal: bool = False, scale: float | None = None, first_dq: bool = False,
                   first_dkv: bool = False) -> None:
    """Gradients of (q, k, v) on the statistics that bwd_stats left in
    `workspace`, added into fp32 sums in place (fa_bwd_accumulate); the first
    flags overwrite instead of adding."""
    B, Hq, Hkv, N, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    for t, name, shape in ((q, "q", (B, Hq, N, D)), (k, "k", (B, Hkv, N, D)), (v, "v", (B, Hkv, N, D)),
                           (do, "do", (B, Hq, N, D))):
        _check(t, name, shape)
    _check(dq_acc, "dq_acc", (B, Hq, N, D), torch.float32)
    _check(dk_acc, "dk_acc", (B, Hkv, N, D), torch.float32)
    _check(dv_acc, "dv_acc", (B, Hkv, N, D), torch.float32)
    dev = _same_device(q, k, v, do, workspace, dq_acc, dk_acc, dv_acc)
    shp = make_shape(B, Hq, Hkv, N, D, scale, causal)
    flags = (FA_ACC_DQ_FIRST if first_dq else 0) | (FA_ACC_DKV_FIRST if first_dkv else 0)
    with torch.cuda.device(dev):
        st = lib().fa_bwd_accumulate(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(),
                                     dq_acc.data_ptr(), dk_acc.data_ptr(), dv_acc.data_ptr(), flags,
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_accumulate")


def lse_merge(o_acc: torch.Tensor, lse_acc: torch.Tensor, o_part: torch.Tensor, lse_part: torch.Tensor,
              first: bool = False, out: torch.Tensor | None = None) -> None:
    """Merge a partial result (o_part bf16 [..., D], lse_part fp32 [...]) over
    one block of keys into the running result (o_acc fp32 [..., D], lse_acc
    fp32 [...]) in place, by the log-sum-exp rule (fa_lse_merge).  With
    first=True the running result is set from the part.  `out` (bf16, shaped
    like o_part) also receives the merged result when given."""
    D = o_part.shape[-1]
    rows = o_part.numel() // D if D else 0
    _check(o_part, "o_part", o_part.shape)
    _check(o_acc, "o_acc", o_part.shape, torch.float32)
    _check(lse_part, "lse_part", o_part.shape[:-1], torch.float32)
    _check(lse_acc, "lse_acc", o_part.shape[:-1], torch.float32)
    if out is not None:
        _check(out, "out", o_part.shape)
    dev = _same_device(o_part, o_acc, lse_part, lse_acc, out)
    with torch.cuda.device(dev):
        st = lib().fa_lse_merge(rows, int(D), o_part.data_ptr(), lse_part.data_ptr(), o_acc.data_ptr(),
                                lse_acc.data_ptr(), None if out is None else out.data_ptr(), 1 if first else 0,
                                _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_lse_merge")


def accumulate(acc: torch.Tensor, src: torch.Tensor | None, first: bool = False,
               out: torch.Tensor | None = None) -> None:
    """acc (fp32) = (0 if first else acc) + src (bf16, same shape; None adds
    nothing), in place (fa_accumulate); `out` (bf16) also receives bf16(acc)."""
    _check(acc, "acc", acc.shape, torch.float32)
    if src is not None:
        _check(src, "src", acc.shape)
    if out is not None:
        _check(out, "out", acc.shape)
    dev = _same_device(acc, src, out)
    with torch.cuda.device(dev):
        st = lib().fa_accumulate(acc.numel(), None if src is None else src.data_ptr(), acc.data_ptr(),
                                 None if out is None else out.data_ptr(), 1 if first else 0, _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_accumulate")


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):   # the status word read is the current device's
        return int(lib().fa_get_device_status(_stream_ptr(dev)))


def selftest_wait_timeout(site: int, site2: int, device=None) -> None:
    """Launch the failure-detection self-test (fa_selftest_wait_timeout) on the
    current stream; read the outcome with device_status() and timeout_sites()."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        st = lib().fa_selftest_wait_timeout(int(site), int(site2), _stream_ptr(dev))
    if st != FA_OK:
        raise FAError(st, "fa_selftest_wait_timeout")


def timeout_sites() -> int:
    return int(lib().fa_debug_timeout_sites())


PROFILE_KINDS = ("fa_fwd_kernel", "fa_bwd_preprocess", "fa_bwd_kernel", "fa_bwd_dq_convert",
                 "fa_bwd_dkdv_kernel", "fa_bwd_dq_kernel", "fa_fwd_fp8_kernel", "fa_decode",
                 "fa_lse_merge_kernel", "fa_accumulate_kernel", "fa_fwd_pair_kernel",
                 "fa_bwd_dkdv_pair_kernel", "fa_bwd_dq_pair_kernel", "fa_bwd_fused_kernel")


def profile_begin() -> None:
    st = lib().fa_profile_begin()
    if st != FA_OK:
        raise FAError(st, "fa_profile_begin")


def profile_end() -> dict:
    """{kernel name: (total ms, launches)} for the launches since profile_begin()."""
    ms = (ctypes.c_float * len(PROFILE_KINDS))()
    n = (ctypes.c_int * len(PROFILE_KINDS))()
    st = lib().fa_profile_end(ms, n)
    if st != FA_OK:
        raise FAError(st, "fa_profile_end")
    return {k: (float(ms[i]), int(n[i])) for i, k in enumerate(PROFILE_KINDS)}
