"""Thin Python binding of libfa.so (argument marshalling only).

The raw functions carry the C names of ``include/fa.h`` and take integer
device pointers; ``forward`` / ``backward`` / ``attention`` accept torch CUDA
tensors, allocate outputs and workspace with torch, pass the current stream
and raise ``FaError`` on a non-zero status. Every step of the computation runs
in the library's CUDA kernels. There is no fallback: if the library is missing
the first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
# FA_LIBRARY may name another build of libfa.so (e.g. one compiled with
# different tile parameters); the default is the in-tree build.
LIB_PATH = os.environ.get("FA_LIBRARY") or os.path.join(PKG, "_lib", "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
FA_F32, FA_BF16 = 0, 1
PATH_AUTO, PATH_SIMT, PATH_TC = 0, 1, 2
FA_STALL_FWD, FA_STALL_BWD, FA_STALL_DQ = 1, 2, 4

# every symbol include/fa.h declares
EXPORTS = ("fa_status_string", "fa_version", "fa_fwd_workspace_size", "fa_bwd_workspace_size",
           "fa_fwd", "fa_fwd_ex", "fa_bwd", "fa_bwd_ex", "fa_bwd_preprocess", "fa_bwd_main",
           "fa_bwd_finalize", "fa_last_launch_count", "fa_get_device_error", "fa_exp2_fma",
           "fa_fwd_varlen", "fa_bwd_varlen", "fa_bwd_varlen_workspace_size",
           "fa_bwd_deterministic", "fa_fwd_window", "fa_bwd_window", "fa_bwd_noalloc",
           "fa_debug_set_stall", "fa_fwd_mod", "fa_bwd_mod")

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t
_FWD_ARGS = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _I, _P, _P]
_BWD_ARGS = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _I, _I, _P, _S,
             _P]


class FaMods(ctypes.Structure):
    """fa_mods of include/fa.h: mask (and score) modifiers."""
    _fields_ = [("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
                ("prefix", ctypes.c_int), ("doc_ids", ctypes.c_void_p),
                ("softcap", ctypes.c_float)]


def mods(window_left: int = -1, window_right: int = -1, prefix: int = 0, doc_ids=None,
         softcap: float = 0.0) -> FaMods:
    """An fa_mods value; doc_ids is an int32 CUDA tensor [N] or None."""
    return FaMods(int(window_left), int(window_right), int(prefix),
                  None if doc_ids is None else doc_ids.data_ptr(), float(softcap))


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Loads libfa.so once (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfa.so not built ({LIB_PATH}); run "
                               "python -m exact_io_aware_45_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_status_string.argtypes = [_I]
        L.fa_version.restype = _I
        L.fa_fwd_workspace_size.restype = _S
        L.fa_bwd_workspace_size.restype = _S
        L.fa_bwd_workspace_size.argtypes = [_I, _I, _I, _I]
        L.fa_fwd.argtypes = _FWD_ARGS
        L.fa_fwd_ex.argtypes = _FWD_ARGS + [_I]
        L.fa_bwd.argtypes = _BWD_ARGS
        for n in ("fa_bwd_ex", "fa_bwd_preprocess", "fa_bwd_main", "fa_bwd_finalize",
                  "fa_bwd_deterministic"):
            getattr(L, n).argtypes = _BWD_ARGS + [_I]
        for n in ("fa_fwd", "fa_fwd_ex", "fa_bwd", "fa_bwd_ex", "fa_bwd_preprocess",
                  "fa_bwd_main", "fa_bwd_finalize", "fa_get_device_error", "fa_bwd_deterministic"):
            getattr(L, n).restype = _I
        L.fa_last_launch_count.restype = _I
        L.fa_get_device_error.argtypes = [_P, _P]
        L.fa_exp2_fma.argtypes = [_P, _P, ctypes.c_longlong, _P]
        L.fa_exp2_fma.restype = _I
        L.fa_fwd_varlen.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                                    _P, _P]
        L.fa_fwd_varlen.restype = _I
        L.fa_bwd_varlen.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                                    _I, _F, _I, _I, _I, _P, _S, _P]
        L.fa_bwd_varlen.restype = _I
        L.fa_fwd_window.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P,
                                    _I, _P, _P]
        L.fa_fwd_window.restype = _I
        L.fa_bwd_window.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F,
                                    _I, _I, _I, _P, _I, _I, _P, _S, _P]
        L.fa_bwd_window.restype = _I
        L.fa_fwd_mod.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P,
                                 ctypes.POINTER(FaMods), _I, _P, _P]
        L.fa_fwd_mod.restype = _I
        L.fa_bwd_mod.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I,
                                 _P, ctypes.POINTER(FaMods), _I, _I, _P, _S, _P]
        L.fa_bwd_mod.restype = _I
        L.fa_debug_set_stall.argtypes = [_I, ctypes.c_longlong]
        L.fa_debug_set_stall.restype = _I
        L.fa_bwd_varlen_workspace_size.argtypes = [_I, _I, _I, _I, _I]
        L.fa_bwd_varlen_workspace_size.restype = _S
        _lib = L
    return _lib


# ------------------------------------------------------------------ raw C functions

def status_string(s: int) -> str:
    return lib().fa_status_string(int(s)).decode()


def fa_version() -> int:
    return lib().fa_version()


def fa_fwd_workspace_size() -> int:
    return lib().fa_fwd_workspace_size()


def fa_bwd_workspace_size(B, Hq, N, d) -> int:
    return lib().fa_bwd_workspace_size(B, Hq, N, d)


def fa_fwd(*args) -> int:
    return lib().fa_fwd(*args)


def fa_fwd_ex(*args) -> int:
    return lib().fa_fwd_ex(*args)


def fa_bwd(*args) -> int:
    return lib().fa_bwd(*args)


def fa_bwd_ex(*args) -> int:
    return lib().fa_bwd_ex(*args)


def fa_bwd_preprocess(*args) -> int:
    return lib().fa_bwd_preprocess(*args)


def fa_bwd_main(*args) -> int:
    return lib().fa_bwd_main(*args)


def fa_bwd_finalize(*args) -> int:
    return lib().fa_bwd_finalize(*args)


def fa_last_launch_count() -> int:
    return lib().fa_last_launch_count()


def fa_get_device_error(workspace_ptr: int, stream_ptr: int) -> int:
    return lib().fa_get_device_error(workspace_ptr, stream_ptr)


def fa_exp2_fma(x_ptr: int, y_ptr: int, n: int, stream_ptr: int) -> int:
    return lib().fa_exp2_fma(x_ptr, y_ptr, n, stream_ptr)


def fa_bwd_deterministic(*args) -> int:
    return lib().fa_bwd_deterministic(*args)


def fa_fwd_window(*args) -> int:
    return lib().fa_fwd_window(*args)


def fa_bwd_window(*args) -> int:
    return lib().fa_bwd_window(*args)


def fa_fwd_varlen(*args) -> int:
    return lib().fa_fwd_varlen(*args)


def fa_bwd_varlen(*args) -> int:
    return lib().fa_bwd_varlen(*args)


def fa_fwd_mod(*args) -> int:
    return lib().fa_fwd_mod(*args)


def fa_bwd_mod(*args) -> int:
    return lib().fa_bwd_mod(*args)


def fa_debug_set_stall(kernels: int, wait_cycles: int) -> int:
    return lib().fa_debug_set_stall(int(kernels), int(wait_cycles))


def fa_bwd_varlen_workspace_size(B, Hq, max_seqlen, total, d) -> int:
    return lib().fa_bwd_varlen_workspace_size(B, Hq, max_seqlen, total, d)


# ------------------------------------------------------------------ torch helpers

def _dtype_code(t) -> int:
    import torch
    if t == torch.float32:
        return FA_F32
    if t == torch.bfloat16:
        return FA_BF16
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _check(status: int, what: str):
    if status != FA_OK:
        raise FaError(status, what)


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def new_workspace(nbytes: int, device):
    """A workspace buffer whose 256-byte error-word block is zeroed."""
    import torch
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def _dims(q, k):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    return B, Hq, Hkv, N, d


def forward(q, k, v, scale: Optional[float] = None, causal: bool = False, block_mask=None,
            path: int = PATH_AUTO, out=None, lse=None, workspace=None):
    """O, LSE = attention(q, k, v). q [B,Hq,N,d], k/v [B,Hkv,N,d] contiguous CUDA
    tensors (bf16 or fp32); block_mask uint8 [nb, nb] CUDA tensor or None;
    scale defaults to 1/sqrt(d)."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    ws = new_workspace(fa_fwd_workspace_size(), q.device) if workspace is None else workspace
    s = fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, Hq, Hkv, N, d, float(scale),
                  int(bool(causal)), _ptr(block_mask), _dtype_code(q.dtype), _ptr(ws), _stream(),
                  int(path))
    _check(s, "fa_fwd")
    return o, l


def backward(q, k, v, o, do, lse, scale: Optional[float] = None, causal: bool = False,
             block_mask=None, grad_dtype=None, path: int = PATH_AUTO, workspace=None,
             deterministic: bool = False):
    """dQ, dK, dV of sum(O * dO). grad_dtype defaults to float32 (the tensor
    cores accumulate in fp32; a bf16 gradient adds its own rounding).
    deterministic: run-to-run identical dQ (fa_bwd_deterministic)."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    gdt = torch.float32 if grad_dtype is None else grad_dtype
    dq = torch.empty(q.shape, dtype=gdt, device=q.device)
    dk = torch.empty(k.shape, dtype=gdt, device=q.device)
    dv = torch.empty(v.shape, dtype=gdt, device=q.device)
    nbytes = fa_bwd_workspace_size(B, Hq, N, d)
    ws = new_workspace(nbytes, q.device) if workspace is None else workspace
    fn = fa_bwd_deterministic if deterministic else fa_bwd_ex
    s = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
           _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)), _ptr(block_mask),
           _dtype_code(q.dtype), _dtype_code(gdt), _ptr(ws), ws.numel(), _stream(), int(path))
    _check(s, "fa_bwd_deterministic" if deterministic else "fa_bwd")
    return dq, dk, dv


def forward_varlen(q, k, v, cu_seqlens, max_seqlen: int, scale: Optional[float] = None,
                   causal: bool = False, out=None, lse=None, workspace=None):
    """Variable-length batch: q [total, Hq, d], k/v [total, Hkv, d] (bf16,
    sequences packed back to back), cu_seqlens int32 CUDA tensor [B + 1].
    Returns O [total, Hq, d] and LSE [Hq, total]."""
    import torch
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((Hq, total), dtype=torch.float32, device=q.device) if lse is None else lse
    ws = new_workspace(fa_fwd_workspace_size(), q.device) if workspace is None else workspace
    s = fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), _ptr(cu_seqlens), B,
                      int(max_seqlen), total, Hq, Hkv, d, float(scale), int(bool(causal)),
                      _dtype_code(q.dtype), _ptr(ws), _stream())
    _check(s, "fa_fwd_varlen")
    return o, l


def backward_varlen(q, k, v, o, do, lse, cu_seqlens, max_seqlen: int,
                    scale: Optional[float] = None, causal: bool = False, grad_dtype=None,
                    workspace=None):
    """dQ, dK, dV of a variable-length batch (layouts as forward_varlen)."""
    import torch
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    gdt = torch.float32 if grad_dtype is None else grad_dtype
    dq = torch.empty(q.shape, dtype=gdt, device=q.device)
    dk = torch.empty(k.shape, dtype=gdt, device=q.device)
    dv = torch.empty(v.shape, dtype=gdt, device=q.device)
    nbytes = fa_bwd_varlen_workspace_size(B, Hq, int(max_seqlen), total, d)
    ws = new_workspace(nbytes, q.device) if workspace is None else workspace
    s = fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                      _ptr(dk), _ptr(dv), _ptr(cu_seqlens), B, int(max_seqlen), total, Hq, Hkv,
                      d, float(scale), int(bool(causal)), _dtype_code(q.dtype), _dtype_code(gdt),
                      _ptr(ws), ws.numel(), _stream())
    _check(s, "fa_bwd_varlen")
    return dq, dk, dv


def forward_window(q, k, v, window_left: int, window_right: int, scale: Optional[float] = None,
                   causal: bool = False, block_mask=None):
    """O, LSE of sliding-window attention (fa_fwd_window); layouts as forward."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    l = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    ws = new_workspace(fa_fwd_workspace_size(), q.device)
    s = fa_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, Hq, Hkv, N, d, float(scale),
                      int(bool(causal)), int(window_left), int(window_right), _ptr(block_mask),
                      _dtype_code(q.dtype), _ptr(ws), _stream())
    _check(s, "fa_fwd_window")
    return o, l


def backward_window(q, k, v, o, do, lse, window_left: int, window_right: int,
                    scale: Optional[float] = None, causal: bool = False, block_mask=None,
                    grad_dtype=None):
    """dQ, dK, dV of sliding-window attention (fa_bwd_window)."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    gdt = torch.float32 if grad_dtype is None else grad_dtype
    dq = torch.empty(q.shape, dtype=gdt, device=q.device)
    dk = torch.empty(k.shape, dtype=gdt, device=q.device)
    dv = torch.empty(v.shape, dtype=gdt, device=q.device)
    ws = new_workspace(fa_bwd_workspace_size(B, Hq, N, d), q.device)
    s = fa_bwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                      _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                      int(window_left), int(window_right), _ptr(block_mask), _dtype_code(q.dtype),
                      _dtype_code(gdt), _ptr(ws), ws.numel(), _stream())
    _check(s, "fa_bwd_window")
    return dq, dk, dv


def forward_mod(q, k, v, m: FaMods, scale: Optional[float] = None, causal: bool = False,
                block_mask=None, workspace=None, out=None, lse=None):
    """O, LSE with mask modifiers (fa_fwd_mod); layouts and out / lse / workspace
    as forward."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    ws = new_workspace(fa_fwd_workspace_size(), q.device) if workspace is None else workspace
    s = fa_fwd_mod(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, Hq, Hkv, N, d, float(scale),
                   int(bool(causal)), _ptr(block_mask), ctypes.byref(m), _dtype_code(q.dtype),
                   _ptr(ws), _stream())
    _check(s, "fa_fwd_mod")
    return o, l


def backward_mod(q, k, v, o, do, lse, m: FaMods, scale: Optional[float] = None,
                 causal: bool = False, block_mask=None, grad_dtype=None, workspace=None):
    """dQ, dK, dV with mask modifiers (fa_bwd_mod); the forward's modifiers."""
    import torch
    B, Hq, Hkv, N, d = _dims(q, k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    gdt = torch.float32 if grad_dtype is None else grad_dtype
    dq = torch.empty(q.shape, dtype=gdt, device=q.device)
    dk = torch.empty(k.shape, dtype=gdt, device=q.device)
    dv = torch.empty(v.shape, dtype=gdt, device=q.device)
    ws = new_workspace(fa_bwd_workspace_size(B, Hq, N, d), q.device) if workspace is None \
        else workspace
    s = fa_bwd_mod(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                   _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)), _ptr(block_mask),
                   ctypes.byref(m), _dtype_code(q.dtype), _dtype_code(gdt), _ptr(ws), ws.numel(),
                   _stream())
    _check(s, "fa_bwd_mod")
    return dq, dk, dv


def device_error(workspace) -> int:
    """Reads and clears the workspace's error word (synchronises the stream)."""
    return fa_get_device_error(_ptr(workspace), _stream())


def _autograd_fn():
    import torch

    class _Attention(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, scale, causal, block_mask):
            o, lse = forward(q, k, v, scale, causal, block_mask)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.scale, ctx.causal, ctx.block_mask = scale, causal, block_mask
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = backward(q, k, v, o, do.contiguous(), lse, ctx.scale, ctx.causal,
                                  ctx.block_mask, grad_dtype=q.dtype)
            return dq, dk, dv, None, None, None

    return _Attention


def attention(q, k, v, scale: Optional[float] = None, causal: bool = False, block_mask=None):
    """Differentiable attention (torch autograd), gradients in the input dtype."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return _autograd_fn().apply(q, k, v, scale, causal, block_mask)
