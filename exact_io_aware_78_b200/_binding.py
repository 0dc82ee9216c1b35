"""ctypes binding of libexactattn.so (argument marshalling only).

Function names match the C ABI in include/exactattn.h.  Every step of the
attention forward runs in the library's CUDA kernels; PyTorch only provides
device memory and the current stream.  There is no CPU fallback: if the
library is missing or the device is not an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libexactattn.so")

EA_BF16, EA_FP8_E4M3, EA_FP32 = 0, 1, 2
EA_OK, EA_EINVAL, EA_EUNSUPPORTED, EA_EALIGN, EA_ELAUNCH, EA_EDEVICE_TIMEOUT, EA_ECUDA, EA_ENOMEM = (
    0, -1, -2, -3, -4, -5, -6, -7)
EA_OPT_WAIT_TIMEOUT_NS, EA_OPT_MAX_CTAS, EA_OPT_SCHEDULE_ORDER, EA_OPT_SKIP_ARRIVE_ONCE = 1, 2, 3, 4
EA_OPT_ITEM_DEAL = 5

# Every function the header declares, with its ctypes signature.
_SIGNATURES = {
    "attn_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "attn_fwd_masked": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p]),
    "attn_bwd": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7 + [ctypes.c_float, ctypes.c_int,
                                                                                ctypes.c_void_p]),
    "attn_bwd_masked": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7 + [ctypes.c_void_p] * 2
                        + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "attn_get_last_error": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int),
                                           ctypes.POINTER(ctypes.c_int)]),
    "attn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "attn_set_option": (ctypes.c_int, [ctypes.c_int, ctypes.c_longlong]),
    "attn_shutdown": (ctypes.c_int, []),
    "attn_version": (ctypes.c_int, []),
    "attn_fwd_fp32_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]),
    "attn_fwd_decode": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
}

_lib = None
_lock = threading.Lock()


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = status_string(status)
        super().__init__(f"{what}: {msg}" if what else msg)


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and return the library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with `python -m exact_io_aware_78_b200.build` "
                    "(nvcc, sm_100a); there is no fallback implementation")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().attn_status_string(int(status)).decode()


_DTYPES = {torch.bfloat16: EA_BF16, torch.float8_e4m3fn: EA_FP8_E4M3, torch.float32: EA_FP32}


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
             causal: bool = False, window: int = 0, scale: Optional[float] = None,
             q_scale: Optional[torch.Tensor] = None, k_scale: Optional[torch.Tensor] = None,
             v_scale: Optional[torch.Tensor] = None, stream=None) -> None:
    """Queue O, LSE = attention(q, k, v) on `stream` (default: the current
    stream).  q [B,N,Hq,d], k/v [B,N,Hkv,d], o [B,N,Hq,d], lse [B,Hq,N] fp32,
    all contiguous CUDA tensors on one device."""
    _forward_call(q, k, v, o, lse, causal, window, None, None, scale, q_scale, k_scale, v_scale, stream)


def attn_fwd_masked(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                    key_lo: torch.Tensor, key_hi: torch.Tensor, causal: bool = False, window: int = 0,
                    scale: Optional[float] = None, q_scale: Optional[torch.Tensor] = None,
                    k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
                    stream=None) -> None:
    """attn_fwd with per-row key ranges: query row i of batch b also needs
    key_lo[b, i] <= j < key_hi[b, i] (int32 [B, N] CUDA tensors, shared by
    all heads)."""
    _forward_call(q, k, v, o, lse, causal, window, key_lo, key_hi, scale, q_scale, k_scale, v_scale, stream)


def _forward_call(q, k, v, o, lse, causal, window, key_lo, key_hi, scale, q_scale, k_scale, v_scale, stream):
    lib = load_library()
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, N, H, d]")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError(f"unsupported or mixed input dtypes {q.dtype}, {k.dtype}, {v.dtype}")
    dtype = _DTYPES[q.dtype]
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if tuple(k.shape) != (B, N, Hkv, d) or tuple(v.shape) != (B, N, Hkv, d):
        raise ValueError("k and v must be [B, N, Hkv, d] matching q")
    want_o = torch.float32 if dtype == EA_FP32 else torch.bfloat16
    if tuple(o.shape) != (B, N, Hq, d) or o.dtype != want_o:
        raise ValueError(f"o must be [B, N, Hq, d] {want_o}")
    if tuple(lse.shape) != (B, Hq, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be [B, Hq, N] float32")
    devs = {t.device for t in (q, k, v, o, lse)}
    if len(devs) != 1:
        raise ValueError("all tensors must be on one device")
    if scale is None:
        scale = d ** -0.5
    for name, t in (("q_scale", q_scale), ("k_scale", k_scale), ("v_scale", v_scale)):
        if t is not None and (not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    if (key_lo is None) != (key_hi is None):
        raise ValueError("key_lo and key_hi come together")
    for name, t in (("key_lo", key_lo), ("key_hi", key_hi)):
        if t is not None and (not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous()
                              or tuple(t.shape) != (B, N) or t.device != q.device):
            raise ValueError(f"{name} must be a contiguous int32 [B, N] tensor on q's device")
    device = q.device
    with torch.cuda.device(device):
        if key_lo is None:
            st = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              B, Hq, Hkv, N, d, int(bool(causal)), int(window), float(scale), dtype,
                              _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _stream_handle(stream, device))
        else:
            st = lib.attn_fwd_masked(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                     B, Hq, Hkv, N, d, int(bool(causal)), int(window), key_lo.data_ptr(),
                                     key_hi.data_ptr(), float(scale), dtype, _ptr(q_scale), _ptr(k_scale),
                                     _ptr(v_scale), _stream_handle(stream, device))
    if st != EA_OK:
        raise AttnError(st, "attn_fwd" if key_lo is None else "attn_fwd_masked")


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, window: int = 0,
            scale: Optional[float] = None, q_scale: Optional[torch.Tensor] = None,
            k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
            stream=None, key_lo: Optional[torch.Tensor] = None,
            key_hi: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Allocate O and LSE on q's device and run attn_fwd (attn_fwd_masked
    when per-row key ranges are given); returns (O, LSE)."""
    B, N, Hq, d = q.shape
    o = torch.empty((B, N, Hq, d), device=q.device,
                    dtype=torch.float32 if q.dtype == torch.float32 else torch.bfloat16)
    lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    _forward_call(q, k, v, o, lse, causal, window, key_lo, key_hi, scale, q_scale, k_scale, v_scale, stream)
    return o, lse


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
             dout: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor, causal: bool = False,
             window: int = 0, scale: Optional[float] = None, stream=None) -> None:
    """Queue dQ, dK, dV = the backward of attn_fwd (bf16) on `stream`.
    q, o, dout, dq [B,N,Hq,d]; k, v, dk, dv [B,N,Hkv,d]; lse [B,Hq,N] fp32;
    all contiguous CUDA tensors on one device; o and lse from the forward."""
    _backward_call(q, k, v, o, lse, dout, dq, dk, dv, causal, window, None, None, scale, stream)


def attn_bwd_masked(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                    dout: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor, key_lo: torch.Tensor,
                    key_hi: torch.Tensor, causal: bool = False, window: int = 0, scale: Optional[float] = None,
                    stream=None) -> None:
    """attn_bwd for a forward with per-row key ranges (int32 [B, N] CUDA
    tensors, the ones given to attn_fwd_masked)."""
    _backward_call(q, k, v, o, lse, dout, dq, dk, dv, causal, window, key_lo, key_hi, scale, stream)


def _backward_call(q, k, v, o, lse, dout, dq, dk, dv, causal, window, key_lo, key_hi, scale, stream):
    lib = load_library()
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, N, H, d]")
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    want = {"q": (q, (B, N, Hq, d)), "k": (k, (B, N, Hkv, d)), "v": (v, (B, N, Hkv, d)), "o": (o, (B, N, Hq, d)),
            "dout": (dout, (B, N, Hq, d)), "dq": (dq, (B, N, Hq, d)), "dk": (dk, (B, N, Hkv, d)),
            "dv": (dv, (B, N, Hkv, d))}
    for name, (t, shape) in want.items():
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16 or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor of shape {shape}")
    if not lse.is_cuda or lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 CUDA tensor [B, Hq, N]")
    if len({t.device for t in (q, k, v, o, lse, dout, dq, dk, dv)}) != 1:
        raise ValueError("all tensors must be on one device")
    if (key_lo is None) != (key_hi is None):
        raise ValueError("key_lo and key_hi come together")
    for name, t in (("key_lo", key_lo), ("key_hi", key_hi)):
        if t is not None and (not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous()
                              or tuple(t.shape) != (B, N) or t.device != q.device):
            raise ValueError(f"{name} must be a contiguous int32 [B, N] tensor on q's device")
    if scale is None:
        scale = d ** -0.5
    device = q.device
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, N, d, int(bool(causal)), int(window))
    with torch.cuda.device(device):
        if key_lo is None:
            st = lib.attn_bwd(*ptrs, float(scale), EA_BF16, _stream_handle(stream, device))
        else:
            st = lib.attn_bwd_masked(*ptrs, key_lo.data_ptr(), key_hi.data_ptr(), float(scale), EA_BF16,
                                     _stream_handle(stream, device))
    if st != EA_OK:
        raise AttnError(st, "attn_bwd" if key_lo is None else "attn_bwd_masked")


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
             dout: torch.Tensor, causal: bool = False, window: int = 0, scale: Optional[float] = None,
             stream=None, key_lo: Optional[torch.Tensor] = None,
             key_hi: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Allocate dQ, dK, dV on q's device and run attn_bwd (attn_bwd_masked
    with per-row key ranges); returns them."""
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    _backward_call(q, k, v, o, lse, dout, dq, dk, dv, causal, window, key_lo, key_hi, scale, stream)
    return dq, dk, dv


def attn_fwd_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                    causal: bool = True, window: int = 0, scale: Optional[float] = None, num_splits: int = 0,
                    stream=None) -> None:
    """Queue O, LSE for Nq new query rows against Nk >= Nq cached keys on
    `stream`.  q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d], o [B,Nq,Hq,d] bf16,
    lse [B,Hq,Nq] fp32, contiguous CUDA tensors on one device; query row i is
    the token at position Nk - Nq + i.  num_splits = 0: the tensor-core
    kernel (up to 32 query rows per kv head); > 0: the CUDA-core kernel with
    that many key ranges per (batch, kv head) (up to 8 rows)."""
    lib = load_library()
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, N, H, d]")
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype or o.dtype != q.dtype:
        raise ValueError("q, k, v, o must be bfloat16")
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Nk, Hkv, d) or tuple(v.shape) != (B, Nk, Hkv, d):
        raise ValueError("k and v must be [B, Nk, Hkv, d] matching q")
    if tuple(o.shape) != (B, Nq, Hq, d):
        raise ValueError("o must be [B, Nq, Hq, d]")
    if tuple(lse.shape) != (B, Hq, Nq) or lse.dtype != torch.float32:
        raise ValueError("lse must be [B, Hq, Nq] float32")
    if len({t.device for t in (q, k, v, o, lse)}) != 1:
        raise ValueError("all tensors must be on one device")
    if scale is None:
        scale = d ** -0.5
    with torch.cuda.device(q.device):
        st = lib.attn_fwd_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq,
                                 Hkv, Nq, Nk, d, int(bool(causal)), int(window), float(scale), EA_BF16,
                                 int(num_splits), _stream_handle(stream, q.device))
    if st != EA_OK:
        raise AttnError(st, "attn_fwd_decode")


def forward_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, window: int = 0,
                   scale: Optional[float] = None, num_splits: int = 0,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Allocate O and LSE on q's device and run attn_fwd_decode."""
    B, Nq, Hq, d = q.shape
    o = torch.empty((B, Nq, Hq, d), device=q.device, dtype=torch.bfloat16)
    lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32)
    attn_fwd_decode(q, k, v, o, lse, causal, window, scale, num_splits, stream)
    return o, lse


def attn_get_last_error(stream=None, device=None) -> Tuple[int, int, int]:
    """Synchronise the stream and read/clear the device error word.
    Returns (status, device_code, site)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    code = ctypes.c_int(0)
    site = ctypes.c_int(0)
    with torch.cuda.device(dev):
        st = lib.attn_get_last_error(_stream_handle(stream, dev), ctypes.byref(code), ctypes.byref(site))
    return st, code.value, site.value


def attn_set_option(option: int, value: int) -> None:
    st = load_library().attn_set_option(int(option), int(value))
    if st != EA_OK:
        raise AttnError(st, "attn_set_option")


def attn_shutdown() -> None:
    st = load_library().attn_shutdown()
    if st != EA_OK:
        raise AttnError(st, "attn_shutdown")


def attn_version() -> int:
    return load_library().attn_version()


def attn_status_string(status: int) -> str:
    return status_string(status)
