"""Exact fused attention for NVIDIA B200 (sm_100a): Python binding of ``include/fa.h``.

This module only marshals arguments: it checks tensor shapes, dtypes and devices, takes raw
device pointers and the current CUDA stream from PyTorch, and calls the C ABI in
``libfa.so`` through ctypes.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback.  If the library is missing or fails to load,
importing this module raises ``ImportError``.

Build the library with ``python io_aware_exact_16_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python io_aware_exact_16_b200/build.py`")
try:
    _lib = ctypes.CDLL(LIB_PATH)
except OSError as exc:  # pragma: no cover
    raise ImportError(f"cannot load {LIB_PATH}: {exc}") from exc

_vp = ctypes.c_void_p
_i = ctypes.c_int


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declares the C signatures of include/fa.h on a loaded library handle."""
    lib.fa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, ctypes.c_float, _i, _vp, _vp]
    lib.fa_fwd.restype = _i
    lib.fa_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                           ctypes.c_float, _i, _vp, _vp, ctypes.c_size_t, _vp]
    lib.fa_bwd.restype = _i
    lib.fa_fwd_gqa.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _i, _vp,
                               _vp]
    lib.fa_fwd_gqa.restype = _i
    lib.fa_bwd_gqa.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                               ctypes.c_float, _i, _vp, _vp, ctypes.c_size_t, _vp]
    lib.fa_bwd_gqa.restype = _i
    lib.fa_fwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                  ctypes.c_float, _i, _vp]
    lib.fa_fwd_varlen.restype = _i
    lib.fa_bwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                  _i, _i, ctypes.c_float, _i, _vp, ctypes.c_size_t, _vp]
    lib.fa_bwd_varlen.restype = _i
    lib.fa_decode_num_splits.argtypes = [_i, _i, _i, _i, _i, _i, _i]
    lib.fa_decode_num_splits.restype = _i
    lib.fa_decode_workspace_size.argtypes = [_i, _i, _i, _i, _i]
    lib.fa_decode_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                  ctypes.c_float, _i, _i, _vp, ctypes.c_size_t, _vp]
    lib.fa_fwd_decode.restype = _i
    lib.fa_fwd_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                               ctypes.c_float, _i, _vp, _vp]
    lib.fa_fwd_fp8.restype = _i
    lib.fa_bwd_workspace_size.argtypes = [_i, _i, _i, _i]
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_check_device_error.argtypes = [_vp]
    lib.fa_check_device_error.restype = _i
    lib.fa_set_kernel_timing_events.argtypes = [_vp, _vp]
    lib.fa_set_kernel_timing_events.restype = None
    lib.fa_selftest_bounds.argtypes = [_vp, _i, _i, _vp]
    lib.fa_selftest_bounds.restype = _i
    lib.fa_debug_checks.argtypes = []
    lib.fa_debug_checks.restype = _i
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_void_p]
    lib.fa_selftest_wait_timeout.restype = _i
    lib.fa_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.fa_set_wait_timeout_ns.restype = None
    lib.fa_status_string.argtypes = [_i]
    lib.fa_status_string.restype = ctypes.c_char_p
    return lib


_bind(_lib)

# Every symbol include/fa.h declares.
EXPORTED = ("fa_fwd", "fa_bwd", "fa_fwd_gqa", "fa_bwd_gqa", "fa_fwd_varlen", "fa_bwd_varlen",
            "fa_decode_num_splits", "fa_decode_workspace_size", "fa_fwd_decode",
            "fa_fwd_fp8", "fa_bwd_workspace_size",
            "fa_check_device_error", "fa_selftest_wait_timeout", "fa_selftest_bounds",
            "fa_debug_checks", "fa_set_wait_timeout_ns",
            "fa_set_kernel_timing_events",
            "fa_status_string",
            "fa_bwd_noalloc")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE = range(6)


class FAError(RuntimeError):
    """A non-FA_OK status from the library."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def status_string(status: int) -> str:
    return _lib.fa_status_string(int(status)).decode()


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_qkv(name: str, t: torch.Tensor, shape, device) -> None:
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _seqlens_ptr(seqlens: Optional[torch.Tensor], B: int, device) -> int:
    if seqlens is None:
        return 0
    if seqlens.dtype != torch.int32 or seqlens.device != device or tuple(seqlens.shape) != (B,):
        raise ValueError("seqlens must be an int32 tensor of shape [B] on the inputs' device")
    if not seqlens.is_contiguous():
        raise ValueError("seqlens must be contiguous")
    return seqlens.data_ptr()


def _kv_heads(q: torch.Tensor, k: torch.Tensor) -> int:
    """Key/value heads of k ([B, H_kv, N, d]); H_kv must divide q's H (grouped-query attention)."""
    if k.dim() != 4:
        raise ValueError(f"k must be [B, H_kv, N, d], got shape {tuple(k.shape)}")
    H, H_kv = q.shape[1], k.shape[1]
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError(f"key/value heads {H_kv} must divide query heads {H}")
    return H_kv


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
            seqlens: Optional[torch.Tensor] = None, scale: Optional[float] = None,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """``fa_fwd_gqa`` (``fa_fwd`` when k, v have as many heads as q): returns
    (O bf16 [B, H, N, d], lse fp32 [B, H, N]) on q's device and current stream.
    k and v may have fewer heads, [B, H_kv, N, d] with H % H_kv == 0."""
    B, H, N, d = q.shape
    dev = q.device
    H_kv = _kv_heads(q, k)
    _check_qkv("q", q, (B, H, N, d), dev)
    for name, t in (("k", k), ("v", v)):
        _check_qkv(name, t, (B, H_kv, N, d), dev)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_qkv("out", out, (B, H, N, d), dev)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    elif lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [B, H, N]")
    sc = float(scale) if scale is not None else 1.0 / (d ** 0.5)
    st = _lib.fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                         B, H, H_kv, N, d, sc, int(bool(causal)), _seqlens_ptr(seqlens, B, dev),
                         _stream_handle(dev))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_gqa")
    return out, lse


def bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.fa_bwd_workspace_size(B, H, N, d))


def backward(q, k, v, o, do, lse, causal: bool = False, seqlens: Optional[torch.Tensor] = None,
             scale: Optional[float] = None, dq=None, dk=None, dv=None,
             workspace: Optional[torch.Tensor] = None):
    """``fa_bwd_gqa`` (``fa_bwd`` when k, v have as many heads as q): returns (dQ, dK, dV) in
    bf16, dK and dV shaped like k and v."""
    B, H, N, d = q.shape
    dev = q.device
    H_kv = _kv_heads(q, k)
    for name, t in (("q", q), ("o", o), ("do", do)):
        _check_qkv(name, t, (B, H, N, d), dev)
    for name, t in (("k", k), ("v", v)):
        _check_qkv(name, t, (B, H_kv, N, d), dev)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [B, H, N]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_qkv("dq", dq, (B, H, N, d), dev)
    for name, t in (("dk", dk), ("dv", dv)):
        _check_qkv(name, t, (B, H_kv, N, d), dev)
    need = bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    sc = float(scale) if scale is not None else 1.0 / (d ** 0.5)
    st = _lib.fa_bwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                         lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, H_kv,
                         N, d, sc, int(bool(causal)), _seqlens_ptr(seqlens, B, dev),
                         workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                         _stream_handle(dev))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_gqa")
    return dq, dk, dv


def _check_packed(q, k, cu_seqlens, max_seqlen):
    """Shapes of the packed layout: q [T, H, d], k [T, H_kv, d], cu_seqlens int32 [B + 1]."""
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed q, k, v must be [total, heads, d]")
    T, H, d = q.shape
    H_kv = k.shape[1]
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError(f"key/value heads {H_kv} must divide query heads {H}")
    if (cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2
            or cu_seqlens.device != q.device or not cu_seqlens.is_contiguous()):
        raise ValueError("cu_seqlens must be a contiguous int32 tensor [B + 1] on q's device")
    if int(max_seqlen) < 1:
        raise ValueError("max_seqlen must be >= 1")
    return T, H, H_kv, d, cu_seqlens.numel() - 1


def forward_varlen(q, k, v, cu_seqlens, max_seqlen: int, causal: bool = False,
                   scale: Optional[float] = None, out=None, lse=None):
    """``fa_fwd_varlen``: packed sequences, q [T, H, d], k and v [T, H_kv, d]; sequence b is
    rows cu_seqlens[b] .. cu_seqlens[b+1].  Returns (O bf16 [T, H, d], lse fp32 [H, T])."""
    T, H, H_kv, d, B = _check_packed(q, k, cu_seqlens, max_seqlen)
    dev = q.device
    _check_qkv("q", q, (T, H, d), dev)
    for name, t in (("k", k), ("v", v)):
        _check_qkv(name, t, (T, H_kv, d), dev)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_qkv("out", out, (T, H, d), dev)
    if lse is None:
        lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    elif lse.dtype != torch.float32 or tuple(lse.shape) != (H, T) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [H, T]")
    sc = float(scale) if scale is not None else 1.0 / (d ** 0.5)
    st = _lib.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr(), cu_seqlens.data_ptr(), B, int(max_seqlen), T, H,
                            H_kv, d, sc, int(bool(causal)), _stream_handle(dev))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_varlen")
    return out, lse


def backward_varlen(q, k, v, o, do, lse, cu_seqlens, max_seqlen: int, causal: bool = False,
                    scale: Optional[float] = None, dq=None, dk=None, dv=None,
                    workspace: Optional[torch.Tensor] = None):
    """``fa_bwd_varlen``: gradients of ``forward_varlen``; returns (dQ, dK, dV) in bf16 shaped
    like q, k and v."""
    T, H, H_kv, d, B = _check_packed(q, k, cu_seqlens, max_seqlen)
    dev = q.device
    for name, t in (("q", q), ("o", o), ("do", do)):
        _check_qkv(name, t, (T, H, d), dev)
    for name, t in (("k", k), ("v", v)):
        _check_qkv(name, t, (T, H_kv, d), dev)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (H, T) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [H, T]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_qkv("dq", dq, (T, H, d), dev)
    for name, t in (("dk", dk), ("dv", dv)):
        _check_qkv(name, t, (T, H_kv, d), dev)
    need = bwd_workspace_size(B, H, int(max_seqlen), d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    sc = float(scale) if scale is not None else 1.0 / (d ** 0.5)
    st = _lib.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                            cu_seqlens.data_ptr(), B, int(max_seqlen), T, H, H_kv, d, sc,
                            int(bool(causal)), workspace.data_ptr(),
                            workspace.numel() * workspace.element_size(), _stream_handle(dev))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_varlen")
    return dq, dk, dv


def _descale_ptr(t: Optional[torch.Tensor], shape, device) -> Optional[int]:
    if t is None:
        return None
    if t.dtype != torch.float32 or tuple(t.shape) != tuple(shape) or t.device != device:
        raise ValueError(f"descale factors must be float32 {tuple(shape)} on {device}")
    if not t.is_contiguous():
        raise ValueError("descale factors must be contiguous")
    return t.data_ptr()


def forward_fp8(q, k, v, q_descale=None, k_descale=None, v_descale=None, causal: bool = False,
                seqlens: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                out=None, lse=None):
    """``fa_fwd_fp8``: q [B, H, N, 128], k, v [B, H_kv, N, 128] as torch.float8_e4m3fn codes
    with per-(batch, head) float32 descale factors ([B, H], [B, H_kv], [B, H_kv]; None = 1).
    Returns (O bf16 [B, H, N, 128], lse fp32 [B, H, N])."""
    B, H, N, d = q.shape
    dev = q.device
    H_kv = k.shape[1]
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError(f"key/value heads {H_kv} must divide query heads {H}")
    for name, t, sh in (("q", q, (B, H, N, d)), ("k", k, (B, H_kv, N, d)),
                        ("v", v, (B, H_kv, N, d))):
        if t.dtype != torch.float8_e4m3fn:
            raise TypeError(f"{name} must be float8_e4m3fn, got {t.dtype}")
        if tuple(t.shape) != sh or t.device != dev or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {sh} tensor on {dev}")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    else:
        _check_qkv("out", out, (B, H, N, d), dev)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    sc = float(scale) if scale is not None else 1.0 / (d ** 0.5)
    st = _lib.fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                         _descale_ptr(q_descale, (B, H), dev), _descale_ptr(k_descale, (B, H_kv), dev),
                         _descale_ptr(v_descale, (B, H_kv), dev), out.data_ptr(), lse.data_ptr(),
                         B, H, H_kv, N, d, sc, int(bool(causal)), _seqlens_ptr(seqlens, B, dev),
                         _stream_handle(dev))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_fp8")
    return out, lse


def decode_num_splits(B: int, H: int, H_kv: int, Nq: int, N: int, d: int,
                      ragged: bool = False) -> int:
    """``fa_decode_num_splits``: ragged = per-sequence cache lengths will be passed."""
    return int(_lib.fa_decode_num_splits(B, H, H_kv, Nq, N, d, int(bool(ragged))))


def decode_workspace_size(B: int, H: int, Nq: int, d: int, splits: int) -> int:
    return int(_lib.fa_decode_workspace_size(B, H, Nq, d, splits))


def decode(q, k_cache, v_cache, cache_lens: Optional[torch.Tensor] = None, causal: bool = False,
           scale: Optional[float] = None, splits: int = 0, out=None, lse=None,
           workspace: Optional[torch.Tensor] = None):
    """``fa_fwd_decode``: q [B, H, Nq, d] against k_cache, v_cache [B, H_kv, N, d] (valid rows
    per sequence: cache_lens int32 [B], or all N).  Returns (O bf16 [B, H, Nq, d],
    lse fp32 [B, H, Nq])."""
    B, H, Nq, d = q.shape
    dev = q.device
    if k_cache.dim() != 4:
        raise ValueError("k_cache must be [B, H_kv, N, d]")
    H_kv, N = k_cache.shape[1], k_cache.shape[2]
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError(f"cache heads {H_kv} must divide query heads {H}")
    _check_qkv("q", q, (B, H, Nq, d), dev)
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _check_qkv(name, t, (B, H_kv, N, d), dev)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_qkv("out", out, (B, H, Nq, d), dev)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    elif lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Nq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [B, H, Nq]")
    if splits == 0:
        splits = decode_num_splits(B, H, H_kv, Nq, N, d, ragged=cache_lens is not None)
    splits = max(1, int(splits))
    need = int(_lib.fa_decode_workspace_size(B, H, Nq, d, splits))  # enough for any count used
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    sc = float(scale) if scale is not None else 1.0 / (d ** 0.5)
    st = _lib.fa_fwd_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                            out.data_ptr(), lse.data_ptr(), _seqlens_ptr(cache_lens, B, dev), B, H,
                            H_kv, Nq, N, d, sc, int(bool(causal)), splits, ws_ptr, ws_bytes,
                            _stream_handle(dev))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_decode")
    return out, lse


def check_device_error(device: Optional[torch.device] = None) -> int:
    """``fa_check_device_error`` on the current stream; returns the status code."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        return int(_lib.fa_check_device_error(_stream_handle(dev)))


def selftest_wait_timeout(device: Optional[torch.device] = None) -> None:
    """``fa_selftest_wait_timeout``: a kernel whose bounded wait can never be satisfied; the next
    check_device_error() returns FA_ERR_TIMEOUT."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        st = _lib.fa_selftest_wait_timeout(_stream_handle(dev))
    if st != FA_OK:
        raise FAError(st, "fa_selftest_wait_timeout")


def set_wait_timeout_ns(ns: int) -> None:
    _lib.fa_set_wait_timeout_ns(int(ns))


def time_next_kernel(start: "torch.cuda.Event", stop: "torch.cuda.Event") -> None:
    """``fa_set_kernel_timing_events``: the next call on this thread records `start` / `stop`
    (torch CUDA events created with enable_timing=True) around its main fused kernel."""
    for e in (start, stop):
        if e.cuda_event == 0:  # torch creates the CUDA event lazily, on its first record
            e.record()
    _lib.fa_set_kernel_timing_events(start.cuda_event, stop.cuda_event)


def raw_library() -> ctypes.CDLL:
    """The loaded ctypes handle of ``libfa.so`` (for direct C-ABI calls)."""
    return _lib


LIB_DEBUG_PATH = os.path.join(_HERE, "libfa_debug.so")
_debug_lib: Optional[ctypes.CDLL] = None


def debug_library() -> ctypes.CDLL:
    """The checking build ``libfa_debug.so`` (same C ABI; every plain global load and store in
    its kernels checks its index against its buffer first, records FA_ERR_INVALID_ARG and skips
    the access when out of range).  Loaded on first use; raises ImportError if it is missing."""
    global _debug_lib
    if _debug_lib is None:
        if not os.path.exists(LIB_DEBUG_PATH):
            raise ImportError(f"{LIB_DEBUG_PATH} is missing: build it with "
                              "`python io_aware_exact_16_b200/build.py`")
        _debug_lib = _bind(ctypes.CDLL(LIB_DEBUG_PATH))
    return _debug_lib


class use_library:
    """Context manager: the functions of this module call `lib` (e.g. debug_library()) instead
    of libfa.so inside the block.  Not thread-safe; meant for tests."""

    def __init__(self, lib: ctypes.CDLL):
        self.lib = lib

    def __enter__(self):
        global _lib
        self.saved, _lib = _lib, self.lib
        return self.lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved

