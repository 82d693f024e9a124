"""Python binding of libqwen3attn.so: the Qwen3 attention core (QK-Norm + RoPE + causal
GQA) on B200.

Argument marshalling only.  Every step of the computation runs in the library's CUDA
kernels; torch supplies device memory and the current stream.  There is no CPU path:
if the library is missing, or a tensor is not on a CUDA device, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqwen3attn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_WORKSPACE = range(6)

HEAD_DIM = 128

class Variant(ctypes.Structure):
    """qwen3_attn_variant: RoPE base, an optional host table of d/2 rotary frequencies,
    the attention_scaling on cos/sin, and the sliding window (0 = full causal)."""
    _fields_ = [("theta", ctypes.c_float), ("inv_freq", ctypes.POINTER(ctypes.c_double)),
                ("attention_scaling", ctypes.c_float), ("window", ctypes.c_int)]


class PagedKV(ctypes.Structure):
    """qwen3_paged_kv: page pools [num_pages, Hkv, page_size, d] bf16 and the block table
    [rows, max_blocks] int32 (device pointers)."""
    _fields_ = [("k_pages", ctypes.c_void_p), ("v_pages", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("num_pages", ctypes.c_int), ("page_size", ctypes.c_int), ("max_blocks", ctypes.c_int)]


# Every symbol include/qwen3_attn.h declares: (name, restype, argtypes)
_P, _I, _F, _Z, _U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
_V = ctypes.POINTER(Variant)
SIGNATURES = {
    "qwen3_qk_norm_rope": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _P]),
    "qwen3_attn_prefill": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _P]),
    "qwen3_attn_prefill_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _Z,
                                   _I, _I, _I, _I, _I, _F, _F, _P]),
    "qwen3_attn_prefill_chunk": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _Z,
                                      _I, _I, _I, _I, _I, _F, _F, _P]),
    "qwen3_attn_decode": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _P, _Z, _P]),
    "qwen3_attn_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _P]),
    "qwen3_qk_norm_rope_variant": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _V, _F, _P]),
    "qwen3_attn_prefill_variant": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _Z,
                                        _I, _I, _I, _I, _I, _V, _F, _P]),
    "qwen3_attn_decode_variant": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _V, _F, _P, _Z,
                                       _P]),
    "qwen3_attn_decode_paged": (_I, [_P, _P, _P, _P, _P, ctypes.POINTER(PagedKV), _P, _P, _P, _I, _I, _I, _I, _V, _F,
                                     _P, _Z, _P]),
    "qwen3_attn_prefill_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(PagedKV), _I, _P, _Z,
                                      _I, _I, _I, _I, _I, _V, _F, _P]),
    "qwen3_attn_prefill_paged_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "qwen3_attn_prefill_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(PagedKV), _P,
                                       ctypes.c_longlong, _P, _Z, _I, _I, _I, _I, _I, _V, _F, _P]),
    "qwen3_attn_prefill_varlen_workspace_size": (_Z, [_I, _I, ctypes.c_longlong, _I, _I, _I]),
    "qwen3_qkv_proj_norm_rope": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _V, _F, _P, _Z, _P]),
    "qwen3_qkv_proj_workspace_size": (_Z, [_I]),
    "qwen3_attn_prefill_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "qwen3_attn_prefill_chunk_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "qwen3_attn_decode_workspace_size": (_Z, [_I, _I, _I, _I]),
    "qwen3_attn_kv_cache_bytes": (_Z, [_I, _I, _I, _I]),
    "qwen3_attn_status_string": (ctypes.c_char_p, [_I]),
    "qwen3_attn_device_status": (_I, [_P, _I, ctypes.POINTER(ctypes.c_int)]),
    "qwen3_attn_set_wait_limit": (_U64, [_U64]),
    "qwen3_attn_set_fault_injection": (None, [_I]),
    "qwen3_attn_set_softmax_path": (_I, [_I]),
    "qwen3_attn_set_sm_pairs": (_I, [_I]),
    "qwen3_attn_version": (ctypes.c_char_p, []),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libqwen3attn.so (built in-tree by `qwen3_qk_norm_rope_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m qwen3_qk_norm_rope_b200.build` "
                               "(there is no fallback implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class Qwen3AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def make_variant(theta: float = 1.0e6, inv_freq=None, attention_scaling: float = 1.0, window: int = 0):
    """A Variant plus the ctypes buffer its inv_freq points into (keep both alive for the call)."""
    buf = None
    if inv_freq is not None:
        vals = [float(x) for x in inv_freq]
        buf = (ctypes.c_double * len(vals))(*vals)
    v = Variant(theta, ctypes.cast(buf, ctypes.POINTER(ctypes.c_double)) if buf is not None else None,
                attention_scaling, int(window))
    return v, buf


def _is_default(inv_freq, attention_scaling, window) -> bool:
    return inv_freq is None and attention_scaling == 1.0 and window == 0


def status_string(status: int) -> str:
    return lib().qwen3_attn_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise Qwen3AttnError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple, device: torch.device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device or t.device.type != "cuda":
        raise ValueError(f"{name} must be on {device} (CUDA); got {t.device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}; got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}; got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def prefill_workspace_size(B: int, T: int, Hq: int, Hkv: int, d: int = HEAD_DIM) -> int:
    return int(lib().qwen3_attn_prefill_workspace_size(B, T, Hq, Hkv, d))


def prefill_chunk_workspace_size(B: int, start: int, T: int, Hq: int, Hkv: int, d: int = HEAD_DIM) -> int:
    """Workspace of a chunk over `start` cached tokens, room for a key-axis split included."""
    return int(lib().qwen3_attn_prefill_chunk_workspace_size(B, start, T, Hq, Hkv, d))


def prefill_paged_workspace_size(B: int, start: int, T: int, Hq: int, Hkv: int, d: int = HEAD_DIM) -> int:
    return int(lib().qwen3_attn_prefill_paged_workspace_size(B, start, T, Hq, Hkv, d))


def _paged(k_pages, v_pages, block_table, dev, Hkv, d):
    num_pages, _, page_size, _ = k_pages.shape
    _need(k_pages, "k_pages", torch.bfloat16, (num_pages, Hkv, page_size, d), dev)
    _need(v_pages, "v_pages", torch.bfloat16, (num_pages, Hkv, page_size, d), dev)
    _need(block_table, "block_table", torch.int32, tuple(block_table.shape), dev)
    if block_table.dim() != 2 or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous [rows, max_blocks] int32 tensor")
    return PagedKV(_ptr(k_pages), _ptr(v_pages), _ptr(block_table), num_pages, page_size, block_table.shape[1])


def decode_workspace_size(N: int, Hq: int, Lmax: int, d: int = HEAD_DIM) -> int:
    return int(lib().qwen3_attn_decode_workspace_size(N, Hq, d, Lmax))


def kv_cache_bytes(N: int, Hkv: int, Lmax: int, d: int = HEAD_DIM) -> int:
    return int(lib().qwen3_attn_kv_cache_bytes(N, Hkv, Lmax, d))


def qk_norm_rope(x, w, pos, dst, v_src=None, v_dst=None, *, write_at_pos: bool = False,
                 theta: float = 1.0e6, eps: float = 1.0e-6, inv_freq=None,
                 attention_scaling: float = 1.0) -> torch.Tensor:
    """QK-Norm + RoPE of x [B,T,H,d] into dst [B,H,Tcap,d] (row t, or row pos[b,t] when
    write_at_pos); optionally copies v_src [B,T,H,d] to v_dst at the same slots.  inv_freq
    (d/2 values) and attention_scaling select another rope type."""
    dev = x.device
    B, T, H, d = x.shape
    Tcap = dst.shape[2]
    _need(x, "x", torch.bfloat16, (B, T, H, d), dev)
    _need(w, "w", torch.float32, (d,), dev)
    _need(pos, "pos", torch.int32, (B, T), dev)
    _need(dst, "dst", torch.bfloat16, (B, H, Tcap, d), dev)
    if v_src is not None:
        _need(v_src, "v_src", torch.bfloat16, (B, T, H, d), dev)
        _need(v_dst, "v_dst", torch.bfloat16, (B, H, Tcap, d), dev)
    if _is_default(inv_freq, attention_scaling, 0):
        _check(lib().qwen3_qk_norm_rope(_ptr(x), _ptr(w), _ptr(pos), _ptr(dst), _ptr(v_src), _ptr(v_dst),
                                        B, T, H, d, Tcap, int(write_at_pos), theta, eps, _stream(dev)),
               "qwen3_qk_norm_rope")
    else:
        var, _keep = make_variant(theta, inv_freq, attention_scaling, 0)
        _check(lib().qwen3_qk_norm_rope_variant(_ptr(x), _ptr(w), _ptr(pos), _ptr(dst), _ptr(v_src), _ptr(v_dst),
                                                B, T, H, d, Tcap, int(write_at_pos), ctypes.byref(var), eps,
                                                _stream(dev)),
               "qwen3_qk_norm_rope_variant")
    return dst


def prefill(q, k, v, q_norm_w, k_norm_w, pos, *, theta: float = 1.0e6, eps: float = 1.0e-6,
            out=None, lse=None, k_cache=None, v_cache=None, workspace=None, window: int = 0, inv_freq=None,
            attention_scaling: float = 1.0):
    """Causal GQA prefill with the QK-Norm+RoPE prologue.  q [B,T,Hq,d], k/v [B,T,Hkv,d] bf16,
    gains [d] fp32, pos [B,T] int32.  Returns out [B,T,Hq,d] bf16 (and writes lse [B,Hq,T]
    fp32 and the caches [B,Hkv,Tcap,d] when given)."""
    if (k_cache is None) != (v_cache is None):
        raise ValueError("k_cache and v_cache are given together or not at all")
    dev = q.device
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(q, "q", torch.bfloat16, (B, T, Hq, d), dev)
    _need(k, "k", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(v, "v", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(pos, "pos", torch.int32, (B, T), dev)
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (B, T, Hq, d), dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq, T), dev)
    Tcap = 0
    if k_cache is not None or v_cache is not None:
        Tcap = k_cache.shape[2]
        _need(k_cache, "k_cache", torch.bfloat16, (B, Hkv, Tcap, d), dev)
        _need(v_cache, "v_cache", torch.bfloat16, (B, Hkv, Tcap, d), dev)
    if workspace is None:
        workspace = torch.empty(prefill_workspace_size(B, T, Hq, Hkv, d), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    if _is_default(inv_freq, attention_scaling, window):
        _check(lib().qwen3_attn_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(pos),
                                           _ptr(out), _ptr(lse), _ptr(k_cache), _ptr(v_cache), Tcap,
                                           _ptr(workspace), ws_bytes, B, T, Hq, Hkv, d, theta, eps, _stream(dev)),
               "qwen3_attn_prefill_ex")
    else:
        var, _keep = make_variant(theta, inv_freq, attention_scaling, window)
        _check(lib().qwen3_attn_prefill_variant(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w),
                                                _ptr(pos), _ptr(out), _ptr(lse), _ptr(k_cache), _ptr(v_cache), 0,
                                                Tcap, _ptr(workspace), ws_bytes, B, T, Hq, Hkv, d,
                                                ctypes.byref(var), eps, _stream(dev)),
               "qwen3_attn_prefill_variant")
    return out


def prefill_chunk(q, k, v, q_norm_w, k_norm_w, pos, k_cache, v_cache, start: int, *, theta: float = 1.0e6,
                  eps: float = 1.0e-6, out=None, lse=None, workspace=None, window: int = 0, inv_freq=None,
                  attention_scaling: float = 1.0):
    """Chunked prefill: T new tokens per batch row over caches [B,Hkv,Tcap,d] that already
    hold `start` tokens.  The new keys (normed, rotated) and values are written to slots
    start..start+T-1, and new token i attends to keys 0..start+i.  Returns out [B,T,Hq,d]."""
    dev = q.device
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(q, "q", torch.bfloat16, (B, T, Hq, d), dev)
    _need(k, "k", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(v, "v", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(pos, "pos", torch.int32, (B, T), dev)
    Tcap = k_cache.shape[2]
    _need(k_cache, "k_cache", torch.bfloat16, (B, Hkv, Tcap, d), dev)
    _need(v_cache, "v_cache", torch.bfloat16, (B, Hkv, Tcap, d), dev)
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (B, T, Hq, d), dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq, T), dev)
    if workspace is None:
        workspace = torch.empty(prefill_chunk_workspace_size(B, start, T, Hq, Hkv, d), dtype=torch.uint8,
                                device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    if _is_default(inv_freq, attention_scaling, window):
        _check(lib().qwen3_attn_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w),
                                              _ptr(pos), _ptr(out), _ptr(lse), _ptr(k_cache), _ptr(v_cache),
                                              int(start), Tcap, _ptr(workspace), ws_bytes, B, T, Hq, Hkv, d, theta,
                                              eps, _stream(dev)),
               "qwen3_attn_prefill_chunk")
    else:
        var, _keep = make_variant(theta, inv_freq, attention_scaling, window)
        _check(lib().qwen3_attn_prefill_variant(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w),
                                                _ptr(pos), _ptr(out), _ptr(lse), _ptr(k_cache), _ptr(v_cache),
                                                int(start), Tcap, _ptr(workspace), ws_bytes, B, T, Hq, Hkv, d,
                                                ctypes.byref(var), eps, _stream(dev)),
               "qwen3_attn_prefill_variant")
    return out


def prefill_simple(q, k, v, q_norm_w, k_norm_w, pos, *, theta: float = 1.0e6, eps: float = 1.0e-6, out=None):
    """qwen3_attn_prefill: the call that obtains its own stream-ordered scratch."""
    dev = q.device
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(q, "q", torch.bfloat16, (B, T, Hq, d), dev)
    _need(k, "k", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(v, "v", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(pos, "pos", torch.int32, (B, T), dev)
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (B, T, Hq, d), dev)
    _check(lib().qwen3_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(pos),
                                    _ptr(out), B, T, Hq, Hkv, d, theta, eps, _stream(dev)), "qwen3_attn_prefill")
    return out


def decode(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, *, theta: float = 1.0e6,
           eps: float = 1.0e-6, out=None, lse=None, workspace=None, window: int = 0, inv_freq=None,
           attention_scaling: float = 1.0):
    """One decode step.  q [N,Hq,d], k_new/v_new [N,Hkv,d] bf16 raw; caches [N,Hkv,Lmax,d]
    bf16 (slot L = cache_lens[n] is written); cache_lens [N] int32 (not advanced).
    Returns out [N,Hq,d] bf16."""
    dev = q.device
    N, Hq, d = q.shape
    Hkv = k_new.shape[1]
    Lmax = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (N, Hq, d), dev)
    _need(k_new, "k_new", torch.bfloat16, (N, Hkv, d), dev)
    _need(v_new, "v_new", torch.bfloat16, (N, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(k_cache, "k_cache", torch.bfloat16, (N, Hkv, Lmax, d), dev)
    _need(v_cache, "v_cache", torch.bfloat16, (N, Hkv, Lmax, d), dev)
    _need(cache_lens, "cache_lens", torch.int32, (N,), dev)
    if out is None:
        out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (N, Hq, d), dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, (N, Hq), dev)
    if workspace is None:
        workspace = torch.empty(decode_workspace_size(N, Hq, Lmax, d), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    if _is_default(inv_freq, attention_scaling, window):
        _check(lib().qwen3_attn_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_norm_w), _ptr(k_norm_w),
                                       _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), _ptr(out), _ptr(lse),
                                       N, Hq, Hkv, d, Lmax, theta, eps, _ptr(workspace), ws_bytes, _stream(dev)),
               "qwen3_attn_decode")
    else:
        var, _keep = make_variant(theta, inv_freq, attention_scaling, window)
        _check(lib().qwen3_attn_decode_variant(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_norm_w), _ptr(k_norm_w),
                                               _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), _ptr(out), _ptr(lse),
                                               N, Hq, Hkv, d, Lmax, ctypes.byref(var), eps, _ptr(workspace),
                                               ws_bytes, _stream(dev)),
               "qwen3_attn_decode_variant")
    return out


def decode_paged(q, k_new, v_new, q_norm_w, k_norm_w, k_pages, v_pages, block_table, cache_lens, *,
                 theta: float = 1.0e6, eps: float = 1.0e-6, out=None, lse=None, workspace=None, window: int = 0,
                 inv_freq=None, attention_scaling: float = 1.0):
    """One decode step over a paged cache: pools [num_pages, Hkv, page_size, d] bf16 and the
    block table [N, max_blocks] int32.  The new key and value go to key index cache_lens[n]."""
    dev = q.device
    N, Hq, d = q.shape
    Hkv = k_new.shape[1]
    _need(q, "q", torch.bfloat16, (N, Hq, d), dev)
    _need(k_new, "k_new", torch.bfloat16, (N, Hkv, d), dev)
    _need(v_new, "v_new", torch.bfloat16, (N, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(cache_lens, "cache_lens", torch.int32, (N,), dev)
    kv = _paged(k_pages, v_pages, block_table, dev, Hkv, d)
    if out is None:
        out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (N, Hq, d), dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, (N, Hq), dev)
    if workspace is None:
        workspace = torch.empty(decode_workspace_size(N, Hq, kv.max_blocks * kv.page_size, d), dtype=torch.uint8,
                                device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    var, _keep = make_variant(theta, inv_freq, attention_scaling, window)
    _check(lib().qwen3_attn_decode_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_norm_w), _ptr(k_norm_w),
                                         ctypes.byref(kv), _ptr(cache_lens), _ptr(out), _ptr(lse), N, Hq, Hkv, d,
                                         ctypes.byref(var), eps, _ptr(workspace), ws_bytes, _stream(dev)),
           "qwen3_attn_decode_paged")
    return out


def prefill_paged(q, k, v, q_norm_w, k_norm_w, pos, k_pages, v_pages, block_table, start: int, *,
                  theta: float = 1.0e6, eps: float = 1.0e-6, out=None, lse=None, workspace=None, window: int = 0,
                  inv_freq=None, attention_scaling: float = 1.0):
    """Chunked prefill over a paged cache (start = 0 for a fresh prompt): the new keys and
    values are written into their pages; returns out [B,T,Hq,d]."""
    dev = q.device
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(q, "q", torch.bfloat16, (B, T, Hq, d), dev)
    _need(k, "k", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(v, "v", torch.bfloat16, (B, T, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(pos, "pos", torch.int32, (B, T), dev)
    kv = _paged(k_pages, v_pages, block_table, dev, Hkv, d)
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (B, T, Hq, d), dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq, T), dev)
    if workspace is None:
        workspace = torch.empty(prefill_paged_workspace_size(B, start, T, Hq, Hkv, d), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    var, _keep = make_variant(theta, inv_freq, attention_scaling, window)
    _check(lib().qwen3_attn_prefill_paged(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(pos),
                                          _ptr(out), _ptr(lse), ctypes.byref(kv), int(start), _ptr(workspace),
                                          ws_bytes, B, T, Hq, Hkv, d, ctypes.byref(var), eps, _stream(dev)),
           "qwen3_attn_prefill_paged")
    return out


def prefill_varlen_workspace_size(B: int, N: int, Hq: int, Hkv: int, key_cap: int = 0, d: int = HEAD_DIM) -> int:
    return int(lib().qwen3_attn_prefill_varlen_workspace_size(B, N, key_cap, Hq, Hkv, d))


def prefill_varlen(q, k, v, q_norm_w, k_norm_w, pos, cu_seqlens, *, k_pages=None, v_pages=None, block_table=None,
                   ctx_lens=None, key_cap: int = 0, theta: float = 1.0e6, eps: float = 1.0e-6, out=None, lse=None,
                   workspace=None, window: int = 0, inv_freq=None, attention_scaling: float = 1.0):
    """Prefill of B sequences packed on one token axis: q [N,Hq,d], k/v [N,Hkv,d], pos [N],
    cu_seqlens [B+1] int32 (sequence b owns tokens cu_seqlens[b] .. cu_seqlens[b+1]-1).
    With k_pages/v_pages/block_table, a paged cache: sequence b has ctx_lens[b] cached keys
    (ctx_lens [B] int32, None = all 0), its new keys and values go to its pages, and key_cap
    must bound the sum of ctx_lens[b] + T_b.  Returns out [N,Hq,d] (rows of tokens outside
    every sequence untouched) and writes lse [Hq,N] when given."""
    dev = q.device
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.shape[0] - 1
    _need(q, "q", torch.bfloat16, (N, Hq, d), dev)
    _need(k, "k", torch.bfloat16, (N, Hkv, d), dev)
    _need(v, "v", torch.bfloat16, (N, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(pos, "pos", torch.int32, (N,), dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    kv = None
    if k_pages is not None:
        kv = _paged(k_pages, v_pages, block_table, dev, Hkv, d)
        if block_table.shape[0] < B:
            raise ValueError(f"block_table has {block_table.shape[0]} rows for {B} sequences")
        if ctx_lens is not None:
            _need(ctx_lens, "ctx_lens", torch.int32, (B,), dev)
    if out is None:
        out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (N, Hq, d), dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, (Hq, N), dev)
    if workspace is None:
        workspace = torch.empty(prefill_varlen_workspace_size(B, N, Hq, Hkv, key_cap, d), dtype=torch.uint8,
                                device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    var, _keep = make_variant(theta, inv_freq, attention_scaling, window)
    _check(lib().qwen3_attn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(pos),
                                           _ptr(cu_seqlens), _ptr(out), _ptr(lse),
                                           ctypes.byref(kv) if kv is not None else None, _ptr(ctx_lens),
                                           int(key_cap), _ptr(workspace), ws_bytes, B, N, Hq, Hkv, d,
                                           ctypes.byref(var), eps, _stream(dev)),
           "qwen3_attn_prefill_varlen")
    return out


def qkv_proj_workspace_size(M: int) -> int:
    return int(lib().qwen3_qkv_proj_workspace_size(M))


def qkv_proj_norm_rope(x, w_qkv, q_norm_w, k_norm_w, pos, Hq: int, Hkv: int, *, theta: float = 1.0e6,
                       eps: float = 1.0e-6, inv_freq=None, attention_scaling: float = 1.0, q_out=None, k_out=None,
                       v_out=None, workspace=None):
    """The merged qkv projection with QK-Norm + RoPE in its epilogue: x [M, hidden] bf16,
    w_qkv [(Hq + 2 Hkv) d, hidden] bf16, pos [M] int32.  Returns (q' [M,Hq,d], k' [M,Hkv,d],
    v [M,Hkv,d]) bf16."""
    dev = x.device
    M, hidden = x.shape
    d = HEAD_DIM
    _need(x, "x", torch.bfloat16, (M, hidden), dev)
    _need(w_qkv, "w_qkv", torch.bfloat16, ((Hq + 2 * Hkv) * d, hidden), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(pos, "pos", torch.int32, (M,), dev)
    if q_out is None:
        q_out = torch.empty((M, Hq, d), dtype=torch.bfloat16, device=dev)
    if k_out is None:
        k_out = torch.empty((M, Hkv, d), dtype=torch.bfloat16, device=dev)
    if v_out is None:
        v_out = torch.empty((M, Hkv, d), dtype=torch.bfloat16, device=dev)
    _need(q_out, "q_out", torch.bfloat16, (M, Hq, d), dev)
    _need(k_out, "k_out", torch.bfloat16, (M, Hkv, d), dev)
    _need(v_out, "v_out", torch.bfloat16, (M, Hkv, d), dev)
    if workspace is None:
        workspace = torch.empty(qkv_proj_workspace_size(M), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    var, _keep = make_variant(theta, inv_freq, attention_scaling, 0)
    _check(lib().qwen3_qkv_proj_norm_rope(_ptr(x), _ptr(w_qkv), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(pos), _ptr(q_out),
                                          _ptr(k_out), _ptr(v_out), M, hidden, Hq, Hkv, d, ctypes.byref(var), eps,
                                          _ptr(workspace), ws_bytes, _stream(dev)),
           "qwen3_qkv_proj_norm_rope")
    return q_out, k_out, v_out


NOALLOC_SCRATCH_BYTES = 48 << 20


def decode_noalloc(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, *, theta: float = 1.0e6,
                   eps: float = 1.0e-6, out=None, lse=None):
    """qwen3_attn_decode_noalloc: `decode` for callers that cannot allocate device memory.
    The split-KV partials live in the library's fixed 48 MiB device region (shared by
    every call on the device; overlapping calls race).  `out`/`lse` are still the
    caller's; pass preallocated ones to keep this call free of allocation on the Python
    side too."""
    dev = q.device
    N, Hq, d = q.shape
    Hkv = k_new.shape[1]
    Lmax = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (N, Hq, d), dev)
    _need(k_new, "k_new", torch.bfloat16, (N, Hkv, d), dev)
    _need(v_new, "v_new", torch.bfloat16, (N, Hkv, d), dev)
    _need(q_norm_w, "q_norm_w", torch.float32, (d,), dev)
    _need(k_norm_w, "k_norm_w", torch.float32, (d,), dev)
    _need(k_cache, "k_cache", torch.bfloat16, (N, Hkv, Lmax, d), dev)
    _need(v_cache, "v_cache", torch.bfloat16, (N, Hkv, Lmax, d), dev)
    _need(cache_lens, "cache_lens", torch.int32, (N,), dev)
    if out is None:
        out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (N, Hq, d), dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, (N, Hq), dev)
    _check(lib().qwen3_attn_decode_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_norm_w), _ptr(k_norm_w),
                                           _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), _ptr(out), _ptr(lse),
                                           N, Hq, Hkv, d, Lmax, theta, eps, _stream(dev)),
           "qwen3_attn_decode_noalloc")
    return out


def device_status(clear: bool = True, device=None) -> tuple[int, int]:
    """Synchronise the current stream and return (status, site) of the device status word."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    site = ctypes.c_int(0)
    st = lib().qwen3_attn_device_status(_stream(dev), int(clear), ctypes.byref(site))
    return int(st), int(site.value)


def set_wait_limit(ns: int) -> int:
    return int(lib().qwen3_attn_set_wait_limit(int(ns)))


def set_fault_injection(flags: int) -> None:
    lib().qwen3_attn_set_fault_injection(int(flags))


SOFTMAX_AUTO, SOFTMAX_RUNNING_MAX = 0, 1


def set_softmax_path(path: int) -> int:
    """Test hook: SOFTMAX_RUNNING_MAX sends every later prefill launch down the running-max
    softmax whatever its gains; SOFTMAX_AUTO (the default) lets the gains' logit bound
    choose.  Returns the previous setting."""
    old = int(lib().qwen3_attn_set_softmax_path(int(path)))
    if old < 0:
        raise ValueError(f"unknown softmax path {path}")
    return old


SM_PAIRS_AUTO, SM_PAIRS_OFF, SM_PAIRS_ALWAYS = 0, 1, 2


def set_sm_pairs(mode: int) -> int:
    """Test hook: how later qkv projections use the SMs.  SM_PAIRS_AUTO (the default) pairs
    SMs on each MMA for long K runs, SM_PAIRS_OFF keeps one SM per tile, SM_PAIRS_ALWAYS
    pairs them whatever the size.  Returns the previous setting."""
    old = int(lib().qwen3_attn_set_sm_pairs(int(mode)))
    if old < 0:
        raise ValueError(f"unknown SM-pair mode {mode}")
    return old


def version() -> str:
    return lib().qwen3_attn_version().decode()
