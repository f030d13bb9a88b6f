"""Sliding-window attention on B200: Python binding of libswa.so.

Argument marshalling only.  Every function here takes torch tensors that live
on a CUDA device, passes their data pointers and sizes to the C ABI declared
in include/swa.h (same names), and raises SwaError on any non-OK status.  All
computation happens in the library's CUDA kernels; there is no fallback: if
libswa.so is missing or cannot be loaded, every call raises.

Layouts: q/o [B,T,Hq,d], k/v [B,T,Hkv,d], lse [B,Hq,T] (fp32), ring caches
[B,Hkv,W,d], decode q/o [B,Hq,d], positions int32.

With the environment variable SWA_DEBUG=1 the debug build libswa_debug.so is
loaded instead: the same kernels with device-side checks of their tile, row
and slot indices, reported as SWA_ERR_INTERNAL by swa_get_device_status.
"""
import ctypes
import os

import torch

__all__ = [
    "SwaError", "load", "library_path", "EXPORTED",
    "swa_prefill", "swa_prefill_global", "swa_prefill_chunk", "swa_prefill_sinks", "swa_prefill_dilated",
    "swa_prefill_dilated_workspace_bytes", "swa_prefill_varlen", "swa_cache_append", "swa_decode",
    "swa_decode_sinks",
    "swa_decode_workspace_bytes", "swa_mask_export", "swa_get_device_status",
    "swa_debug_expire_wait", "swa_set_wait_limit_ns", "swa_status_string", "swa_decode_noalloc",
    "swa_cache_append_paged", "swa_decode_paged",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG = os.environ.get("SWA_DEBUG", "0") not in ("", "0")
library_path = os.path.join(_HERE, "libswa_debug.so" if DEBUG else "libswa.so")

SWA_OK, SWA_ERR_INVALID_ARG, SWA_ERR_UNSUPPORTED, SWA_ERR_CUDA, SWA_ERR_TIMEOUT = 0, 1, 2, 3, 4
SWA_ERR_INTERNAL = 5
SWA_DTYPE_F32, SWA_DTYPE_BF16 = 0, 1

# every symbol include/swa.h declares
EXPORTED = [
    "swa_prefill", "swa_prefill_global", "swa_prefill_chunk", "swa_prefill_sinks", "swa_decode_sinks",
    "swa_prefill_dilated", "swa_prefill_dilated_workspace_bytes", "swa_prefill_varlen",
    "swa_cache_append", "swa_decode_workspace_bytes",
    "swa_decode", "swa_mask_export", "swa_get_device_status", "swa_debug_expire_wait",
    "swa_set_wait_limit_ns", "swa_status_string", "swa_decode_noalloc", "swa_cache_append_paged",
    "swa_decode_paged", "swa_prefill_backward", "swa_prefill_backward_workspace_bytes",
]

_lib = None


class SwaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, swa_status_string(status), status))


def load():
    """Load libswa.so (built by decode_swa_prefill_b200.build); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError("%s not found; build it with `python -m decode_swa_prefill_b200.build%s`"
                           % (library_path, " --debug" if DEBUG else ""))
    lib = ctypes.CDLL(library_path)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.swa_prefill.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.swa_prefill_global.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, P]
    lib.swa_prefill_chunk.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.swa_prefill_sinks.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, I, P]
    lib.swa_prefill_dilated.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, P, ctypes.c_size_t, P]
    lib.swa_prefill_dilated_workspace_bytes.argtypes = [I, I, I, I, I, I, I, I]
    lib.swa_prefill_dilated_workspace_bytes.restype = ctypes.c_size_t
    lib.swa_prefill_varlen.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, P]
    lib.swa_decode_sinks.argtypes = [P, P, P, P, P, I, P, P, P, I, I, I, I, I, F, I, P, ctypes.c_size_t, P]
    lib.swa_cache_append.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P]
    lib.swa_decode_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.swa_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.swa_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, P, ctypes.c_size_t, P]
    lib.swa_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, P]
    lib.swa_cache_append_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
    lib.swa_decode_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, P, ctypes.c_size_t, P]
    lib.swa_prefill_backward.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, P,
                                         ctypes.c_size_t, P]
    lib.swa_prefill_backward_workspace_bytes.argtypes = [I, I, I]
    lib.swa_prefill_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.swa_mask_export.argtypes = [P, I, I, I, P, I, P]
    lib.swa_get_device_status.argtypes = [P]
    lib.swa_debug_expire_wait.argtypes = [I, P]
    lib.swa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.swa_set_wait_limit_ns.restype = None
    lib.swa_status_string.argtypes = [I]
    lib.swa_status_string.restype = ctypes.c_char_p
    for name in ("swa_prefill", "swa_prefill_global", "swa_prefill_chunk", "swa_prefill_sinks", "swa_decode_sinks",
                 "swa_prefill_dilated", "swa_prefill_varlen",
                 "swa_cache_append", "swa_decode",
                 "swa_decode_noalloc", "swa_mask_export", "swa_get_device_status", "swa_debug_expire_wait",
                 "swa_cache_append_paged", "swa_decode_paged", "swa_prefill_backward"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def swa_status_string(status):
    return load().swa_status_string(int(status)).decode()


def _check(status, where):
    if status != SWA_OK:
        raise SwaError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return SWA_DTYPE_BF16
    if t.dtype == torch.float32:
        return SWA_DTYPE_F32
    raise SwaError(SWA_ERR_UNSUPPORTED, "dtype %s" % t.dtype)


def _need(cond, what):
    if not cond:
        raise SwaError(SWA_ERR_INVALID_ARG, what)


def _dev_contig(*ts):
    for t in ts:
        if t is not None:
            _need(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")


def swa_prefill(q, k, v, W, scale=None, o=None, lse=None, stream=None):
    """Causal sliding-window prefill; returns o (and fills lse when given)."""
    _dev_contig(q, k, v, o, lse)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k.shape == (B, T, Hkv, d) and v.shape == k.shape, "k/v shape")
    if o is None:
        o = torch.empty_like(q)
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, Hq, Hkv, d, W,
                            float(scale), _dtype_code(q), _stream(stream))
    _check(st, "swa_prefill")
    return o


def swa_prefill_varlen(q, k, v, cu_seqlens, W, max_seqlen, scale=None, o=None, lse=None, stream=None):
    """Causal window over packed sequences q [total,Hq,d], k/v [total,Hkv,d];
    cu_seqlens int32 [nseq+1] on the device; max_seqlen is the longest
    sequence (a host integer the caller knows, like the offsets themselves).
    W is one window for every sequence (int) or one per sequence (int32
    tensor [nseq] on the device)."""
    windows = W if isinstance(W, torch.Tensor) else None
    _dev_contig(q, k, v, o, lse, cu_seqlens, windows)
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    _need(k.shape == (total, Hkv, d) and v.shape == k.shape, "k/v shape")
    _need(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1, "cu_seqlens int32 [nseq+1]")
    nseq = cu_seqlens.numel() - 1
    if windows is not None:
        _need(windows.dtype == torch.int32 and windows.shape == (nseq,), "windows int32 [nseq]")
    if o is None:
        o = torch.empty_like(q)
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens), _ptr(windows),
                                   nseq, total, int(max_seqlen), Hq, Hkv, d, 1 if windows is not None else int(W),
                                   float(scale), _dtype_code(q), _stream(stream))
    _check(st, "swa_prefill_varlen")
    return o


def swa_prefill_dilated_workspace_bytes(B, T, Hq, Hkv, d, dil, dtype=torch.bfloat16, with_lse=False):
    code = SWA_DTYPE_BF16 if dtype == torch.bfloat16 else SWA_DTYPE_F32
    return int(load().swa_prefill_dilated_workspace_bytes(B, T, Hq, Hkv, d, dil, code, int(bool(with_lse))))


def swa_prefill_dilated(q, k, v, W, dil, symmetric=False, scale=None, o=None, lse=None, workspace=None,
                        stream=None):
    """Dilated window (every dil-th key, W keys, or W//2 per side when
    symmetric); the workspace is allocated here when not given."""
    _dev_contig(q, k, v, o, lse, workspace)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k.shape == (B, T, Hkv, d) and v.shape == k.shape, "k/v shape")
    if o is None:
        o = torch.empty_like(q)
    need = swa_prefill_dilated_workspace_bytes(B, T, Hq, Hkv, d, dil, q.dtype, lse is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_prefill_dilated(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(dil), int(bool(symmetric)),
                                    B, T, Hq, Hkv, d, W, float(scale), _dtype_code(q), _ptr(workspace), ws_bytes,
                                    _stream(stream))
    _check(st, "swa_prefill_dilated")
    return o


def swa_prefill_backward_workspace_bytes(B, T, Hq):
    return int(load().swa_prefill_backward_workspace_bytes(B, T, Hq))


def swa_prefill_backward(q, k, v, o, lse, dout, W, symmetric=False, scale=None, dq=None, dk=None, dv=None,
                         workspace=None, stream=None):
    """Gradients of the window prefill (causal, or symmetric without
    globals) for the upstream gradient dout: returns dq, dk, dv.  o and lse
    are the forward call's outputs for the same q, k, v; the workspace (fp32
    [B,Hq,T]) is allocated here when not given."""
    _dev_contig(q, k, v, o, lse, dout, dq, dk, dv, workspace)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k.shape == (B, T, Hkv, d) and v.shape == k.shape, "k/v shape")
    _need(o.shape == q.shape and dout.shape == q.shape, "o/dout shape")
    _need(lse.shape == (B, Hq, T) and lse.dtype == torch.float32, "lse must be fp32 [B,Hq,T]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = swa_prefill_backward_workspace_bytes(B, T, Hq)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                     _ptr(dv), int(bool(symmetric)), B, T, Hq, Hkv, d, W, float(scale),
                                     _dtype_code(q), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "swa_prefill_backward")
    return dq, dk, dv


def swa_prefill_sinks(q, k, v, W, n_sink, scale=None, o=None, lse=None, stream=None):
    """Causal window W plus the first n_sink tokens of each sequence as
    attention sinks; returns o (and fills lse when given)."""
    _dev_contig(q, k, v, o, lse)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k.shape == (B, T, Hkv, d) and v.shape == k.shape, "k/v shape")
    if o is None:
        o = torch.empty_like(q)
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_prefill_sinks(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(n_sink), B, T, Hq, Hkv, d, W,
                                  float(scale), _dtype_code(q), _stream(stream))
    _check(st, "swa_prefill_sinks")
    return o


def swa_prefill_chunk(q, k, v, k_cache, v_cache, pos, scale=None, o=None, lse=None, stream=None):
    """Causal prefill of a chunk q/k/v [B,n,H,d] at positions pos[b].. (int32
    [B]) that reads earlier keys from the rings k_cache/v_cache [B,Hkv,W,d]
    (not yet holding the chunk); returns o (and fills lse [B,Hq,n])."""
    _dev_contig(q, k, v, o, lse, k_cache, v_cache, pos)
    B, n, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k.shape == (B, n, Hkv, d) and v.shape == k.shape, "k/v shape")
    W = k_cache.shape[2]
    _need(k_cache.shape == (B, Hkv, W, d) and v_cache.shape == k_cache.shape, "cache shape")
    _need(pos.dtype == torch.int32 and pos.shape == (B,), "pos [B] int32")
    if o is None:
        o = torch.empty_like(q)
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(pos), B, n, Hq, Hkv, d, W, float(scale), _dtype_code(q), _stream(stream))
    _check(st, "swa_prefill_chunk")
    return o


def swa_prefill_global(q, k, v, global_idx, W, scale=None, o=None, lse=None, stream=None):
    """Symmetric window (half-width W//2) plus global tokens global_idx [B,g] int32."""
    _dev_contig(q, k, v, o, lse, global_idx)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k.shape == (B, T, Hkv, d) and v.shape == k.shape, "k/v shape")
    g = 0 if global_idx is None else global_idx.shape[-1]
    if global_idx is not None:
        _need(global_idx.dtype == torch.int32 and global_idx.shape == (B, g), "global_idx [B,g] int32")
    if o is None:
        o = torch.empty_like(q)
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_prefill_global(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                   _ptr(global_idx) if g > 0 else None, g, B, T, Hq, Hkv, d, W,
                                   float(scale), _dtype_code(q), _stream(stream))
    _check(st, "swa_prefill_global")
    return o


def swa_cache_append(k_cache, v_cache, k_new, v_new, pos, slot_out=None, stream=None):
    """Write k_new/v_new [B,n,Hkv,d] into slots (pos[b]+t) mod W of the rings."""
    _dev_contig(k_cache, v_cache, k_new, v_new, pos, slot_out)
    B, Hkv, W, d = k_cache.shape
    n = k_new.shape[1]
    _need(k_new.shape == (B, n, Hkv, d) and v_new.shape == k_new.shape, "k_new/v_new shape")
    _need(pos.dtype == torch.int32 and pos.numel() == B, "pos [B] int32")
    st = load().swa_cache_append(_ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new), _ptr(pos),
                                 _ptr(slot_out), B, n, Hkv, d, W, _dtype_code(k_cache), _stream(stream))
    _check(st, "swa_cache_append")


def swa_cache_append_paged(k_pages, v_pages, k_new, v_new, pos, page_table, slot_out=None, stream=None):
    """Write k_new/v_new [B,n,Hkv,d] into ring slots (pos[b]+t) mod W of a
    paged ring: pools [num_pages,Hkv,P,d], page_table int32 [B, W/P]."""
    _dev_contig(k_pages, v_pages, k_new, v_new, pos, page_table, slot_out)
    num_pages, Hkv, P, d = k_pages.shape
    B, n = k_new.shape[0], k_new.shape[1]
    _need(k_new.shape == (B, n, Hkv, d) and v_new.shape == k_new.shape, "k_new/v_new shape")
    _need(v_pages.shape == k_pages.shape, "pool shape")
    _need(page_table.dtype == torch.int32 and page_table.dim() == 2 and page_table.shape[0] == B, "page_table")
    _need(pos.dtype == torch.int32 and pos.numel() == B, "pos [B] int32")
    W = P * page_table.shape[1]
    st = load().swa_cache_append_paged(_ptr(k_pages), _ptr(v_pages), _ptr(k_new), _ptr(v_new), _ptr(pos),
                                       _ptr(page_table), _ptr(slot_out), B, n, Hkv, d, W, P, num_pages,
                                       _dtype_code(k_pages), _stream(stream))
    _check(st, "swa_cache_append_paged")


def swa_decode_paged(q, k_pages, v_pages, page_table, pos, scale=None, o=None, lse=None, workspace=None,
                     stream=None):
    """One decode step over a paged ring (pools [num_pages,Hkv,P,d],
    page_table int32 [B, W/P]); pos[b] already appended."""
    _dev_contig(q, k_pages, v_pages, page_table, pos, o, lse, workspace)
    B, Hq, d = q.shape
    num_pages, Hkv, P = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    _need(page_table.dtype == torch.int32 and page_table.dim() == 2 and page_table.shape[0] == B, "page_table")
    _need(pos.dtype == torch.int32 and pos.numel() == B, "pos [B] int32")
    W = P * page_table.shape[1]
    if o is None:
        o = torch.empty_like(q)
    need = swa_decode_workspace_bytes(B, Hq, Hkv, d, W)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(o), _ptr(lse),
                                 _ptr(pos), B, Hq, Hkv, d, W, P, num_pages, float(scale), _dtype_code(q),
                                 _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "swa_decode_paged")
    return o


def swa_decode_workspace_bytes(B, Hq, Hkv, d, W):
    return int(load().swa_decode_workspace_bytes(B, Hq, Hkv, d, W))


def swa_decode(q, k_cache, v_cache, pos, scale=None, o=None, lse=None, workspace=None, stream=None):
    """One decode step: q [B,Hq,d] over rings [B,Hkv,W,d]; pos[b] already appended."""
    _dev_contig(q, k_cache, v_cache, pos, o, lse, workspace)
    B, Hq, d = q.shape
    Hkv, W = k_cache.shape[1], k_cache.shape[2]
    _need(pos.dtype == torch.int32 and pos.numel() == B, "pos [B] int32")
    if o is None:
        o = torch.empty_like(q)
    need = swa_decode_workspace_bytes(B, Hq, Hkv, d, W)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), _ptr(pos),
                           B, Hq, Hkv, d, W, float(scale), _dtype_code(q), _ptr(workspace),
                           ws_bytes, _stream(stream))
    _check(st, "swa_decode")
    return o


def swa_decode_sinks(q, k_cache, v_cache, k_sink, v_sink, pos, scale=None, o=None, lse=None, workspace=None,
                     stream=None):
    """swa_decode plus attention sinks: k_sink/v_sink [B,Hkv,n_sink,d] hold
    positions 0..n_sink-1 and are seen beside the window."""
    _dev_contig(q, k_cache, v_cache, k_sink, v_sink, pos, o, lse, workspace)
    B, Hq, d = q.shape
    Hkv, W = k_cache.shape[1], k_cache.shape[2]
    n_sink = k_sink.shape[2]
    _need(k_sink.shape == (B, Hkv, n_sink, d) and v_sink.shape == k_sink.shape, "sink cache shape")
    _need(pos.dtype == torch.int32 and pos.numel() == B, "pos [B] int32")
    if o is None:
        o = torch.empty_like(q)
    need = swa_decode_workspace_bytes(B, Hq, Hkv, d, W)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_decode_sinks(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_sink), _ptr(v_sink), n_sink,
                                 _ptr(o), _ptr(lse), _ptr(pos), B, Hq, Hkv, d, W, float(scale), _dtype_code(q),
                                 _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "swa_decode_sinks")
    return o


NOALLOC_SCRATCH_BYTES = 16 << 20


def swa_decode_noalloc(q, k_cache, v_cache, pos, scale=None, o=None, lse=None, stream=None):
    """swa_decode without a workspace, for callers that cannot allocate device
    memory while decoding.  Its scratch is a 16 MiB static device array shared
    by all calls (overlapping calls on one GPU race); sizes needing more are
    rejected.  `o` is allocated here only when not given."""
    _dev_contig(q, k_cache, v_cache, pos, o, lse)
    B, Hq, d = q.shape
    Hkv, W = k_cache.shape[1], k_cache.shape[2]
    _need(pos.dtype == torch.int32 and pos.numel() == B, "pos [B] int32")
    need = swa_decode_workspace_bytes(B, Hq, Hkv, d, W)
    if need > NOALLOC_SCRATCH_BYTES:
        raise SwaError(SWA_ERR_UNSUPPORTED, "swa_decode_noalloc: these sizes need %d bytes of scratch, "
                       "above the %d-byte static array" % (need, NOALLOC_SCRATCH_BYTES))
    if o is None:
        o = torch.empty_like(q)
    scale = d ** -0.5 if scale is None else scale
    st = load().swa_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), _ptr(pos),
                                   B, Hq, Hkv, d, W, float(scale), _dtype_code(q), _stream(stream))
    _check(st, "swa_decode_noalloc")
    return o


def swa_mask_export(T, W, symmetric=False, global_idx=None, device=None, stream=None):
    """[T,T] uint8 visibility mask from the kernels' own predicate (debug)."""
    device = device or torch.device("cuda")
    mask = torch.empty((T, T), dtype=torch.uint8, device=device)
    g = 0 if global_idx is None else global_idx.numel()
    st = load().swa_mask_export(_ptr(mask), T, W, int(bool(symmetric)),
                                _ptr(global_idx) if g > 0 else None, g, _stream(stream))
    _check(st, "swa_mask_export")
    return mask


def swa_get_device_status(stream=None):
    """Synchronise and read/clear the device status word; returns the status code."""
    return int(load().swa_get_device_status(_stream(stream)))


def swa_debug_expire_wait(timeout_us, stream=None):
    _check(load().swa_debug_expire_wait(int(timeout_us), _stream(stream)), "swa_debug_expire_wait")


def swa_set_wait_limit_ns(ns):
    load().swa_set_wait_limit_ns(int(ns))
