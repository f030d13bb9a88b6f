"""fp64 CPU oracle for sliding-window attention.

TEST INFRASTRUCTURE: only tests/, the smoke check and the benchmark's
CPU-baseline leg use this package.  It shares no code with the CUDA path
(decode_swa_prefill_b200); neither imports the other.

The arithmetic lives in oracle.c (plain C, fp64, two-pass softmax); this module
only marshals numpy/torch arrays into fp64 C buffers and back.  Each wrapper
names the page passage its C function follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

CAUSAL = 0
SYMMETRIC = 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        c_long, c_int, c_double = ctypes.c_long, ctypes.c_int, ctypes.c_double
        p = ctypes.c_void_p
        lib.oracle_in_window.argtypes = [c_long, c_long, c_long, c_long, c_int]
        lib.oracle_in_window.restype = c_int
        lib.oracle_allowed.argtypes = [c_long, c_long, c_long, c_long, c_int, p, c_long]
        lib.oracle_allowed.restype = c_int
        lib.oracle_mask.argtypes = [p, c_long, c_long, c_int, p, c_long]
        lib.oracle_mask.restype = None
        lib.oracle_count_pairs.argtypes = [c_long, c_long, c_int, p, c_long]
        lib.oracle_count_pairs.restype = ctypes.c_longlong
        lib.oracle_reach.argtypes = [p, c_long, c_long, c_int]
        lib.oracle_reach.restype = c_int
        lib.oracle_slot.argtypes = [c_long, c_long]
        lib.oracle_slot.restype = c_long
        lib.oracle_ring_append.argtypes = [p, p, p, p, p, p, c_long, c_long, c_long, c_long, c_long]
        lib.oracle_ring_append.restype = None
        lib.oracle_swa_prefill.argtypes = [p, p, p, p, p, c_long, c_long, c_long, c_long, c_long,
                                           c_long, c_double, p, c_long, c_int]
        lib.oracle_swa_prefill.restype = c_int
        lib.oracle_swa_prefill_global.argtypes = [p, p, p, p, p, p, c_long, c_long, c_long, c_long,
                                                  c_long, c_long, c_long, c_double, p, c_long, c_int]
        lib.oracle_swa_prefill_global.restype = c_int
        lib.oracle_swa_decode.argtypes = [p, p, p, p, p, p, c_long, c_long, c_long, c_long, c_long,
                                          c_double]
        lib.oracle_swa_decode.restype = c_int
        lib.oracle_swa_prefill_chunk.argtypes = [p, p, p, p, p, p, p, p, c_long, c_long, c_long, c_long,
                                                 c_long, c_long, c_double]
        lib.oracle_swa_prefill_chunk.restype = c_int
        lib.oracle_sink_allowed.argtypes = [c_long, c_long, c_long, c_long, c_long]
        lib.oracle_sink_allowed.restype = c_int
        lib.oracle_count_pairs_sinks.argtypes = [c_long, c_long, c_long]
        lib.oracle_count_pairs_sinks.restype = ctypes.c_longlong
        lib.oracle_swa_prefill_sinks.argtypes = [p, p, p, p, p, c_long, c_long, c_long, c_long, c_long,
                                                 c_long, c_long, c_double, p, c_long, c_int]
        lib.oracle_swa_prefill_sinks.restype = c_int
        lib.oracle_swa_decode_sinks.argtypes = [p, p, p, p, p, p, p, p, c_long, c_long, c_long, c_long,
                                                c_long, c_long, c_double]
        lib.oracle_swa_decode_sinks.restype = c_int
        lib.oracle_dilated_allowed.argtypes = [c_long, c_long, c_long, c_long, c_long, c_int]
        lib.oracle_dilated_allowed.restype = c_int
        lib.oracle_count_pairs_dilated.argtypes = [c_long, c_long, c_long, c_int]
        lib.oracle_count_pairs_dilated.restype = ctypes.c_longlong
        lib.oracle_swa_prefill_dilated.argtypes = [p, p, p, p, p, c_long, c_long, c_long, c_long, c_long,
                                                   c_long, c_long, c_int, c_double, p, c_long, c_int]
        lib.oracle_swa_prefill_dilated.restype = c_int
        lib.oracle_varlen_allowed.argtypes = [c_long, c_long, p, c_long, p]
        lib.oracle_varlen_allowed.restype = c_int
        lib.oracle_count_pairs_varlen.argtypes = [p, c_long, p]
        lib.oracle_count_pairs_varlen.restype = ctypes.c_longlong
        lib.oracle_swa_prefill_varlen.argtypes = [p, p, p, p, p, p, c_long, p, c_long, c_long, c_long, c_long,
                                                  c_double, p, c_long, c_int]
        lib.oracle_swa_prefill_varlen.restype = c_int
        lib.oracle_paged_append.argtypes = [p, p, p, p, p, p, p, c_long, c_long, c_long, c_long, c_long, c_long,
                                            c_long]
        lib.oracle_paged_append.restype = c_int
        lib.oracle_swa_decode_paged.argtypes = [p, p, p, p, p, p, p, c_long, c_long, c_long, c_long, c_long,
                                                c_long, c_long, c_double]
        lib.oracle_swa_decode_paged.restype = c_int
        lib.oracle_swa_backward.argtypes = [p, p, p, p, p, p, p, c_long, c_long, c_long, c_long, c_long, c_long,
                                            c_int, c_double, c_int]
        lib.oracle_swa_backward.restype = c_int
        _lib = lib
    return _lib


def _f64(x):
    """fp64, C-contiguous numpy copy of a numpy array or (CPU) torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _i32(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads():
    return max(1, len(os.sched_getaffinity(0)))


# ------------------------------------------------------------------ masks --

def in_window(i, j, T, W, mode=CAUSAL):
    """Window membership: causal i-W+1<=j<=i, symmetric |i-j|<=W//2
    (robocikowo.com "Sliding Window Attention", opening definition)."""
    return bool(_load().oracle_in_window(i, j, T, W, mode))


def mask(T, W, mode=CAUSAL, global_idx=None):
    """Explicit [T,T] uint8 visibility mask, globals included (Longformer
    global attention: aivaro.ru answer 629, section 4.3)."""
    g = 0 if global_idx is None else len(global_idx)
    gi = None if global_idx is None else _i32(global_idx)
    out = np.zeros((T, T), dtype=np.uint8)
    _load().oracle_mask(_ptr(out), T, W, mode, _ptr(gi), g)
    return out


def count_pairs(T, W, mode=CAUSAL, global_idx=None):
    """Scores computed per layer (Ultralytics glossary, depth section)."""
    g = 0 if global_idx is None else len(global_idx)
    gi = None if global_idx is None else _i32(global_idx)
    return int(_load().oracle_count_pairs(T, W, mode, _ptr(gi), g))


def reach(T, W, L):
    """Last-token reach after 1..L stacked causal layers, by boolean mask
    products (Ultralytics glossary, depth section)."""
    out = np.zeros(L, dtype=np.int32)
    rc = _load().oracle_reach(_ptr(out), T, W, L)
    assert rc == 0
    return [int(x) for x in out]


def slot(pos, W):
    """Ring slot of a position (Ultralytics glossary, ring-buffer paragraph)."""
    return int(_load().oracle_slot(pos, W))


def ring_append(k_cache, v_cache, k_new, v_new, pos):
    """Sequential FIFO append into [B,Hkv,W,d] caches; returns (kc, vc, slots)
    as new fp64 arrays (robocikowo.com rolling-buffer entry)."""
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    kn, vn = _f64(k_new), _f64(v_new)
    B, Hkv, W, d = kc.shape
    n = kn.shape[1]
    slots = np.zeros((B, n), dtype=np.int32)
    _load().oracle_ring_append(_ptr(kc), _ptr(vc), _ptr(kn), _ptr(vn), _ptr(_i32(pos)), _ptr(slots),
                               B, n, Hkv, d, W)
    return kc, vc, slots


def paged_append(k_pages, v_pages, k_new, v_new, pos, page_table):
    """FIFO append into a paged ring: pools [num_pages,Hkv,P,d], page_table
    [B,W/P] (ring slot s of sequence b is row s % P of page page_table[b,
    s // P]); W = P * page_table.shape[1].  Returns (kp, vp, slots) as new
    fp64 arrays (Ultralytics ring-buffer paragraph; robocikowo.com
    rolling-buffer entry)."""
    kp, vp = _f64(k_pages).copy(), _f64(v_pages).copy()
    kn, vn = _f64(k_new), _f64(v_new)
    tbl = _i32(page_table)
    num_pages, Hkv, P, d = kp.shape
    B, n = kn.shape[0], kn.shape[1]
    W = P * tbl.shape[1]
    slots = np.zeros((B, n), dtype=np.int32)
    rc = _load().oracle_paged_append(_ptr(kp), _ptr(vp), _ptr(kn), _ptr(vn), _ptr(_i32(pos)), _ptr(tbl),
                                     _ptr(slots), B, n, Hkv, d, W, P, num_pages)
    if rc != 0:
        raise ValueError("page table names a page outside the pool")
    return kp, vp, slots


def swa_decode_paged(q, k_pages, v_pages, page_table, pos, scale=None):
    """One decode step over a paged ring (layout as paged_append); the
    current token at pos[b] already appended.  Returns o [B,Hq,d], lse
    [B,Hq]."""
    q, kp, vp = _f64(q), _f64(k_pages), _f64(v_pages)
    tbl = _i32(page_table)
    B, Hq, d = q.shape
    num_pages, Hkv, P = kp.shape[0], kp.shape[1], kp.shape[2]
    W = P * tbl.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, d)); lse = np.zeros((B, Hq))
    rc = _load().oracle_swa_decode_paged(_ptr(q), _ptr(kp), _ptr(vp), _ptr(tbl), _ptr(_i32(pos)), _ptr(o),
                                         _ptr(lse), B, Hq, Hkv, d, W, P, num_pages, float(scale))
    if rc != 0:
        raise ValueError("negative position or a page outside the pool")
    return o, lse


# ---------------------------------------------------------------- prefill --

def _rows_arg(rows, B, Hq, T):
    if rows is None:
        return np.arange(B * Hq * T, dtype=np.int64)
    return np.ascontiguousarray(rows, dtype=np.int64)


def row_ids(b, h, i, Hq, T):
    """Flattened row id used by the row-subset entry points."""
    return (np.asarray(b, dtype=np.int64) * Hq + np.asarray(h, dtype=np.int64)) * T + np.asarray(i, dtype=np.int64)


def _unflatten(o_rows, lse_rows, rows, full, B, T, Hq, d):
    if not full:
        return o_rows, lse_rows
    # rows enumerate (b, h, i) in order; reshape to [B,T,Hq,d] and [B,Hq,T]
    o = o_rows.reshape(B, Hq, T, d).transpose(0, 2, 1, 3).copy()
    lse = lse_rows.reshape(B, Hq, T).copy()
    return o, lse


def swa_prefill(q, k, v, W, scale=None, rows=None, nthreads=None):
    """Causal SWA (robocikowo.com opening definition; aivaro.ru section 3).

    q [B,T,Hq,d], k/v [B,T,Hkv,d].  rows=None returns the full o [B,T,Hq,d]
    and lse [B,Hq,T]; otherwise rows are flattened (b*Hq+h)*T+i ids and the
    result is o [nrows,d], lse [nrows]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = _rows_arg(rows, B, Hq, T)
    o = np.zeros((len(r), d)); lse = np.zeros(len(r))
    _load().oracle_swa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, Hq, Hkv, d, W,
                               float(scale), _ptr(r), len(r), nthreads or default_threads())
    return _unflatten(o, lse, r, rows is None, B, T, Hq, d)


def swa_prefill_global(q, k, v, global_idx, W, scale=None, rows=None, nthreads=None):
    """Symmetric window |i-j|<=W//2 plus global tokens (aivaro.ru sections
    4.1 and 4.3).  global_idx [B,g] (g may be 0)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    gi = _i32(global_idx).reshape(B, -1) if global_idx is not None else np.zeros((B, 0), np.int32)
    g = gi.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = _rows_arg(rows, B, Hq, T)
    o = np.zeros((len(r), d)); lse = np.zeros(len(r))
    _load().oracle_swa_prefill_global(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(gi), g,
                                      B, T, Hq, Hkv, d, W, float(scale), _ptr(r), len(r),
                                      nthreads or default_threads())
    return _unflatten(o, lse, r, rows is None, B, T, Hq, d)


def swa_decode(q, k_cache, v_cache, pos, scale=None):
    """One decode step over W-slot rings (Ultralytics ring-buffer paragraph).
    q [B,Hq,d], caches [B,Hkv,W,d], pos [B] = position of the current token,
    already appended.  Returns o [B,Hq,d], lse [B,Hq]."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, d = q.shape
    Hkv, W = kc.shape[1], kc.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, d)); lse = np.zeros((B, Hq))
    _load().oracle_swa_decode(_ptr(q), _ptr(kc), _ptr(vc), _ptr(_i32(pos)), _ptr(o), _ptr(lse),
                              B, Hq, Hkv, d, W, float(scale))
    return o, lse


def swa_prefill_chunk(q, k, v, k_cache, v_cache, pos, scale=None):
    """Causal prefill of a chunk of n tokens at positions pos[b].. that reads
    the keys before pos[b] from the W-slot ring (Ultralytics ring-buffer
    paragraph; robocikowo.com opening definition).  q [B,n,Hq,d], k/v
    [B,n,Hkv,d], caches [B,Hkv,W,d] not yet holding the chunk, pos [B].
    Returns o [B,n,Hq,d], lse [B,Hq,n]."""
    q, k, v, kc, vc = _f64(q), _f64(k), _f64(v), _f64(k_cache), _f64(v_cache)
    B, n, Hq, d = q.shape
    Hkv, W = kc.shape[1], kc.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, n, Hq, d)); lse = np.zeros((B, Hq, n))
    rc = _load().oracle_swa_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(kc), _ptr(vc), _ptr(_i32(pos)),
                                          _ptr(o), _ptr(lse), B, n, Hq, Hkv, d, W, float(scale))
    if rc != 0:
        raise ValueError("negative position")
    return o, lse


# ------------------------------------------------------------------ sinks --

def sink_allowed(i, j, T, W, s):
    """Causal window plus the first s tokens as attention sinks (Ultralytics
    glossary, related-terms entry on attention sinks)."""
    return bool(_load().oracle_sink_allowed(i, j, T, W, s))


def count_pairs_sinks(T, W, s):
    return int(_load().oracle_count_pairs_sinks(T, W, s))


def swa_prefill_sinks(q, k, v, W, sinks, scale=None, rows=None, nthreads=None):
    """Causal window W plus the first `sinks` tokens of each sequence; shapes
    and row selection as swa_prefill."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = _rows_arg(rows, B, Hq, T)
    o = np.zeros((len(r), d)); lse = np.zeros(len(r))
    _load().oracle_swa_prefill_sinks(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, Hq, Hkv, d, W,
                                     int(sinks), float(scale), _ptr(r), len(r), nthreads or default_threads())
    return _unflatten(o, lse, r, rows is None, B, T, Hq, d)


def swa_decode_sinks(q, k_cache, v_cache, k_sink, v_sink, pos, scale=None):
    """One decode step over the ring plus sink caches [B,Hkv,s,d] holding
    positions 0..s-1 (the current token already appended to the ring)."""
    q, kc, vc, ks, vs = _f64(q), _f64(k_cache), _f64(v_cache), _f64(k_sink), _f64(v_sink)
    B, Hq, d = q.shape
    Hkv, W = kc.shape[1], kc.shape[2]
    s = ks.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, d)); lse = np.zeros((B, Hq))
    rc = _load().oracle_swa_decode_sinks(_ptr(q), _ptr(kc), _ptr(vc), _ptr(ks), _ptr(vs), _ptr(_i32(pos)),
                                         _ptr(o), _ptr(lse), B, Hq, Hkv, d, W, s, float(scale))
    if rc != 0:
        raise ValueError("negative position")
    return o, lse


# ---------------------------------------------------------------- dilated --

def dilated_allowed(i, j, T, W, dil, mode=CAUSAL):
    """Dilated window (aivaro.ru section 4.2): causal keys i - dil*m,
    m = 0..W-1; symmetric keys i + dil*m, |m| <= W//2."""
    return bool(_load().oracle_dilated_allowed(i, j, T, W, dil, mode))


def count_pairs_dilated(T, W, dil, mode=CAUSAL):
    return int(_load().oracle_count_pairs_dilated(T, W, dil, mode))


def swa_prefill_dilated(q, k, v, W, dil, mode=CAUSAL, scale=None, rows=None, nthreads=None):
    """Dilated sliding-window prefill (aivaro.ru section 4.2); shapes and row
    selection as swa_prefill."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = _rows_arg(rows, B, Hq, T)
    o = np.zeros((len(r), d)); lse = np.zeros(len(r))
    rc = _load().oracle_swa_prefill_dilated(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, Hq, Hkv, d, W,
                                            int(dil), int(mode), float(scale), _ptr(r), len(r),
                                            nthreads or default_threads())
    if rc != 0:
        raise ValueError("bad dilation or mode")
    return _unflatten(o, lse, r, rows is None, B, T, Hq, d)


# ----------------------------------------------------------------- varlen --

def _windows(W, nseq):
    """One window per sequence: W is an int (every sequence) or a sequence of
    nseq ints."""
    if np.ndim(W) == 0:
        return np.full(nseq, int(W), dtype=np.int32)
    w = _i32(W).reshape(-1)
    assert len(w) == nseq, "one window per sequence"
    return w


def varlen_allowed(r, j, cu_seqlens, W):
    """Packed rows: row r sees row j of its own sequence with r-W_s+1 <= j <= r
    (robocikowo.com opening definition, per sequence)."""
    cu = _i32(cu_seqlens)
    return bool(_load().oracle_varlen_allowed(r, j, _ptr(cu), len(cu) - 1, _ptr(_windows(W, len(cu) - 1))))


def count_pairs_varlen(cu_seqlens, W):
    cu = _i32(cu_seqlens)
    return int(_load().oracle_count_pairs_varlen(_ptr(cu), len(cu) - 1, _ptr(_windows(W, len(cu) - 1))))


def swa_prefill_varlen(q, k, v, cu_seqlens, W, scale=None, rows=None, nthreads=None):
    """Causal window over packed sequences: q [total,Hq,d], k/v
    [total,Hkv,d]; sequence s holds rows cu_seqlens[s] .. cu_seqlens[s+1]-1
    and attends within itself only, with its own window W[s] (W an int: the
    same window for all).  Every sequence is its own causal prefill
    (robocikowo.com opening definition); the windows may differ as between
    the local layers of different models (Ultralytics glossary, section on
    alternating local and global layers).  rows=None returns o [total,Hq,d]
    and lse [Hq,total]; otherwise rows are flattened h*total + r ids and the
    result is o [nrows,d], lse [nrows]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = _i32(cu_seqlens)
    nseq = len(cu) - 1
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    w = _windows(W, nseq)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = _rows_arg(rows, 1, Hq, total)
    o = np.zeros((len(r), d)); lse = np.zeros(len(r))
    rc = _load().oracle_swa_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu), nseq, _ptr(w),
                                           total, Hq, Hkv, d, float(scale), _ptr(r), len(r),
                                           nthreads or default_threads())
    if rc != 0:
        raise ValueError("inconsistent offsets or a window below 1")
    if rows is not None:
        return o, lse
    o, lse = _unflatten(o, lse, r, True, 1, total, Hq, d)
    return o[0], lse[0]


def swa_backward(q, k, v, dout, W, symmetric=False, scale=None, nthreads=None):
    """Gradients (dq [B,T,Hq,d], dk, dv [B,T,Hkv,d]) of the causal (or, with
    symmetric=True, the |i-j| <= W//2) window prefill for the upstream
    gradient dout [B,T,Hq,d].  The pages define only the forward pass; this is
    its definition differentiated by the chain rule (see oracle.c)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    rc = _load().oracle_swa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dq), _ptr(dk), _ptr(dv),
                                     B, T, Hq, Hkv, d, W, 1 if symmetric else 0, float(scale),
                                     nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_swa_backward: bad arguments")
    return dq, dk, dv
