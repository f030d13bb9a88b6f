"""Pins of the oracle's attention values.

Each test reduces a case to something fixed independently of oracle.c:
torch's fp64 scaled_dot_product_attention (full causal, full bidirectional,
GQA grouping, explicit boolean masks), scipy's softmax on an explicit
[T,T] -inf mask (the brute-force recipe of the aivaro.ru pet-project section),
exact special cases (W=1 returns V), and cross-path invariants (one decode step
over the ring equals the matching prefill row).  CPU only.
"""
import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle

ATOL = 1e-12


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def sdpa(q, k, v, mask=None, causal=False, scale=None):
    """torch fp64 SDPA on [B,T,H,d] arrays; K/V heads grouped like GQA."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    am = None if mask is None else torch.from_numpy(mask.astype(bool))
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, is_causal=causal, scale=scale,
                                       enable_gqa=qt.shape[1] != kt.shape[1])
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("T,W", [(1, 1), (7, 7), (16, 16), (16, 40), (33, 33)])
def test_window_at_least_T_is_full_causal(T, W):
    q, k, v = rnd((2, T, 3, 16), 1), rnd((2, T, 3, 16), 2), rnd((2, T, 3, 16), 3)
    o, _ = oracle.swa_prefill(q, k, v, W)
    np.testing.assert_allclose(o, sdpa(q, k, v, causal=True), atol=ATOL, rtol=0)


@pytest.mark.parametrize("T", [1, 5, 16])
def test_window_one_returns_v(T):
    q, k, v = rnd((1, T, 4, 8), 4), rnd((1, T, 2, 8), 5), rnd((1, T, 2, 8), 6)
    o, lse = oracle.swa_prefill(q, k, v, 1)
    # query head h reads kv head h*Hkv//Hq = h//2
    for h in range(4):
        assert np.array_equal(o[:, :, h], v[:, :, h // 2])


@pytest.mark.parametrize("T,W,Hq,Hkv", [(16, 4, 1, 1), (40, 7, 8, 2), (37, 5, 6, 3), (64, 16, 4, 4)])
def test_causal_window_matches_sdpa_masked(T, W, Hq, Hkv):
    d = 12
    q, k, v = rnd((2, T, Hq, d), 7), rnd((2, T, Hkv, d), 8), rnd((2, T, Hkv, d), 9)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    band = (j <= i) & (j > i - W)
    o, lse = oracle.swa_prefill(q, k, v, W, scale=0.3)
    np.testing.assert_allclose(o, sdpa(q, k, v, mask=band, scale=0.3), atol=ATOL, rtol=0)


def test_causal_window_row_by_row_slices():
    # each row separately: plain (unmasked) SDPA over the contiguous key slice
    T, W, d = 30, 6, 8
    q, k, v = rnd((1, T, 2, d), 10), rnd((1, T, 1, d), 11), rnd((1, T, 1, d), 12)
    o, lse = oracle.swa_prefill(q, k, v, W)
    for i in range(T):
        lo = max(0, i - W + 1)
        ref = sdpa(q[:, i:i + 1], k[:, lo:i + 1], v[:, lo:i + 1])
        np.testing.assert_allclose(o[:, i:i + 1], ref, atol=ATOL, rtol=0)
        s = (q[0, i, 0] @ k[0, lo:i + 1, 0].T) / np.sqrt(d)
        assert abs(lse[0, 0, i] - scipy.special.logsumexp(s)) < ATOL


@pytest.mark.parametrize("T", [1, 2, 5, 9, 16, 24])
@pytest.mark.parametrize("mode", [oracle.CAUSAL, oracle.SYMMETRIC])
@pytest.mark.parametrize("g", [0, 1, 3])
def test_bruteforce_explicit_minus_inf(T, mode, g):
    """Build the [T,T] mask, put -inf at forbidden scores, softmax, weighted
    sum (aivaro.ru answer 629, pet-project steps)."""
    if mode == oracle.CAUSAL and g > 0:
        pytest.skip("globals only in the symmetric mode")
    d, Hq, Hkv = 8, 2, 1
    q, k, v = rnd((1, T, Hq, d), 13 + T), rnd((1, T, Hkv, d), 14 + T), rnd((1, T, Hkv, d), 15 + T)
    gi = np.sort(np.random.default_rng(T).permutation(T)[:min(g, T)]).astype(np.int32)
    for W in sorted({1, 2, 3, 4, max(1, T - 1), T, T + 5}):
        m = oracle.mask(T, W, mode, gi if g else None).astype(bool)
        s = np.einsum("bihd,bjd->bhij", q, k[:, :, 0]) / np.sqrt(d)
        s = np.where(m[None, None], s, -np.inf)
        p = scipy.special.softmax(s, axis=-1)
        ref = np.einsum("bhij,bjd->bihd", p, v[:, :, 0])
        if mode == oracle.CAUSAL:
            o, _ = oracle.swa_prefill(q, k, v, W)
        else:
            o, _ = oracle.swa_prefill_global(q, k, v, gi[None] if g else None, W)
        np.testing.assert_allclose(o, ref, atol=ATOL, rtol=0)


@pytest.mark.parametrize("T,W", [(10, 18), (10, 30), (17, 40)])
def test_symmetric_wide_window_is_full_bidirectional(T, W):
    q, k, v = rnd((1, T, 2, 8), 20), rnd((1, T, 2, 8), 21), rnd((1, T, 2, 8), 22)
    o, _ = oracle.swa_prefill_global(q, k, v, None, W)
    np.testing.assert_allclose(o, sdpa(q, k, v), atol=ATOL, rtol=0)


def test_all_tokens_global_is_full_bidirectional():
    T = 12
    q, k, v = rnd((2, T, 2, 8), 23), rnd((2, T, 1, 8), 24), rnd((2, T, 1, 8), 25)
    gi = np.tile(np.arange(T, dtype=np.int32), (2, 1))
    o, _ = oracle.swa_prefill_global(q, k, v, gi, 2)
    np.testing.assert_allclose(o, sdpa(q, k, v), atol=ATOL, rtol=0)


def test_global_rows_and_gathered_keys():
    """Global rows equal full-sequence attention; other rows equal plain
    attention over the gathered key set band(i) U G (aivaro.ru s.4.3)."""
    T, W, d = 40, 6, 8
    q, k, v = rnd((1, T, 2, d), 26), rnd((1, T, 2, d), 27), rnd((1, T, 2, d), 28)
    gi = np.array([[3, 20, 39]], dtype=np.int32)
    o, lse = oracle.swa_prefill_global(q, k, v, gi, W)
    full = sdpa(q, k, v)
    for i in range(T):
        if i in gi[0]:
            np.testing.assert_allclose(o[:, i], full[:, i], atol=ATOL, rtol=0)
            continue
        keys = sorted(set(range(max(0, i - W // 2), min(T, i + W // 2 + 1))) | set(gi[0].tolist()))
        ref = sdpa(q[:, i:i + 1], k[:, keys], v[:, keys])
        np.testing.assert_allclose(o[:, i:i + 1], ref, atol=ATOL, rtol=0)


def test_no_globals_equals_symmetric_window():
    T, W = 33, 8
    q, k, v = rnd((1, T, 2, 8), 29), rnd((1, T, 2, 8), 30), rnd((1, T, 2, 8), 31)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    band = np.abs(i - j) <= W // 2
    o, _ = oracle.swa_prefill_global(q, k, v, np.zeros((1, 0), np.int32), W)
    np.testing.assert_allclose(o, sdpa(q, k, v, mask=band), atol=ATOL, rtol=0)


def test_row_subset_matches_full():
    T, W = 50, 9
    q, k, v = rnd((2, T, 4, 8), 32), rnd((2, T, 2, 8), 33), rnd((2, T, 2, 8), 34)
    o, lse = oracle.swa_prefill(q, k, v, W)
    b = np.array([0, 1, 1, 0]); h = np.array([3, 0, 2, 1]); i = np.array([0, 49, 17, 8])
    o2, l2 = oracle.swa_prefill(q, k, v, W, rows=oracle.row_ids(b, h, i, 4, T))
    for r in range(4):
        assert np.array_equal(o2[r], o[b[r], i[r], h[r]])
        assert l2[r] == lse[b[r], h[r], i[r]]


@pytest.mark.parametrize("W,P", [(8, 3), (8, 8), (8, 21), (5, 40)])
def test_decode_over_ring_equals_last_window(W, P):
    """Fill a ring by appending a whole sequence, decode the last token: equal
    to plain attention over the last min(P, W) tokens, and to prefill row P-1."""
    B, Hq, Hkv, d = 2, 4, 2, 8
    k, v = rnd((B, P, Hkv, d), 35), rnd((B, P, Hkv, d), 36)
    q = rnd((B, P, Hq, d), 37)
    kc = np.zeros((B, Hkv, W, d)); vc = np.zeros((B, Hkv, W, d))
    kc, vc, _ = oracle.ring_append(kc, vc, k, v, np.zeros(B, np.int32))
    pos = np.full(B, P - 1, np.int32)
    o, lse = oracle.swa_decode(q[:, P - 1], kc, vc, pos)
    lo = max(0, P - W)
    ref = sdpa(q[:, P - 1:P], k[:, lo:], v[:, lo:])[:, 0]
    np.testing.assert_allclose(o, ref, atol=ATOL, rtol=0)
    op, lp = oracle.swa_prefill(q, k, v, W)
    np.testing.assert_allclose(o, op[:, P - 1], atol=ATOL, rtol=0)
    np.testing.assert_allclose(lse, lp[:, :, P - 1], atol=ATOL, rtol=0)


def test_decode_step_by_step_matches_prefill_rows():
    B, Hq, Hkv, d, W, P = 1, 2, 1, 8, 6, 20
    k, v, q = rnd((B, P, Hkv, d), 38), rnd((B, P, Hkv, d), 39), rnd((B, P, Hq, d), 40)
    op, _ = oracle.swa_prefill(q, k, v, W)
    kc = np.zeros((B, Hkv, W, d)); vc = np.zeros((B, Hkv, W, d))
    for t in range(P):
        kc, vc, _ = oracle.ring_append(kc, vc, k[:, t:t + 1], v[:, t:t + 1], np.array([t], np.int32))
        o, _ = oracle.swa_decode(q[:, t], kc, vc, np.array([t], np.int32))
        np.testing.assert_allclose(o, op[:, t], atol=ATOL, rtol=0)


def test_lse_matches_logsumexp():
    T, W, d = 20, 5, 8
    q, k, v = rnd((1, T, 1, d), 41), rnd((1, T, 1, d), 42), rnd((1, T, 1, d), 43)
    m = oracle.mask(T, W).astype(bool)
    s = (q[0, :, 0] @ k[0, :, 0].T) / np.sqrt(d)
    ref = scipy.special.logsumexp(np.where(m, s, -np.inf), axis=-1)
    _, lse = oracle.swa_prefill(q, k, v, W)
    np.testing.assert_allclose(lse[0, 0], ref, atol=ATOL, rtol=0)
