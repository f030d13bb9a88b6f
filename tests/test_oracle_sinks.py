"""Pins of the oracle's attention sinks (the first s tokens kept beside the
causal window): special cases that reduce to independently pinned functions
(no sinks: the plain window; s >= T: full causal attention, checked against
torch's SDPA), the closed-form pair count, and the decode step over ring plus
sink caches agreeing with the prefill row by row across ring wrap-around."""
import numpy as np
import pytest
import torch

import oracle


def _rand(rng, *shape):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("T,W,s", [(16, 4, 0), (16, 4, 2), (30, 7, 3), (9, 20, 4), (40, 1, 5), (12, 3, 12)])
def test_pair_count_closed_form(T, W, s):
    # every row: its window, plus the sinks older than the window
    expect = sum(min(i + 1, W) + max(0, min(s, i - W + 1)) for i in range(T))
    assert oracle.count_pairs_sinks(T, W, s) == expect


def test_no_sinks_is_the_window():
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 2, 33, 4, 8), _rand(rng, 2, 33, 2, 8), _rand(rng, 2, 33, 2, 8)
    o, lse = oracle.swa_prefill_sinks(q, k, v, 5, 0)
    o_ref, lse_ref = oracle.swa_prefill(q, k, v, 5)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


@pytest.mark.parametrize("W", [1, 4])
def test_all_tokens_sinks_is_full_causal(W):
    rng = np.random.default_rng(2)
    T = 20
    q, k, v = _rand(rng, 1, T, 2, 8), _rand(rng, 1, T, 2, 8), _rand(rng, 1, T, 2, 8)
    o, _ = oracle.swa_prefill_sinks(q, k, v, W, T)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
    assert np.allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_mask_counts_sinks_once():
    # a sink inside the window is one key, not two
    T, W, s = 10, 4, 3
    for i in range(T):
        for j in range(T):
            in_w = oracle.in_window(i, j, T, W)
            sink = j < s and j <= i
            assert oracle.sink_allowed(i, j, T, W, s) == (in_w or sink)


@pytest.mark.parametrize("W,s", [(4, 2), (6, 1), (5, 5), (8, 3)])
def test_decode_steps_match_prefill_rows(W, s):
    # token by token: append to the ring, keep the first s tokens in the sink
    # caches, decode; every step equals the prefill row of that position
    rng = np.random.default_rng(W * 10 + s)
    T, Hq, Hkv, d = 23, 4, 2, 8
    q, k, v = _rand(rng, 1, T, Hq, d), _rand(rng, 1, T, Hkv, d), _rand(rng, 1, T, Hkv, d)
    o_ref, lse_ref = oracle.swa_prefill_sinks(q, k, v, W, s)
    kc = np.zeros((1, Hkv, W, d)); vc = np.zeros((1, Hkv, W, d))
    ks = np.zeros((1, Hkv, s, d)); vs = np.zeros((1, Hkv, s, d))
    for t in range(T):
        kc, vc, _ = oracle.ring_append(kc, vc, k[:, t:t + 1], v[:, t:t + 1], [t])
        if t < s:
            ks[0, :, t] = k[0, t]; vs[0, :, t] = v[0, t]
        o, lse = oracle.swa_decode_sinks(q[:, t], kc, vc, ks, vs, [t])
        assert np.allclose(o, o_ref[:, t], rtol=0, atol=1e-12)
        assert np.allclose(lse, lse_ref[:, :, t], rtol=0, atol=1e-12)


def test_decode_without_sinks_is_the_plain_decode():
    rng = np.random.default_rng(5)
    B, Hq, Hkv, d, W = 2, 4, 2, 8, 6
    q, kc, vc = _rand(rng, B, Hq, d), _rand(rng, B, Hkv, W, d), _rand(rng, B, Hkv, W, d)
    empty = np.zeros((B, Hkv, 0, d))
    o, lse = oracle.swa_decode_sinks(q, kc, vc, empty, empty, [3, 40])
    o_ref, lse_ref = oracle.swa_decode(q, kc, vc, [3, 40])
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)
