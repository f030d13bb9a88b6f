"""Pins of the oracle's chunked prefill (a chunk of new tokens continuing a
sequence whose earlier keys live in the W-slot ring), against functions that
are pinned independently: the plain causal prefill and the decode step."""
import numpy as np
import pytest

import oracle


def _rand(rng, *shape):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("n,W,Hq,Hkv", [(7, 3, 2, 1), (5, 9, 4, 2), (16, 16, 2, 2)])
def test_empty_ring_is_plain_prefill(n, W, Hq, Hkv):
    # nothing before position 0: the chunk is a whole sequence
    rng = np.random.default_rng(n + W)
    d = 8
    q, k, v = _rand(rng, 2, n, Hq, d), _rand(rng, 2, n, Hkv, d), _rand(rng, 2, n, Hkv, d)
    kc, vc = _rand(rng, 2, Hkv, W, d), _rand(rng, 2, Hkv, W, d)  # contents must not matter
    o, lse = oracle.swa_prefill_chunk(q, k, v, kc, vc, [0, 0])
    o_ref, lse_ref = oracle.swa_prefill(q, k, v, W)
    assert np.array_equal(o, o_ref)
    assert np.array_equal(lse, lse_ref)


@pytest.mark.parametrize("W,sizes", [(4, [3, 1, 5, 2, 9]), (6, [6, 6, 1, 13]), (5, [1] * 11),
                                     (8, [20, 3, 8])])
def test_chunks_over_the_ring_rebuild_the_whole_prefill(W, sizes):
    # run a sequence chunk by chunk, appending each chunk to the ring after its
    # prefill; the outputs must be the rows of the one-shot prefill
    rng = np.random.default_rng(W * 100 + len(sizes))
    T, Hq, Hkv, d = sum(sizes), 4, 2, 8
    q, k, v = _rand(rng, 1, T, Hq, d), _rand(rng, 1, T, Hkv, d), _rand(rng, 1, T, Hkv, d)
    o_ref, lse_ref = oracle.swa_prefill(q, k, v, W)
    kc = np.zeros((1, Hkv, W, d)); vc = np.zeros((1, Hkv, W, d))
    p = 0
    for n in sizes:
        sl = slice(p, p + n)
        o, lse = oracle.swa_prefill_chunk(q[:, sl], k[:, sl], v[:, sl], kc, vc, [p])
        assert np.array_equal(o, o_ref[:, sl])
        assert np.array_equal(lse, lse_ref[:, :, sl])
        kc, vc, _ = oracle.ring_append(kc, vc, k[:, sl], v[:, sl], [p])
        p += n


def test_one_token_chunk_is_a_decode_step():
    rng = np.random.default_rng(7)
    B, Hq, Hkv, d, W = 3, 4, 2, 8, 6
    pos = [0, 4, 23]
    kc, vc = _rand(rng, B, Hkv, W, d), _rand(rng, B, Hkv, W, d)
    q, k, v = _rand(rng, B, 1, Hq, d), _rand(rng, B, 1, Hkv, d), _rand(rng, B, 1, Hkv, d)
    o, lse = oracle.swa_prefill_chunk(q, k, v, kc, vc, pos)
    kc2, vc2, _ = oracle.ring_append(kc, vc, k, v, pos)
    o_dec, lse_dec = oracle.swa_decode(q[:, 0], kc2, vc2, pos)
    # the decode lists its keys in slot order, the chunk in position order
    assert np.allclose(o[:, 0], o_dec, rtol=0, atol=1e-12)
    assert np.allclose(lse[:, :, 0], lse_dec, rtol=0, atol=1e-12)


def test_partially_filled_ring_uses_only_existing_positions():
    # pos < W: slots pos..W-1 hold nothing yet and must be ignored
    rng = np.random.default_rng(11)
    W, p, n, d = 10, 3, 4, 8
    q, k, v = _rand(rng, 1, p + n, 2, d), _rand(rng, 1, p + n, 1, d), _rand(rng, 1, p + n, 1, d)
    kc = np.full((1, 1, W, d), 1e6); vc = np.full((1, 1, W, d), -1e6)
    kc[0, 0, :p] = k[0, :p, 0]; vc[0, 0, :p] = v[0, :p, 0]
    o, _ = oracle.swa_prefill_chunk(q[:, p:], k[:, p:], v[:, p:], kc, vc, [p])
    o_ref, _ = oracle.swa_prefill(q, k, v, W)
    assert np.array_equal(o, o_ref[:, p:])


def test_negative_position_is_rejected():
    z = np.zeros((1, 1, 1, 8))
    with pytest.raises(ValueError):
        oracle.swa_prefill_chunk(z, z, z, np.zeros((1, 1, 4, 8)), np.zeros((1, 1, 4, 8)), [-1])
