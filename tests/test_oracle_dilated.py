"""Pins of the oracle's dilated window (aivaro.ru section 4.2): dilation 1 is
the plain window, the pair counts follow closed forms, and a dilated prefill
equals the plain window applied to each of the dil strided sub-sequences
(rows i = r, r+dil, r+2dil, ...), the identity the GPU path is built on."""
import numpy as np
import pytest

import oracle


def _rand(rng, *shape):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("T,W,dil", [(16, 4, 2), (30, 5, 3), (9, 20, 4), (40, 1, 7), (12, 3, 12)])
def test_causal_pair_count_closed_form(T, W, dil):
    expect = sum(min(W, i // dil + 1) for i in range(T))
    assert oracle.count_pairs_dilated(T, W, dil, oracle.CAUSAL) == expect


@pytest.mark.parametrize("T,W,dil", [(16, 4, 2), (30, 6, 3), (9, 20, 4), (40, 2, 7)])
def test_symmetric_pair_count_closed_form(T, W, dil):
    h = W // 2
    expect = sum(min(h, i // dil) + min(h, (T - 1 - i) // dil) + 1 for i in range(T))
    assert oracle.count_pairs_dilated(T, W, dil, oracle.SYMMETRIC) == expect


def test_dilation_one_is_the_plain_window():
    rng = np.random.default_rng(3)
    q, k, v = _rand(rng, 2, 37, 4, 8), _rand(rng, 2, 37, 2, 8), _rand(rng, 2, 37, 2, 8)
    o, lse = oracle.swa_prefill_dilated(q, k, v, 6, 1, oracle.CAUSAL)
    o_ref, lse_ref = oracle.swa_prefill(q, k, v, 6)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)
    o, lse = oracle.swa_prefill_dilated(q, k, v, 6, 1, oracle.SYMMETRIC)
    o_ref, lse_ref = oracle.swa_prefill_global(q, k, v, None, 6)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


@pytest.mark.parametrize("mode", [oracle.CAUSAL, oracle.SYMMETRIC])
@pytest.mark.parametrize("T,W,dil", [(37, 4, 3), (40, 5, 4), (20, 8, 2), (11, 3, 11)])
def test_dilated_equals_plain_window_on_strided_subsequences(mode, T, W, dil):
    rng = np.random.default_rng(T * dil + W)
    q, k, v = _rand(rng, 2, T, 4, 8), _rand(rng, 2, T, 2, 8), _rand(rng, 2, T, 2, 8)
    o, lse = oracle.swa_prefill_dilated(q, k, v, W, dil, mode)
    for r in range(dil):
        sub = slice(r, None, dil)
        qs, ks, vs = (np.ascontiguousarray(x[:, sub]) for x in (q, k, v))
        if mode == oracle.CAUSAL:
            o_r, lse_r = oracle.swa_prefill(qs, ks, vs, W)
        else:
            o_r, lse_r = oracle.swa_prefill_global(qs, ks, vs, None, W)
        assert np.array_equal(o[:, sub], o_r)
        assert np.array_equal(lse[:, :, sub], lse_r)


def test_bad_arguments_rejected():
    z = np.zeros((1, 4, 1, 8))
    with pytest.raises(ValueError):
        oracle.swa_prefill_dilated(z, z, z, 4, 0)
