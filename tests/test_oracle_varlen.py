"""Pins of the oracle's packed variable-length prefill: one sequence is the
plain prefill, equal lengths are the batched prefill, and no row ever sees a
key of another sequence (checked by changing the other sequences)."""
import numpy as np

import oracle


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_one_sequence_is_the_plain_prefill():
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 40, 4, 8), _rand(rng, 40, 2, 8), _rand(rng, 40, 2, 8)
    o, lse = oracle.swa_prefill_varlen(q, k, v, [0, 40], 7)
    o_ref, lse_ref = oracle.swa_prefill(q[None], k[None], v[None], 7)
    assert np.array_equal(o, o_ref[0]) and np.array_equal(lse, lse_ref[0])


def test_equal_lengths_are_the_batched_prefill():
    rng = np.random.default_rng(2)
    B, T = 3, 17
    q, k, v = _rand(rng, B, T, 4, 8), _rand(rng, B, T, 2, 8), _rand(rng, B, T, 2, 8)
    o, lse = oracle.swa_prefill_varlen(q.reshape(B * T, 4, 8), k.reshape(B * T, 2, 8), v.reshape(B * T, 2, 8),
                                       [0, T, 2 * T, 3 * T], 5)
    o_ref, lse_ref = oracle.swa_prefill(q, k, v, 5)
    assert np.array_equal(o, o_ref.reshape(B * T, 4, 8))
    assert np.array_equal(lse.reshape(4, B, T).transpose(1, 0, 2), lse_ref)


def test_sequences_do_not_see_each_other():
    rng = np.random.default_rng(3)
    cu = [0, 5, 5, 31, 40]          # includes an empty sequence
    q, k, v = _rand(rng, 40, 2, 8), _rand(rng, 40, 1, 8), _rand(rng, 40, 1, 8)
    o, _ = oracle.swa_prefill_varlen(q, k, v, cu, 9)
    k2, v2 = k.copy(), v.copy()
    k2[:5] += 3.0; v2[:5] -= 2.0     # change sequence 0 only
    k2[31:] *= -1.0                  # and the last one
    o2, _ = oracle.swa_prefill_varlen(q, k2, v2, cu, 9)
    assert np.array_equal(o[5:31], o2[5:31])
    assert not np.array_equal(o[:5], o2[:5])


# ---------------------------------------------------- one window per sequence --
# A packed batch whose sequences have different windows (as the local layers
# of Gemma 2 and Gemma 3 do: 4,096 and 1,024 tokens, Ultralytics glossary,
# section on alternating local and global layers).

LENGTHS = [6, 0, 23, 1, 17, 9]
WINDOWS = [3, 5, 1, 4, 40, 9]     # one sequence of one token, one window wider than its sequence


def _packed(seed, Hq=4, Hkv=2, d=8):
    rng = np.random.default_rng(seed)
    total = sum(LENGTHS)
    cu = np.concatenate([[0], np.cumsum(LENGTHS)]).astype(np.int32)
    return cu, _rand(rng, total, Hq, d), _rand(rng, total, Hkv, d), _rand(rng, total, Hkv, d)


def test_each_sequence_is_the_plain_prefill_with_its_own_window():
    cu, q, k, v = _packed(4)
    o, lse = oracle.swa_prefill_varlen(q, k, v, cu, WINDOWS)
    for s, W in enumerate(WINDOWS):
        lo, hi = cu[s], cu[s + 1]
        if hi == lo:
            continue
        o_ref, lse_ref = oracle.swa_prefill(q[None, lo:hi], k[None, lo:hi], v[None, lo:hi], W)
        assert np.array_equal(o[lo:hi], o_ref[0]), s
        assert np.array_equal(lse[:, lo:hi], lse_ref[0]), s


def test_same_window_everywhere_equals_the_scalar_call():
    cu, q, k, v = _packed(5)
    o1, l1 = oracle.swa_prefill_varlen(q, k, v, cu, 4)
    o2, l2 = oracle.swa_prefill_varlen(q, k, v, cu, [4] * len(LENGTHS))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_pair_count_is_the_sum_of_causal_closed_forms():
    cu, _, _, _ = _packed(6)

    def causal(T, W):
        return W * T - W * (W - 1) // 2 if T >= W else T * (T + 1) // 2

    expect = sum(causal(T, W) for T, W in zip(LENGTHS, WINDOWS))
    assert oracle.count_pairs_varlen(cu, WINDOWS) == expect


def test_brute_force_packed_mask():
    import scipy.special
    cu, q, k, v = _packed(7, Hq=2, Hkv=1, d=6)
    total = len(q)
    seq = np.repeat(np.arange(len(LENGTHS)), LENGTHS)          # sequence of each packed row
    r, j = np.arange(total)[:, None], np.arange(total)[None, :]
    w = np.asarray(WINDOWS)[seq][:, None]
    allowed = (seq[:, None] == seq[None, :]) & (j <= r) & (j > r - w)
    for x in range(total):
        for y in range(total):
            assert oracle.varlen_allowed(x, y, cu, WINDOWS) == bool(allowed[x, y])
    o, lse = oracle.swa_prefill_varlen(q, k, v, cu, WINDOWS, scale=0.4)
    for h in range(2):
        s = 0.4 * q[:, h] @ k[:, 0].T
        s = np.where(allowed, s, -np.inf)
        p = scipy.special.softmax(s, axis=1)
        np.testing.assert_allclose(o[:, h], p @ v[:, 0], atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[h], scipy.special.logsumexp(s, axis=1), atol=1e-12, rtol=0)


def test_windows_below_one_or_bad_offsets_are_rejected():
    cu, q, k, v = _packed(8)
    import pytest
    with pytest.raises(ValueError):
        oracle.swa_prefill_varlen(q, k, v, cu, [1, 1, 0, 1, 1, 1])
    bad = cu.copy()
    bad[2] = bad[3] + 1
    with pytest.raises(ValueError):
        oracle.swa_prefill_varlen(q, k, v, bad, 3)
