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
