"""Pins of the fp64 oracle's counting and ring logic against what the pages
print and against closed forms.  CPU only."""
import numpy as np
import pytest

import oracle


# ------------------------------------------------------------ page values --

def test_scores_per_layer_golden(golden):
    g = golden("ultralytics_depth_section.txt")
    assert oracle.count_pairs(g["T"], g["W"]) == g["scores_windowed"]
    # full causal attention is the window at W >= T
    assert oracle.count_pairs(g["T"], g["T"]) == g["scores_full_causal"]
    assert oracle.count_pairs(g["T"], g["T"] + 5) == g["scores_full_causal"]
    assert int(oracle.mask(g["T"], g["W"]).sum()) == g["scores_windowed"]


def test_reach_golden(golden):
    g = golden("ultralytics_depth_section.txt")
    assert oracle.reach(g["T"], g["W"], 4) == g["reach_layers_1_to_4"]


@pytest.mark.parametrize("W,L", [(2, 5), (3, 4), (5, 3), (7, 2), (1, 3)])
def test_reach_closed_form(W, L):
    # each stacked layer adds W-1 tokens of history: L*(W-1)+1, capped at T
    T = 24
    got = oracle.reach(T, W, L)
    assert got == [min(T, l * (W - 1) + 1) for l in range(1, L + 1)]


def test_mistral_reach_bound(golden):
    g = golden("mistral_reach_and_cache.txt")
    W, L = g["W"], g["L"]
    # the pages' "~131k" is L*W; the exact +W-1-per-layer rule (pinned above on
    # small cases) stays just under it
    exact = L * (W - 1) + 1
    assert exact == 131041
    assert exact <= g["reach_upper_bound"] == L * W


def test_cache_reduction_golden(golden):
    g = golden("mistral_reach_and_cache.txt")
    W, P = g["W"], g["cache_tokens"]
    # append P positions one by one into a W-slot ring (d = 1, content = position)
    kc = np.full((1, 1, W, 1), -1.0)
    vc = np.full((1, 1, W, 1), -1.0)
    kn = np.arange(P, dtype=np.float64).reshape(1, P, 1, 1)
    kc, vc, slots = oracle.ring_append(kc, vc, kn, kn, np.array([0]))
    stored = kc.reshape(-1)
    assert (stored >= 0).sum() == W            # ring never holds more than W
    assert P // (stored >= 0).sum() == g["cache_reduction"]


# ------------------------------------------------------------ closed forms --

def causal_pairs(T, W):
    return W * T - W * (W - 1) // 2 if T >= W else T * (T + 1) // 2


def symmetric_pairs(T, W):
    h = W // 2
    assert T >= 2 * h
    return T * (2 * h + 1) - h * (h + 1)


@pytest.mark.parametrize("T", [1, 2, 5, 16, 33, 100, 257])
@pytest.mark.parametrize("W", [1, 2, 3, 4, 7, 32, 64, 300])
def test_causal_pair_count_closed_form(T, W):
    assert oracle.count_pairs(T, W) == causal_pairs(T, W)


@pytest.mark.parametrize("T", [16, 33, 100, 257])
@pytest.mark.parametrize("W", [0, 1, 2, 3, 4, 8, 15, 32])
def test_symmetric_pair_count_closed_form(T, W):
    if T < 2 * (W // 2):
        pytest.skip("closed form needs T >= W")
    assert oracle.count_pairs(T, W, oracle.SYMMETRIC) == symmetric_pairs(T, W)


def test_config_pair_counts():
    # the exact in-window pair counts the throughput figures are built on
    assert causal_pairs(2048, 32) == 65040
    assert causal_pairs(32768, 4096) == 125_831_168
    assert symmetric_pairs(4096, 512) == 2_035_456
    # and the oracle agrees on scaled-down instances of the same shapes
    assert oracle.count_pairs(2048, 32) == 65040
    assert oracle.count_pairs(1024, 512, oracle.SYMMETRIC) == symmetric_pairs(1024, 512)


def test_window_bounds_explicit():
    # causal [i-W+1, i]; symmetric [i-W/2, i+W/2] (both ends included)
    T, W = 40, 8
    for i in range(T):
        row = [oracle.in_window(i, j, T, W) for j in range(T)]
        assert row == [(i - W + 1) <= j <= i for j in range(T)]
        rows = [oracle.in_window(i, j, T, W, oracle.SYMMETRIC) for j in range(T)]
        assert sum(rows) == min(T - 1, i + 4) - max(0, i - 4) + 1
        assert rows[i] and (i < 4 or rows[i - 4]) and (i + 4 >= T or rows[i + 4])
        assert (i < 5 or not rows[i - 5]) and (i + 5 >= T or not rows[i + 5])


def test_global_mask_rows_and_columns():
    T, W = 50, 6
    gi = np.array([0, 17, 49], dtype=np.int32)
    m = oracle.mask(T, W, oracle.SYMMETRIC, gi)
    band = oracle.mask(T, W, oracle.SYMMETRIC)
    for x in gi:
        assert m[x].all() and m[:, x].all()       # sees all, seen by all
    others = np.setdiff1d(np.arange(T), gi)
    sub = np.ix_(others, others)
    assert (m[sub] == band[sub]).all()              # elsewhere: the band
    assert oracle.count_pairs(T, W, oracle.SYMMETRIC, gi) == int(m.sum())


# ------------------------------------------------------------------- ring --

@pytest.mark.parametrize("W", [1, 4, 7, 32])
def test_ring_slots_and_contents(W):
    P = 3 * W + 5
    kc = np.full((1, 1, W, 1), -1.0)
    kn = np.arange(P, dtype=np.float64).reshape(1, P, 1, 1)
    step = kc
    for p in range(P):
        # one token at a time, like decode: the ring holds [max(0,p+1-W), p]
        step, _, _ = oracle.ring_append(step, step, kn[:, p:p + 1], kn[:, p:p + 1], np.array([p]))
        held = sorted(x for x in step.reshape(-1).tolist() if x >= 0)
        assert held == list(range(max(0, p + 1 - W), p + 1))
    kc2, _, slots = oracle.ring_append(kc, kc, kn, kn, np.array([0]))
    assert list(slots[0]) == [p % W for p in range(P)]
    # holds exactly the last W positions, each in slot pos mod W
    held = kc2.reshape(-1)
    assert sorted(held.tolist()) == list(range(P - W, P))
    for s in range(W):
        assert int(held[s]) % W == s
    assert oracle.slot(123456, 4096) == 123456 % 4096


def test_ring_partial_fill():
    W = 10
    kc = np.full((2, 1, W, 1), -1.0)
    kn = np.arange(6, dtype=np.float64).reshape(1, 6, 1, 1).repeat(2, 0)
    kc2, _, slots = oracle.ring_append(kc, kc, kn, kn, np.array([0, 7]))
    assert list(kc2[0, 0, :, 0]) == [0, 1, 2, 3, 4, 5, -1, -1, -1, -1]
    # second row starts at position 7: slots 7,8,9,0,1,2
    assert list(slots[1]) == [7, 8, 9, 0, 1, 2]


def test_kv_does_not_grow_golden(golden):
    g = golden("kv_growth_check_yourself.txt")
    W, a, b = g["W"], g["first_token"], g["last_token"]
    # tokens are 1-based in the question; positions are 0-based here
    kn = np.arange(b, dtype=np.float64).reshape(1, b, 1, 1)
    kc0 = np.full((1, 1, W, 1), -1.0)
    held_a = oracle.ring_append(kc0, kc0, kn[:, :a], kn[:, :a], np.array([0]))[0]
    held_b = oracle.ring_append(kc0, kc0, kn, kn, np.array([0]))[0]
    assert (held_a >= 0).sum() == (held_b >= 0).sum() == W
    assert sorted(held_b.reshape(-1).tolist()) == list(range(b - W, b))
