"""Pins of the oracle's paged ring: the W slots of each sequence's ring live
in W/P pages of a shared pool, in any order (Ultralytics glossary,
ring-buffer paragraph: position i in slot i mod w; dupenodi.dev check-yourself
question 1: only the window is kept).  Gathering the pages back through the
table must give exactly the dense ring that oracle.ring_append builds; a
decode step over the pages must equal, bit for bit, the dense decode; pages no
table names are never written; and stepping a sequence token by token through
the paged ring reproduces the prefill rows.  CPU only."""
import numpy as np
import pytest

import oracle


def unpage(pool, table):
    """Dense [B,Hkv,W,d] ring from pool [num_pages,Hkv,P,d] and table [B,W/P]."""
    P = pool.shape[2]
    B, npg = table.shape
    W = npg * P
    s = np.arange(W)
    return np.stack([pool[table[b, s // P], :, s % P].transpose(1, 0, 2) for b in range(B)])


def setup(seed, B=3, Hkv=2, d=8, W=24, P=4, spare=5):
    rng = np.random.default_rng(seed)
    npg = W // P
    num_pages = B * npg + spare
    table = rng.permutation(num_pages)[:B * npg].reshape(B, npg).astype(np.int32)
    kp = rng.standard_normal((num_pages, Hkv, P, d))
    vp = rng.standard_normal((num_pages, Hkv, P, d))
    return rng, table, kp, vp


@pytest.mark.parametrize("n", [1, 5, 24, 27])
def test_paged_append_is_the_dense_ring(n):
    rng, table, kp, vp = setup(n)
    B, Hkv, d = 3, 2, 8
    kn, vn = rng.standard_normal((B, n, Hkv, d)), rng.standard_normal((B, n, Hkv, d))
    pos = np.array([0, 7, 1000], dtype=np.int32)
    kp2, vp2, slots = oracle.paged_append(kp, vp, kn, vn, pos, table)
    rk, rv, rs = oracle.ring_append(unpage(kp, table), unpage(vp, table), kn, vn, pos)
    assert np.array_equal(unpage(kp2, table), rk) and np.array_equal(unpage(vp2, table), rv)
    assert np.array_equal(slots, rs)
    unused = np.setdiff1d(np.arange(kp.shape[0]), table.reshape(-1))
    assert len(unused) and np.array_equal(kp2[unused], kp[unused]) and np.array_equal(vp2[unused], vp[unused])


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (2, 2), (8, 1)])
def test_paged_decode_is_the_dense_decode(Hq, Hkv):
    rng, table, kp, vp = setup(Hq * 10 + Hkv, Hkv=Hkv)
    q = rng.standard_normal((3, Hq, 8))
    pos = np.array([3, 23, 5000], dtype=np.int32)      # partly filled, exactly full, wrapped
    o, lse = oracle.swa_decode_paged(q, kp, vp, table, pos)
    o_ref, lse_ref = oracle.swa_decode(q, unpage(kp, table), unpage(vp, table), pos)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


def test_paged_steps_follow_the_prefill_rows():
    # one sequence appended token by token into pages of 4 slots, W = 12,
    # with a scrambled table: each decode step equals the prefill row
    rng = np.random.default_rng(9)
    T, Hq, Hkv, d, W, P = 40, 4, 2, 8, 12, 4
    q, k, v = (rng.standard_normal((1, T, h, d)) for h in (Hq, Hkv, Hkv))
    ref, _ = oracle.swa_prefill(q, k, v, W)
    table = np.array([[5, 0, 3]], dtype=np.int32)
    kp = np.full((6, Hkv, P, d), np.nan)           # never-written rows are NaN
    vp = np.full((6, Hkv, P, d), np.nan)
    for t in range(T):
        pos = np.array([t], dtype=np.int32)
        kp, vp, _ = oracle.paged_append(kp, vp, k[:, t:t + 1], v[:, t:t + 1], pos, table)
        o, _ = oracle.swa_decode_paged(q[:, t], kp, vp, table, pos)
        np.testing.assert_allclose(o, ref[:, t], atol=1e-12, rtol=0)


def test_page_outside_the_pool_is_an_error():
    rng, table, kp, vp = setup(3)
    bad = table.copy()
    bad[1, 2] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.swa_decode_paged(rng.standard_normal((3, 4, 8)), kp, vp, bad, np.array([30, 30, 30], np.int32))
    with pytest.raises(ValueError):
        oracle.paged_append(kp, vp, np.zeros((3, 24, 2, 8)), np.zeros((3, 24, 2, 8)), np.zeros(3, np.int32), bad)
