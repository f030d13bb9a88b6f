"""Pins of the oracle's backward pass: the gradient of the window prefill
(robocikowo.com opening definition; aivaro.ru sections 3 and 4.1) with
respect to q, k and v.  The pages define only the forward computation, so
the pins are what fixes a derivative: a library's automatic differentiation
of the plain masked attention, central finite differences of the oracle's
own forward pass, and the closed form of a one-key window."""
import numpy as np
import pytest
import torch

import oracle


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _dense_masked(q, k, v, W, symmetric, scale):
    """Attention with an explicit [T,T] mask of -inf (fp64 torch), the
    textbook form the window reduces to."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = (abs(i - j) <= W // 2) if symmetric else ((j <= i) & (j > i - W))
    bias = torch.zeros(T, T, dtype=torch.float64).masked_fill(~allowed, float("-inf"))
    hk = torch.arange(Hq) * Hkv // Hq
    kk, vv = k[:, :, hk], v[:, :, hk]                     # [B,T,Hq,d]
    s = torch.einsum("bihe,bjhe->bhij", q, kk) * scale + bias
    p = torch.softmax(s, dim=-1)
    return torch.einsum("bhij,bjhe->bihe", p, vv)


@pytest.mark.parametrize("W,symmetric", [(1, False), (3, False), (5, False), (20, False), (4, True), (7, True),
                                         (40, True)])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (4, 1)])
def test_matches_autograd_of_the_masked_attention(W, symmetric, Hq, Hkv):
    rng = np.random.default_rng(100 + W + 10 * Hq + Hkv + (7 if symmetric else 0))
    B, T, d = 2, 13, 6
    q, k, v = _rand(rng, B, T, Hq, d), _rand(rng, B, T, Hkv, d), _rand(rng, B, T, Hkv, d)
    g = _rand(rng, B, T, Hq, d)
    scale = 0.45
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = _dense_masked(tq, tk, tv, W, symmetric, scale)
    o.backward(torch.tensor(g))
    dq, dk, dv = oracle.swa_backward(q, k, v, g, W, symmetric=symmetric, scale=scale)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12, rtol=1e-10)


def _loss(q, k, v, g, W, symmetric, scale):
    if symmetric:
        o, _ = oracle.swa_prefill_global(q, k, v, None, W, scale=scale)
    else:
        o, _ = oracle.swa_prefill(q, k, v, W, scale=scale)
    return float((o * g).sum())


@pytest.mark.parametrize("symmetric", [False, True])
def test_central_differences_of_the_forward_oracle(symmetric):
    rng = np.random.default_rng(7 if symmetric else 8)
    B, T, Hq, Hkv, d, W = 1, 11, 4, 2, 5, 4
    q, k, v = _rand(rng, B, T, Hq, d), _rand(rng, B, T, Hkv, d), _rand(rng, B, T, Hkv, d)
    g = _rand(rng, B, T, Hq, d)
    scale = 0.6
    grads = oracle.swa_backward(q, k, v, g, W, symmetric=symmetric, scale=scale)
    eps = 1e-6
    for which, x in enumerate((q, k, v)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]; args_p[which] = xp
            args_m = [q, k, v]; args_m[which] = xm
            fd = (_loss(*args_p, g, W, symmetric, scale) - _loss(*args_m, g, W, symmetric, scale)) / (2 * eps)
            assert abs(fd - grads[which][idx]) < 1e-7 * max(1.0, abs(fd)), (which, idx, fd, grads[which][idx])


def test_one_key_window_closed_form():
    # W = 1: each row's softmax is over itself alone, p = 1 whatever q and k
    # are, so dq = dk = 0 and dv sums the upstream gradient of its query heads
    rng = np.random.default_rng(9)
    B, T, Hq, Hkv, d = 2, 7, 4, 2, 3
    q, k, v = _rand(rng, B, T, Hq, d), _rand(rng, B, T, Hkv, d), _rand(rng, B, T, Hkv, d)
    g = _rand(rng, B, T, Hq, d)
    dq, dk, dv = oracle.swa_backward(q, k, v, g, 1)
    assert np.array_equal(dq, np.zeros_like(dq)) and np.array_equal(dk, np.zeros_like(dk))
    np.testing.assert_allclose(dv, g.reshape(B, T, Hkv, Hq // Hkv, d).sum(axis=3), atol=1e-15, rtol=0)


def test_gradient_of_a_constant_upstream_along_v_is_zero_for_q_and_k():
    # dO_i = c for every row with v_j = u for every key: o_i = u whatever p
    # is, so the loss c.u does not depend on q or k
    rng = np.random.default_rng(10)
    B, T, Hq, Hkv, d, W = 1, 9, 2, 1, 4, 3
    q, k = _rand(rng, B, T, Hq, d), _rand(rng, B, T, Hkv, d)
    v = np.broadcast_to(_rand(rng, d), (B, T, Hkv, d)).copy()
    g = np.broadcast_to(_rand(rng, d), (B, T, Hq, d)).copy()
    dq, dk, _ = oracle.swa_backward(q, k, v, g, W)
    assert np.abs(dq).max() < 1e-13 and np.abs(dk).max() < 1e-13
