"""GPU backward pass against the fp64 oracle: dq, dk, dv of the causal and
symmetric window prefill (the pages' forward definition differentiated; see
oracle.swa_backward), through the C ABI.  Inputs are seeded bf16, the
upstream gradient too; the oracle sees the same bf16 values upcast."""
import numpy as np
import pytest
import torch

import oracle
from decode_swa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu

# bf16 inputs, bf16 P and dS inside the MMAs, fp32 accumulation, bf16 outputs
TOL = 2e-2


def _case(B, T, Hq, Hkv, d, W, symmetric, seed):
    import decode_swa_prefill_b200 as swa
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, torch.bfloat16, seed)
    g = torch.Generator().manual_seed(seed + 500)
    dout = torch.randn(B, T, Hq, d, generator=g).to(torch.bfloat16)
    qd, kd, vd, gd = (x.cuda() for x in (q, k, v, dout))
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    if symmetric:
        o = swa.swa_prefill_global(qd, kd, vd, None, W, lse=lse)
    else:
        o = swa.swa_prefill(qd, kd, vd, W, lse=lse)
    dq, dk, dv = swa.swa_prefill_backward(qd, kd, vd, o, lse, gd, W, symmetric=symmetric)
    torch.cuda.synchronize()
    assert swa.swa_get_device_status() == 0
    ref = oracle.swa_backward(q, k, v, dout, W, symmetric=symmetric)
    out = [x.float().cpu().numpy() for x in (dq, dk, dv)]
    return out, ref


def _check(out, ref, what):
    for name, a, b in zip(("dq", "dk", "dv"), out, ref):
        assert np.isfinite(a).all(), (what, name)
        err = np.abs(a - b).max()
        assert err <= TOL * max(1.0, np.abs(b).max()), (what, name, err, np.abs(b).max())


@pytest.mark.parametrize("T,W", [(1, 1), (130, 1), (257, 17), (300, 128), (300, 129), (200, 400), (384, 256)])
@pytest.mark.parametrize("d", [64, 128])
def test_causal(T, W, d):
    out, ref = _case(2, T, 4, 2, d, W, False, seed=T + W + d)
    _check(out, ref, ("causal", T, W, d))


@pytest.mark.parametrize("T,W", [(257, 2), (300, 64), (300, 257), (150, 600)])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1)])
def test_symmetric(T, W, Hq, Hkv):
    out, ref = _case(1, T, Hq, Hkv, 64, W, True, seed=3 * T + W + Hq)
    _check(out, ref, ("symmetric", T, W, Hq, Hkv))


@pytest.mark.parametrize("Hq,Hkv", [(8, 1), (8, 8), (6, 2)])
def test_group_sizes(Hq, Hkv):
    out, ref = _case(1, 333, Hq, Hkv, 128, 200, False, seed=Hq * 10 + Hkv)
    _check(out, ref, ("groups", Hq, Hkv))


def test_one_key_window_gives_zero_dq_dk():
    # W = 1: p = 1, so ds = dp - D = dO.v - dO.o with o = v.  The kernel takes
    # dp from the MMA and D from a separate fp32 dot product, so the two
    # differ by the rounding of one d-term fp32 sum (about d * 2^-24 * sum of
    # |dO_e v_e|), not by more
    out, ref = _case(1, 200, 4, 2, 64, 1, False, seed=77)
    dq, dk, dv = out
    assert np.abs(dq).max() < 1e-4 and np.abs(dk).max() < 1e-4
    _check(out, ref, "W=1")


def test_larger_mistral_shaped_case():
    # Mistral-7B heads (32/8 scaled down to 8/2), d = 128, a 1024-key window
    # over 2048 tokens: many key tiles per query tile and query tiles per key
    # tile, rows near and far from the sequence start
    out, ref = _case(1, 2048, 8, 2, 128, 1024, False, seed=2024)
    _check(out, ref, "mistral-shaped")
