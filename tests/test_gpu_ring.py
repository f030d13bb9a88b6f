"""Ring-cache append, mask export and decode on the GPU against the oracle,
through the C ABI.  Masks and slot indices must match bit for bit."""
import numpy as np
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, poison_unfilled

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ mask --

@pytest.mark.parametrize("T,W,sym,g", [(16, 4, False, 0), (16, 16, False, 0), (257, 33, False, 0),
                                       (300, 64, True, 0), (4096, 512, True, 16), (100, 7, True, 100)])
def test_mask_bitexact(T, W, sym, g):
    gi = wl.global_positions(1, T, g, seed=T)[0] if g else None
    m = swa.swa_mask_export(T, W, symmetric=sym, global_idx=None if gi is None else gi.to(dev()))
    ref = oracle.mask(T, W, oracle.SYMMETRIC if sym else oracle.CAUSAL, gi)
    assert np.array_equal(m.cpu().numpy(), ref)


def test_mask_page_counts(golden):
    gld = golden("ultralytics_depth_section.txt")
    assert int(swa.swa_mask_export(gld["T"], gld["W"]).sum()) == gld["scores_windowed"]
    assert int(swa.swa_mask_export(gld["T"], gld["T"]).sum()) == gld["scores_full_causal"]


# ---------------------------------------------------------------- append --

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n,W", [(1, 8), (5, 8), (8, 8), (19, 8), (3, 1), (40, 4096)])
def test_append_bitexact(dtype, n, W):
    B, Hkv, d = 3, 2, 64
    gen = torch.Generator().manual_seed(n * 100 + W)
    kc = torch.randn(B, Hkv, W, d, generator=gen).to(dtype)
    vc = torch.randn(B, Hkv, W, d, generator=gen).to(dtype)
    kn = torch.randn(B, n, Hkv, d, generator=gen).to(dtype)
    vn = torch.randn(B, n, Hkv, d, generator=gen).to(dtype)
    pos = torch.tensor([0, 7, 123456], dtype=torch.int32)
    kcd, vcd = kc.to(dev()), vc.to(dev())
    slots = torch.full((B, n), -7, dtype=torch.int32, device=dev())
    swa.swa_cache_append(kcd, vcd, kn.to(dev()), vn.to(dev()), pos.to(dev()), slot_out=slots)
    rk, rv, rs = oracle.ring_append(kc, vc, kn, vn, pos)
    assert np.array_equal(slots.cpu().numpy(), rs)
    # bit copies: compare the exact values
    assert np.array_equal(kcd.cpu().double().numpy(), rk)
    assert np.array_equal(vcd.cpu().double().numpy(), rv)


def test_append_size_constant_and_holds_last_window():
    # append P > W positions one call at a time; content = position
    B, Hkv, d, W, P = 1, 1, 8, 16, 75
    kc = torch.full((B, Hkv, W, d), -1.0, device=dev())
    for p in range(P):
        val = torch.full((B, 1, Hkv, d), float(p), device=dev())
        swa.swa_cache_append(kc, kc, val, val, torch.tensor([p], dtype=torch.int32, device=dev()))
        held = sorted(x for x in kc[0, 0, :, 0].tolist() if x >= 0)
        assert held == list(range(max(0, p + 1 - W), p + 1))
    assert kc.shape == (B, Hkv, W, d)


def test_negative_position_reported():
    kc = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device=dev())
    new = torch.ones(1, 1, 1, 64, dtype=torch.bfloat16, device=dev())
    assert swa.swa_get_device_status() == 0
    swa.swa_cache_append(kc, kc, new, new, torch.tensor([-3], dtype=torch.int32, device=dev()))
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert kc.abs().sum().item() == 0       # untouched
    assert swa.swa_get_device_status() == 0  # cleared


# ---------------------------------------------------------------- decode --

def run_decode(B, Hq, Hkv, d, W, dtype, seed, lo, hi):
    q, kc, vc, kn, vn, pos = wl.decode_inputs(B, Hq, Hkv, d, W, dtype, seed, lo, hi)
    # slots past the current token are never written yet: NaN there pins that
    # the decode never reads them (not merely that it masks them)
    poison_unfilled(kc, vc, [min(int(p) + 1, W) for p in pos])
    kcd, vcd = kc.to(dev()), vc.to(dev())
    swa.swa_cache_append(kcd, vcd, kn.to(dev()), vn.to(dev()), pos.to(dev()))
    lse = torch.full((B, Hq), float("nan"), device=dev())
    o = swa.swa_decode(q.to(dev()), kcd, vcd, pos.to(dev()), lse=lse)
    rk, rv, _ = oracle.ring_append(kc, vc, kn, vn, pos)
    ref_o, ref_lse = oracle.swa_decode(q, rk, rv, pos)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, 2e-2), (torch.float32, 1e-5)])
@pytest.mark.parametrize("Hq,Hkv,d,W,lo,hi", [(8, 2, 64, 50, 0, 200), (4, 4, 32, 300, 0, 1000),
                                               (16, 2, 128, 1000, 500, 3000), (8, 1, 128, 7, 0, 20),
                                               (4, 2, 64, 4096, 0, 9000), (8, 4, 128, 129, 0, 300)])
def test_decode_small(dtype, tol, Hq, Hkv, d, W, lo, hi):
    o, lse, ref_o, ref_lse = run_decode(5, Hq, Hkv, d, W, dtype, seed=W + d + Hq, lo=lo, hi=hi)
    assert max_err(o, ref_o) <= tol
    assert max_err(lse, ref_lse) <= max(tol, 1e-5)


def test_decode_full_config():
    w = wl.MISTRAL_DECODE
    o, lse, ref_o, ref_lse = run_decode(w.B, w.Hq, w.Hkv, w.d, w.W, w.dtype, w.seed, w.pos_lo, w.pos_hi)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


def test_decode_steps_match_prefill_rows_across_wrap():
    """Append one token at a time and decode: step t equals prefill row t
    (the ring wraps several times)."""
    B, T, Hq, Hkv, d, W = 2, 150, 8, 2, 128, 48
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, torch.bfloat16, seed=31)
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    full = swa.swa_prefill(qd, kd, vd, W)
    ref_full, _ = oracle.swa_prefill(q, k, v, W)
    # the ring starts as NaN: a decode step that read a slot not yet written
    # would return NaN
    kc = torch.full((B, Hkv, W, d), float("nan"), dtype=torch.bfloat16, device=dev())
    vc = torch.full_like(kc, float("nan"))
    worst_vs_prefill = 0.0
    for t in range(T):
        pos = torch.full((B,), t, dtype=torch.int32, device=dev())
        swa.swa_cache_append(kc, vc, kd[:, t:t + 1].contiguous(), vd[:, t:t + 1].contiguous(), pos)
        o = swa.swa_decode(qd[:, t].contiguous(), kc, vc, pos)
        assert max_err(o, ref_full[:, t]) <= 2e-2
        worst_vs_prefill = max(worst_vs_prefill, max_err(o, full[:, t].float().cpu().numpy()))
    assert worst_vs_prefill <= 2e-2
