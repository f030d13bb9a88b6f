"""Causal windows of at most 64 keys with d = 32 or 64 run on the single-pass
narrow-window kernel (one S tile per 128-row query tile, persistent CTAs):
parity with the oracle across both pads (W <= 32, W <= 64), ragged tails,
group sizes, more units than SMs, and the window-of-one identity."""
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err

pytestmark = pytest.mark.gpu


def run(B, T, Hq, Hkv, d, W, seed):
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, torch.bfloat16, seed)
    lse = torch.full((B, Hq, T), float("nan"), device=dev())
    o = swa.swa_prefill(q.to(dev()), k.to(dev()), v.to(dev()), W, lse=lse)
    torch.cuda.synchronize()
    assert swa.swa_get_device_status() == 0
    ref_o, ref_lse = oracle.swa_prefill(q, k, v, W)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("W", [1, 2, 31, 32, 33, 48, 63, 64])
@pytest.mark.parametrize("T", [1, 100, 128, 129, 390])
def test_narrow_windows(d, W, T):
    o, lse, ref_o, ref_lse = run(2, T, 4, 2, d, W, seed=d * 1000 + W * 10 + T)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (3, 1), (6, 2), (8, 1), (5, 5), (4, 4), (6, 6)])
@pytest.mark.parametrize("W", [20, 60])
@pytest.mark.parametrize("d", [32, 64])
def test_narrow_group_sizes(Hq, Hkv, W, d):
    # d = 32 with one query head per kv head and an even head count loads
    # two heads per tile row
    o, lse, ref_o, ref_lse = run(1, 300, Hq, Hkv, d, W, seed=Hq * 10 + Hkv + W + d)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


@pytest.mark.parametrize("W", [1, 32, 33, 64])
@pytest.mark.parametrize("T", [129, 390])
def test_narrow_paired_heads(W, T):
    o, lse, ref_o, ref_lse = run(2, T, 8, 8, 32, W, seed=W * 7 + T)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


@pytest.mark.parametrize("d,W,Hq,Hkv", [(32, 32, 16, 8), (64, 64, 16, 8), (32, 50, 16, 16)])
def test_narrow_more_units_than_sms(d, W, Hq, Hkv):
    # 3 * 8 * 16 = 384 units of (batch, kv heads, tile) or more: every CTA loops
    o, lse, ref_o, ref_lse = run(3, 2000, Hq, Hkv, d, W, seed=d + W + Hq)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


@pytest.mark.parametrize("d,Hq,Hkv", [(32, 4, 2), (64, 4, 2), (32, 4, 4)])
def test_narrow_window_one_returns_v_exactly(d, Hq, Hkv):
    q, k, v = wl.prefill_inputs(1, 300, Hq, Hkv, d, torch.bfloat16, 8)
    o = swa.swa_prefill(q.to(dev()), k.to(dev()), v.to(dev()), 1)
    assert torch.equal(o.cpu(), v.repeat_interleave(Hq // Hkv, dim=2))


def test_narrow_output_untouched_outside_rows():
    # a ragged last tile: rows past T are not written (the output buffer is a
    # view into a larger tensor whose next rows hold a sentinel)
    B, T, Hq, Hkv, d, W = 1, 130, 4, 2, 32, 16
    q, k, v = (t.to(dev()) for t in wl.prefill_inputs(B, T, Hq, Hkv, d, torch.bfloat16, 4))
    big = torch.full((B, T + 130, Hq, d), 7.0, dtype=torch.bfloat16, device=dev())
    o = big[:, :T]
    swa.swa_prefill(q, k, v, W, o=o)
    torch.cuda.synchronize()
    assert torch.all(big[:, T:] == 7.0)
