"""CUDA prefill (tcgen05 bf16 path, SIMT fp32 path) against the fp64 oracle,
through the C ABI.  Small cases span several 128-row tiles with ragged tails;
the named workloads run at full size with sampled rows."""
import numpy as np
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, tol_for

pytestmark = pytest.mark.gpu


def run_causal(B, T, Hq, Hkv, d, W, dtype, seed, with_lse=True):
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, dtype, seed)
    lse = torch.full((B, Hq, T), float("nan"), device=dev()) if with_lse else None
    o = swa.swa_prefill(q.to(dev()), k.to(dev()), v.to(dev()), W, lse=lse)
    torch.cuda.synchronize()
    ref_o, ref_lse = oracle.swa_prefill(q, k, v, W)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("T,W", [(1, 1), (127, 5), (128, 128), (300, 40), (300, 1), (517, 200),
                                 (400, 400), (257, 1000)])
def test_causal_bf16_small(d, T, W):
    o, lse, ref_o, ref_lse = run_causal(2, T, 4, 2, d, W, torch.bfloat16, seed=T * 7 + W + d)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (8, 1), (6, 3), (8, 8)])
def test_causal_bf16_heads(Hq, Hkv):
    o, lse, ref_o, ref_lse = run_causal(1, 260, Hq, Hkv, 64, 70, torch.bfloat16, seed=Hq * 10 + Hkv)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


def test_toy_f32_config():
    w = wl.TOY
    o, lse, ref_o, ref_lse = run_causal(w.B, w.T, w.Hq, w.Hkv, w.d, w.W, w.dtype, w.seed)
    assert max_err(o, ref_o) <= 1e-5
    assert max_err(lse, ref_lse) <= 1e-5


@pytest.mark.parametrize("d", [4, 36, 64, 128])
@pytest.mark.parametrize("T,W", [(33, 4), (70, 70), (90, 200)])
def test_causal_f32_small(d, T, W):
    o, lse, ref_o, ref_lse = run_causal(2, T, 4, 2, d, W, torch.float32, seed=d + T + W)
    assert max_err(o, ref_o) <= 1e-5
    assert max_err(lse, ref_lse) <= 1e-5


def test_window_ge_T_matches_full_causal_on_gpu():
    o, _, ref_o, _ = run_causal(1, 300, 2, 1, 64, 300, torch.bfloat16, seed=5)
    o2, _, _, _ = run_causal(1, 300, 2, 1, 64, 5000, torch.bfloat16, seed=5)
    assert torch.equal(o, o2)
    assert max_err(o, ref_o) <= 2e-2


def test_window_one_returns_v_exactly():
    q, k, v = wl.prefill_inputs(1, 200, 4, 2, 128, torch.bfloat16, 6)
    o = swa.swa_prefill(q.to(dev()), k.to(dev()), v.to(dev()), 1)
    # P == 1 for the single key: O = V rounded through fp32 -> bf16 exactly
    assert torch.equal(o.cpu(), v.repeat_interleave(2, dim=2))


# --------------------------------------------------------------- global --

def run_global(B, T, H, Hkv, d, W, g, dtype, seed, rows=None):
    q, k, v = wl.prefill_inputs(B, T, H, Hkv, d, dtype, seed)
    gi = wl.global_positions(B, T, g, seed)
    lse = torch.full((B, H, T), float("nan"), device=dev())
    o = swa.swa_prefill_global(q.to(dev()), k.to(dev()), v.to(dev()), gi.to(dev()), W, lse=lse)
    torch.cuda.synchronize()
    ref_o, ref_lse = oracle.swa_prefill_global(q, k, v, gi, W)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("T,W,g", [(300, 64, 0), (300, 64, 5), (517, 100, 17), (130, 9, 1),
                                   (200, 2, 130), (64, 500, 3)])
def test_global_bf16_small(d, T, W, g):
    o, lse, ref_o, ref_lse = run_global(2, T, 3, 3, d, W, g, torch.bfloat16, seed=T + W + g + d)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


def test_global_gqa_bf16():
    o, lse, ref_o, ref_lse = run_global(1, 400, 8, 2, 64, 128, 9, torch.bfloat16, seed=77)
    assert max_err(o, ref_o) <= 2e-2


@pytest.mark.parametrize("T,W,g", [(50, 8, 0), (50, 8, 4), (70, 200, 2)])
def test_global_f32_small(T, W, g):
    o, lse, ref_o, ref_lse = run_global(2, T, 2, 1, 64, W, g, torch.float32, seed=T + g)
    assert max_err(o, ref_o) <= 1e-5
    assert max_err(lse, ref_lse) <= 1e-5


# ------------------------------------------------------ full workloads --

def sample_rows(B, Hq, T, W, heads, n_random, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(B):
        for h in heads:
            pick = set(range(min(T, 130))) | set(range(max(0, T - 130), T))
            pick |= {x for c in (127, 128, 255, 256, W - 1, W, W + 1, W + 127, W + 128) for x in (c,) if 0 <= x < T}
            pick |= set(rng.integers(0, T, n_random).tolist())
            rows += [(b, h, i) for i in sorted(pick)]
    b, h, i = map(np.array, zip(*rows))
    return b, h, i


def test_tinymistral_full():
    w = wl.TINYMISTRAL
    inp = wl.make(w)
    lse = torch.empty((w.B, w.Hq, w.T), device=dev())
    o = swa.swa_prefill(inp["q"].to(dev()), inp["k"].to(dev()), inp["v"].to(dev()), w.W, lse=lse)
    ref_o, ref_lse = oracle.swa_prefill(inp["q"], inp["k"], inp["v"], w.W)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


def test_mistral_prefill_full_sampled():
    w = wl.MISTRAL_PREFILL
    inp = wl.make(w)
    lse = torch.empty((w.B, w.Hq, w.T), device=dev())
    o = swa.swa_prefill(inp["q"].to(dev()), inp["k"].to(dev()), inp["v"].to(dev()), w.W, lse=lse)
    b, h, i = sample_rows(w.B, w.Hq, w.T, w.W, heads=[0, 5, 18, 31], n_random=200, seed=1)
    ref_o, ref_lse = oracle.swa_prefill(inp["q"], inp["k"], inp["v"], w.W,
                                        rows=oracle.row_ids(b, h, i, w.Hq, w.T))
    got = o.cpu()[b, i, h]
    assert max_err(got, ref_o) <= 2e-2
    assert max_err(lse.cpu()[b, h, i], ref_lse) <= 2e-2
    # every row: finite, and rows of one head group share keys only
    assert torch.isfinite(o).all()


def test_longformer_full_sampled():
    w = wl.LONGFORMER
    inp = wl.make(w)
    lse = torch.empty((w.B, w.Hq, w.T), device=dev())
    gi = inp["global_idx"]
    o = swa.swa_prefill_global(inp["q"].to(dev()), inp["k"].to(dev()), inp["v"].to(dev()),
                               gi.to(dev()), w.W, lse=lse)
    b, h, i = sample_rows(w.B, w.Hq, w.T, w.W // 2, heads=[0, 7, 11], n_random=100, seed=2)
    # add every global row of the sampled heads
    extra = [(bb, hh, int(x)) for bb in range(w.B) for hh in (0, 7, 11) for x in gi[bb]]
    b = np.concatenate([b, [e[0] for e in extra]]); h = np.concatenate([h, [e[1] for e in extra]])
    i = np.concatenate([i, [e[2] for e in extra]])
    ref_o, ref_lse = oracle.swa_prefill_global(inp["q"], inp["k"], inp["v"], gi, w.W,
                                               rows=oracle.row_ids(b, h, i, w.Hq, w.T))
    assert max_err(o.cpu()[b, i, h], ref_o) <= 2e-2
    assert max_err(lse.cpu()[b, h, i], ref_lse) <= 2e-2
    assert torch.isfinite(o).all()
