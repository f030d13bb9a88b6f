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
                                 (400, 400), (257, 1000), (700, 256), (650, 255), (1300, 1024), (1300, 1025)])
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


@pytest.mark.parametrize("W", [64, 2048])
def test_large_scores_exercise_every_rescale(W):
    # q scaled by 4 (exact in bf16): log2-unit scores with a standard
    # deviation near 6, so a row's running maximum is raised again and again,
    # in a third of the rows also in the middle of a key tile -- the paths
    # that rescale l, O and (in the 128-key kernel) the P chunks already
    # written; W = 2048 at d = 128 runs the 128-key kernel, W = 64 the 64-key
    # band kernel.  (Scaled by 8 or 16, the scores are so spread that bf16
    # probabilities alone cost about 0.016 of max error, and every kernel
    # here reaches 0.020-0.022.)
    q, k, v = wl.prefill_inputs(1, 3000, 8, 2, 128, torch.bfloat16, seed=W)
    q = q * 4
    lse = torch.full((1, 8, 3000), float("nan"), device=dev())
    o = swa.swa_prefill(q.to(dev()), k.to(dev()), v.to(dev()), W, lse=lse)
    ref_o, ref_lse = oracle.swa_prefill(q, k, v, W)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


@pytest.mark.parametrize("d", [64, 128])
def test_masked_keys_weigh_exactly_zero(d):
    # W = 1: in each key tile every key but one is masked for a row.  Odd
    # keys carry 2^127, so a masked key given any weight at all (even the
    # smallest normal float, 2^-126, times 2^127 is 2) would move an even
    # row's output away from 1.0; the rows must return their own V exactly.
    q, k, v = wl.prefill_inputs(1, 256, 2, 1, d, torch.bfloat16, 8)
    v = torch.ones_like(v)
    v[:, 1::2] = 2.0 ** 127
    o = swa.swa_prefill(q.to(dev()), k.to(dev()), v.to(dev()), 1)
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
                                   (200, 2, 130), (64, 500, 3),
                                   # symmetric windows of 256+ keys without globals: the 128-key kernel
                                   (300, 300, 0), (517, 600, 0), (260, 254, 0), (700, 256, 0),
                                   # spans of 1023 and 1101 keys: either side of its persistent form
                                   (1100, 1022, 0), (1400, 1100, 0)])
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
# Every head of every sequence at the headline shapes: the rows where the
# window is still filling or clipped (the first W+128 and the last 128 of a
# causal sequence; the first and last W/2+128 of a symmetric one), every
# global row, and at least 1% of the rows drawn at random per head.

def head_rows(T, head_start, tail, n_random, rng, extra=()):
    pick = set(range(min(T, head_start))) | set(range(max(0, T - tail), T)) | set(int(x) for x in extra)
    mid = np.array(sorted(set(range(T)) - pick))
    if len(mid):
        pick |= set(rng.choice(mid, size=min(len(mid), n_random), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def all_head_rows(B, H, T, head_start, tail, seed, extra=None):
    rng = np.random.default_rng(seed)
    n_random = -(-T // 100)          # at least 1% of the rows of each head
    bs, hs, is_ = [], [], []
    for b in range(B):
        for h in range(H):
            r = head_rows(T, head_start, tail, n_random, rng, extra[b] if extra is not None else ())
            bs.append(np.full(len(r), b)); hs.append(np.full(len(r), h)); is_.append(r)
    return np.concatenate(bs), np.concatenate(hs), np.concatenate(is_)


def f64(*ts):
    return [t.double().numpy() for t in ts]


def test_tinymistral_full():
    w = wl.TINYMISTRAL
    inp = wl.make(w)
    lse = torch.empty((w.B, w.Hq, w.T), device=dev())
    o = swa.swa_prefill(inp["q"].to(dev()), inp["k"].to(dev()), inp["v"].to(dev()), w.W, lse=lse)
    ref_o, ref_lse = oracle.swa_prefill(inp["q"], inp["k"], inp["v"], w.W)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 2e-2


def test_mistral_prefill_full_every_head():
    w = wl.MISTRAL_PREFILL
    inp = wl.make(w)
    lse = torch.empty((w.B, w.Hq, w.T), device=dev())
    o = swa.swa_prefill(inp["q"].to(dev()), inp["k"].to(dev()), inp["v"].to(dev()), w.W, lse=lse)
    o_cpu, lse_cpu = o.cpu(), lse.cpu()
    assert torch.isfinite(o_cpu).all() and torch.isfinite(lse_cpu).all()
    b, h, i = all_head_rows(w.B, w.Hq, w.T, w.W + 128, 128, seed=1)
    assert len(set(h.tolist())) == w.Hq
    q, k, v = f64(inp["q"], inp["k"], inp["v"])
    ref_o, ref_lse = oracle.swa_prefill(q, k, v, w.W, rows=oracle.row_ids(b, h, i, w.Hq, w.T))
    assert max_err(o_cpu[b, i, h], ref_o) <= 2e-2
    assert max_err(lse_cpu[b, h, i], ref_lse) <= 2e-2


def test_longformer_full_every_head():
    w = wl.LONGFORMER
    inp = wl.make(w)
    lse = torch.empty((w.B, w.Hq, w.T), device=dev())
    gi = inp["global_idx"]
    o = swa.swa_prefill_global(inp["q"].to(dev()), inp["k"].to(dev()), inp["v"].to(dev()),
                               gi.to(dev()), w.W, lse=lse)
    o_cpu, lse_cpu = o.cpu(), lse.cpu()
    assert torch.isfinite(o_cpu).all() and torch.isfinite(lse_cpu).all()
    b, h, i = all_head_rows(w.B, w.Hq, w.T, w.W // 2 + 128, w.W // 2 + 128, seed=2, extra=gi.numpy())
    assert len(set(h.tolist())) == w.Hq and len(set(b.tolist())) == w.B
    q, k, v = f64(inp["q"], inp["k"], inp["v"])
    ref_o, ref_lse = oracle.swa_prefill_global(q, k, v, gi, w.W, rows=oracle.row_ids(b, h, i, w.Hq, w.T))
    assert max_err(o_cpu[b, i, h], ref_o) <= 2e-2
    assert max_err(lse_cpu[b, h, i], ref_lse) <= 2e-2
