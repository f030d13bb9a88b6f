"""Attention sinks (the first tokens kept beside the window) on the GPU
against the oracle, through the C ABI: the prefill with sinks in one or two
gathered key tiles, sinks inside and outside the window, and the decode step
over ring plus sink caches."""
import numpy as np
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, poison_unfilled, tol_for

pytestmark = pytest.mark.gpu

PREFILL_CASES = [
    (1, 300, 8, 2, 64, 4),     # a few sinks, causal window of 64
    (2, 517, 4, 4, 100, 70),   # 70 sinks: two gathered key tiles, ragged T
    (1, 130, 4, 1, 200, 3),    # window wider than T: sinks always inside it
    (1, 200, 2, 2, 1, 5),      # window of one token
    (1, 64, 4, 2, 16, 64),     # every token a sink: full causal attention
    # windows of 256+ keys (the 128-key kernel with one gathered sink tile)
    (1, 700, 8, 2, 256, 4),    # later rows see their sinks only through the sink tile
    (2, 900, 4, 4, 300, 100),  # 100 sinks, inside the window for the first rows
    (1, 400, 4, 1, 600, 8),    # window wider than T: the sink tile is all masked
    (1, 1000, 8, 8, 257, 128), # a full sink tile
    # windows of more than 1024 keys (the one-unit-per-CTA form of that kernel)
    (1, 1400, 4, 2, 1100, 8),
    (2, 1200, 4, 4, 1025, 100),
]


def run_prefill(case, d, dtype, seed):
    B, T, Hq, Hkv, W, s = case
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, dtype, seed)
    lse = torch.zeros(B, Hq, T, dtype=torch.float32, device=dev())
    o = swa.swa_prefill_sinks(q.to(dev()), k.to(dev()), v.to(dev()), W, s, lse=lse)
    assert swa.swa_get_device_status() == 0
    ref_o, ref_lse = oracle.swa_prefill_sinks(q, k, v, W, s)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("case", PREFILL_CASES)
def test_prefill_sinks_bf16(d, case):
    o, lse, ref_o, ref_lse = run_prefill(case, d, torch.bfloat16, seed=sum(case) + d)
    assert max_err(o, ref_o) <= tol_for(torch.bfloat16)
    assert max_err(lse, ref_lse) <= 1e-2


@pytest.mark.parametrize("case", PREFILL_CASES)
def test_prefill_sinks_f32(case):
    o, lse, ref_o, ref_lse = run_prefill(case, 64, torch.float32, seed=sum(case))
    assert max_err(o, ref_o) <= tol_for(torch.float32)
    assert max_err(lse, ref_lse) <= 1e-5


def test_no_sinks_is_the_plain_prefill():
    q, k, v = (t.to(dev()) for t in wl.prefill_inputs(1, 300, 8, 2, 128, torch.bfloat16, 3))
    a = swa.swa_prefill_sinks(q, k, v, 70, 0)
    b = swa.swa_prefill(q, k, v, 70)
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d,Hq,Hkv", [(128, 32, 8), (64, 8, 8), (32, 8, 1)])
def test_decode_sinks(dtype, d, Hq, Hkv):
    B, W, s = 5, 256, 4
    q, kc, vc, _, _, _ = wl.decode_inputs(B, Hq, Hkv, d, W, dtype, seed=d + Hq, pos_lo=0, pos_hi=1)
    _, ks, vs, _, _, _ = wl.decode_inputs(B, Hq, Hkv, d, s, dtype, seed=d + Hq + 1, pos_lo=0, pos_hi=1)
    # before any sink left the window, at the edge, long after, wrapped
    pos = torch.tensor([2, 255, 258, 5000, 100000], dtype=torch.int32)
    # ring slots not written yet, and sink rows the step must take from the
    # ring instead (sinks still inside the window), are NaN: never read
    poison_unfilled(kc, vc, [min(int(p) + 1, W) for p in pos])
    poison_unfilled(ks, vs, [max(0, min(s, int(p) - W + 1)) for p in pos])
    lse = torch.zeros(B, Hq, dtype=torch.float32, device=dev())
    o = swa.swa_decode_sinks(q.to(dev()), kc.to(dev()), vc.to(dev()), ks.to(dev()), vs.to(dev()), pos.to(dev()),
                             lse=lse)
    assert swa.swa_get_device_status() == 0
    ref_o, ref_lse = oracle.swa_decode_sinks(q, kc, vc, ks, vs, pos)
    assert max_err(o, ref_o) <= tol_for(dtype)
    assert max_err(lse, ref_lse) <= (1e-2 if dtype == torch.bfloat16 else 1e-5)


def test_decode_steps_follow_the_prefill():
    # token by token into the ring (and the first s into the sink caches):
    # each decode step equals the prefill row of its position
    B, T, Hq, Hkv, d, W, s = 1, 300, 8, 2, 128, 64, 4
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, torch.bfloat16, seed=12)
    ref_o, _ = oracle.swa_prefill_sinks(q, k, v, W, s)
    # caches start as NaN: a step that read a row not yet written returns NaN
    kc = torch.full((B, Hkv, W, d), float("nan"), dtype=torch.bfloat16, device=dev())
    vc = torch.full_like(kc, float("nan"))
    ks = torch.full((B, Hkv, s, d), float("nan"), dtype=torch.bfloat16, device=dev())
    vs = torch.full_like(ks, float("nan"))
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    errs = []
    for t in range(T):
        pos = torch.tensor([t], dtype=torch.int32, device=dev())
        kt, vt = kd[:, t:t + 1].contiguous(), vd[:, t:t + 1].contiguous()
        swa.swa_cache_append(kc, vc, kt, vt, pos)
        if t < s:
            swa.swa_cache_append(ks, vs, kt, vt, pos)
        if t % 7 == 0 or t > T - 5:
            o = swa.swa_decode_sinks(qd[:, t].contiguous(), kc, vc, ks, vs, pos)
            errs.append(max_err(o, ref_o[:, t]))
    assert swa.swa_get_device_status() == 0
    assert max(errs) <= 2e-2
