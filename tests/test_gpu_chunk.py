"""Chunked prefill over the W-slot ring (a chunk of new tokens continuing
sequences whose earlier keys are in the ring) on the GPU against the oracle,
through the C ABI: ring tiles read by TMA, ring tiles that wrap around the
ring's end or meet the chunk's first row read by row gathers, partly filled
rings, one-token chunks, and a whole sequence run chunk by chunk."""
import numpy as np
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, poison_unfilled, tol_for

pytestmark = pytest.mark.gpu


def run_chunk(B, n, Hq, Hkv, d, W, pos, dtype, seed):
    q, k, v, kc, vc = wl.chunk_inputs(B, n, Hq, Hkv, d, W, dtype, seed)
    # a ring holding positions 0..pos-1 has written only slots 0..pos-1 when
    # pos < W: the others are NaN, and must never be read
    poison_unfilled(kc, vc, [min(p, W) for p in pos])
    p = torch.tensor(pos, dtype=torch.int32)
    lse = torch.zeros(B, Hq, n, dtype=torch.float32, device=dev())
    o = swa.swa_prefill_chunk(q.to(dev()), k.to(dev()), v.to(dev()), kc.to(dev()), vc.to(dev()), p.to(dev()),
                              lse=lse)
    assert swa.swa_get_device_status() == 0
    ref_o, ref_lse = oracle.swa_prefill_chunk(q, k, v, kc, vc, p)
    return o, lse, ref_o, ref_lse


CASES = [
    (2, 300, 8, 2, 256, [0, 1000]),     # empty ring; ring wrapping inside a tile, chunk start inside a tile
    (1, 130, 4, 4, 100, [37]),          # ring not yet full (37 < W), W below a key tile
    (2, 64, 8, 1, 4096, [5000, 64]),    # tile-aligned chunk starts, ring tiles by TMA
    (3, 1, 8, 2, 50, [0, 7, 123]),      # one-token chunks
    (1, 517, 2, 2, 64, [128]),          # chunk longer than the window
]


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("case", CASES)
def test_chunk_bf16_matches_oracle(d, case):
    B, n, Hq, Hkv, W, pos = case
    o, lse, ref_o, ref_lse = run_chunk(B, n, Hq, Hkv, d, W, pos, torch.bfloat16, seed=n + W + d)
    assert max_err(o, ref_o) <= tol_for(torch.bfloat16)
    assert max_err(lse, ref_lse) <= 1e-2


@pytest.mark.parametrize("case", CASES)
def test_chunk_f32_matches_oracle(case):
    B, n, Hq, Hkv, W, pos = case
    o, lse, ref_o, ref_lse = run_chunk(B, n, Hq, Hkv, 64, W, pos, torch.float32, seed=n + W)
    assert max_err(o, ref_o) <= tol_for(torch.float32)
    assert max_err(lse, ref_lse) <= 1e-5


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 64)])
def test_sequence_chunk_by_chunk_equals_one_prefill(dtype, d):
    # prefill each chunk from the ring, then append it: the rows equal the
    # one-shot prefill of the whole sequence
    sizes, W, Hq, Hkv = [256, 1, 200, 243, 64], 300, 8, 2
    T = sum(sizes)
    q, k, v = wl.prefill_inputs(1, T, Hq, Hkv, d, dtype, seed=d)
    ref_o, _ = oracle.swa_prefill(q, k, v, W)
    kc = torch.full((1, Hkv, W, d), float("nan"), dtype=dtype, device=dev())   # never-written slots
    vc = torch.full_like(kc, float("nan"))
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    p = 0
    outs = []
    for n in sizes:
        pos = torch.tensor([p], dtype=torch.int32, device=dev())
        sl = slice(p, p + n)
        outs.append(swa.swa_prefill_chunk(qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous(),
                                          kc, vc, pos))
        swa.swa_cache_append(kc, vc, kd[:, sl].contiguous(), vd[:, sl].contiguous(), pos)
        p += n
    assert swa.swa_get_device_status() == 0
    assert max_err(torch.cat(outs, dim=1), ref_o) <= tol_for(dtype)


def test_chunk_then_decode_continue_the_ring():
    # chunk prefill, append, then decode the next token: matches the oracle
    B, n, Hq, Hkv, d, W = 2, 96, 8, 2, 128, 128
    q, k, v, kc, vc = wl.chunk_inputs(B, n, Hq, Hkv, d, W, torch.bfloat16, seed=3)
    pos = torch.tensor([200, 5], dtype=torch.int32)
    kcd, vcd = kc.to(dev()), vc.to(dev())
    o = swa.swa_prefill_chunk(q.to(dev()), k.to(dev()), v.to(dev()), kcd, vcd, pos.to(dev()))
    ref_o, _ = oracle.swa_prefill_chunk(q, k, v, kc, vc, pos)
    assert max_err(o, ref_o) <= 2e-2
    swa.swa_cache_append(kcd, vcd, k.to(dev()), v.to(dev()), pos.to(dev()))
    rk, rv, _ = oracle.ring_append(kc, vc, k, v, pos)
    assert np.array_equal(kcd.cpu().double().numpy(), rk)
    q1, k1, v1, _, _ = wl.chunk_inputs(B, 1, Hq, Hkv, d, W, torch.bfloat16, seed=4)
    p1 = pos + n
    swa.swa_cache_append(kcd, vcd, k1.to(dev()), v1.to(dev()), p1.to(dev()))
    rk, rv, _ = oracle.ring_append(rk, rv, k1, v1, p1)
    od = swa.swa_decode(q1[:, 0].contiguous().to(dev()), kcd, vcd, p1.to(dev()))
    ref_d, _ = oracle.swa_decode(q1[:, 0], rk, rv, p1)
    assert max_err(od, ref_d) <= 2e-2


def test_chunk_negative_position_reported():
    B, n, Hq, Hkv, d, W = 1, 16, 2, 1, 64, 32
    q, k, v, kc, vc = wl.chunk_inputs(B, n, Hq, Hkv, d, W, torch.bfloat16, seed=9)
    assert swa.swa_get_device_status() == 0
    swa.swa_prefill_chunk(q.to(dev()), k.to(dev()), v.to(dev()), kc.to(dev()), vc.to(dev()),
                          torch.tensor([-4], dtype=torch.int32, device=dev()))
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_get_device_status() == 0
