"""Paged ring caches on the GPU, through the C ABI: the W slots of each
sequence's ring live in W/P pages of a shared pool, in any order, addressed
through a [B, W/P] page table.  Appends match the oracle's paged append bit
for bit (slots included, pages no table names untouched); decode steps match
the oracle's paged decode within the tolerance and equal, bit for bit, the
dense decode over the same ring gathered back into [B,Hkv,W,d]; a sequence
stepped token by token through a NaN-filled pool follows the prefill rows; a
page outside the pool is reported."""
import numpy as np
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, tol_for

pytestmark = pytest.mark.gpu


def scrambled_table(B, W, P, spare, seed):
    npg = W // P
    g = torch.Generator().manual_seed(seed)
    num_pages = B * npg + spare
    return torch.randperm(num_pages, generator=g)[:B * npg].reshape(B, npg).to(torch.int32), num_pages


def unpage(pool, table):
    """Dense [B,Hkv,W,d] ring gathered from pool [num_pages,Hkv,P,d]."""
    P = pool.shape[2]
    W = table.shape[1] * P
    s = torch.arange(W, device=pool.device)
    table = table.to(pool.device).long()
    rows = [pool[table[b, s // P], :, s % P].permute(1, 0, 2) for b in range(table.shape[0])]
    return torch.stack(rows).contiguous()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n,W,P", [(1, 64, 16), (5, 64, 16), (70, 64, 16), (3, 4096, 64), (2, 8, 1)])
def test_paged_append_bitexact(dtype, n, W, P):
    B, Hkv, d = 3, 2, 64
    table, num_pages = scrambled_table(B, W, P, spare=3, seed=n + W)
    g = torch.Generator().manual_seed(n * 7 + P)
    kp = torch.randn(num_pages, Hkv, P, d, generator=g).to(dtype)
    vp = torch.randn(num_pages, Hkv, P, d, generator=g).to(dtype)
    kn = torch.randn(B, n, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(B, n, Hkv, d, generator=g).to(dtype)
    pos = torch.tensor([0, 9, 123457], dtype=torch.int32)
    kpd, vpd = kp.to(dev()), vp.to(dev())
    slots = torch.full((B, n), -7, dtype=torch.int32, device=dev())
    swa.swa_cache_append_paged(kpd, vpd, kn.to(dev()), vn.to(dev()), pos.to(dev()), table.to(dev()), slot_out=slots)
    assert swa.swa_get_device_status() == 0
    rk, rv, rs = oracle.paged_append(kp, vp, kn, vn, pos, table)
    assert np.array_equal(slots.cpu().numpy(), rs)
    assert np.array_equal(kpd.cpu().double().numpy(), rk)
    assert np.array_equal(vpd.cpu().double().numpy(), rv)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,Hq,Hkv,d,W,P,lo,hi", [
    (5, 8, 2, 128, 256, 16, 0, 600),       # partly filled and wrapped rings
    (4, 8, 8, 64, 1024, 64, 1000, 5000),
    (3, 32, 4, 32, 128, 32, 0, 200),       # group of 8
    (64, 32, 8, 128, 4096, 16, 4096, 131072),   # the 64-sequence decode workload, 16-slot pages
])
def test_paged_decode(dtype, B, Hq, Hkv, d, W, P, lo, hi):
    table, num_pages = scrambled_table(B, W, P, spare=2, seed=W + d)
    q, kc, vc, kn, vn, pos = wl.decode_inputs(B, Hq, Hkv, d, W, dtype, seed=d + B, pos_lo=lo, pos_hi=hi)
    # the dense ring scattered into pages; slots not yet written are NaN
    for b in range(B):
        filled = min(int(pos[b]) + 1, W)
        kc[b, :, filled:] = float("nan")
        vc[b, :, filled:] = float("nan")
    kp = torch.full((num_pages, Hkv, P, d), float("nan"), dtype=dtype)
    vp = torch.full_like(kp, float("nan"))
    s = torch.arange(W)
    for b in range(B):
        kp[table[b, s // P].long(), :, s % P] = kc[b].permute(1, 0, 2)
        vp[table[b, s // P].long(), :, s % P] = vc[b].permute(1, 0, 2)
    kpd, vpd, tbl, posd = kp.to(dev()), vp.to(dev()), table.to(dev()), pos.to(dev())
    swa.swa_cache_append_paged(kpd, vpd, kn.to(dev()), vn.to(dev()), posd, tbl)
    lse = torch.full((B, Hq), float("nan"), device=dev())
    o = swa.swa_decode_paged(q.to(dev()), kpd, vpd, tbl, posd, lse=lse)
    assert swa.swa_get_device_status() == 0
    rk, rv, _ = oracle.paged_append(kp, vp, kn, vn, pos, table)
    ref_o, ref_lse = oracle.swa_decode_paged(q, rk, rv, table, pos)
    assert max_err(o, ref_o) <= tol_for(dtype)
    assert max_err(lse, ref_lse) <= max(tol_for(dtype), 1e-5)
    # the same kernels over the ring gathered back: bit for bit
    lse_d = torch.full((B, Hq), float("nan"), device=dev())
    od = swa.swa_decode(q.to(dev()), unpage(kpd, tbl), unpage(vpd, tbl), posd, lse=lse_d)
    assert torch.equal(o, od) and torch.equal(lse, lse_d)


def test_paged_steps_follow_the_prefill_rows():
    B, T, Hq, Hkv, d, W, P = 2, 150, 8, 2, 128, 48, 16
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, torch.bfloat16, seed=41)
    ref, _ = oracle.swa_prefill(q, k, v, W)
    table, num_pages = scrambled_table(B, W, P, spare=4, seed=5)
    kp = torch.full((num_pages, Hkv, P, d), float("nan"), dtype=torch.bfloat16, device=dev())
    vp = torch.full_like(kp, float("nan"))
    tbl = table.to(dev())
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    worst = 0.0
    for t in range(T):
        pos = torch.full((B,), t, dtype=torch.int32, device=dev())
        swa.swa_cache_append_paged(kp, vp, kd[:, t:t + 1].contiguous(), vd[:, t:t + 1].contiguous(), pos, tbl)
        o = swa.swa_decode_paged(qd[:, t].contiguous(), kp, vp, tbl, pos)
        worst = max(worst, max_err(o, ref[:, t]))
    assert swa.swa_get_device_status() == 0
    assert worst <= 2e-2


def test_page_outside_the_pool_reported():
    B, Hq, Hkv, d, W, P = 2, 4, 2, 64, 64, 16
    table, num_pages = scrambled_table(B, W, P, spare=0, seed=1)
    table[1, 2] = num_pages                      # one page past the pool
    kp = torch.zeros(num_pages, Hkv, P, d, dtype=torch.bfloat16, device=dev())
    new = torch.ones(B, 1, Hkv, d, dtype=torch.bfloat16, device=dev())
    pos = torch.tensor([5, 2 * P + 1], dtype=torch.int32, device=dev())   # row 1 writes into the bad page
    assert swa.swa_get_device_status() == 0
    swa.swa_cache_append_paged(kp, kp, new, new, pos, table.to(dev()))
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert kp.sum().item() == Hkv * d            # only row 0's token was written
    swa.swa_decode_paged(torch.zeros(B, Hq, d, dtype=torch.bfloat16, device=dev()), kp, kp, table.to(dev()),
                         torch.tensor([5, W + 3], dtype=torch.int32, device=dev()))
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_get_device_status() == 0
