"""Packed variable-length causal prefill on the GPU against the oracle,
through the C ABI: sequences shorter and longer than a query tile, empty
sequences, lengths that end inside a tile (rows written one by one there),
and an inconsistent offset table reported through the status word."""
import numpy as np
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, tol_for

pytestmark = pytest.mark.gpu

LENGTHS = [
    [300],                       # one sequence
    [1, 130, 0, 257, 64, 5],     # short, ragged, empty, tile-aligned
    [512, 512],                  # equal lengths
    [17, 400, 3],                # a long one between short ones
]


def run(lengths, Hq, Hkv, d, W, dtype, seed):
    total = sum(lengths)
    q, k, v = wl.prefill_inputs(1, total, Hq, Hkv, d, dtype, seed)
    q, k, v = q[0], k[0], v[0]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    lse = torch.zeros(Hq, total, dtype=torch.float32, device=dev())
    o = swa.swa_prefill_varlen(q.to(dev()), k.to(dev()), v.to(dev()), cu.to(dev()), W, max(lengths), lse=lse)
    assert swa.swa_get_device_status() == 0
    ref_o, ref_lse = oracle.swa_prefill_varlen(q, k, v, cu, W)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("lengths", LENGTHS)
def test_varlen_bf16(d, lengths):
    o, lse, ref_o, ref_lse = run(lengths, 8, 2, d, 100, torch.bfloat16, seed=len(lengths) + d)
    assert max_err(o, ref_o) <= tol_for(torch.bfloat16)
    assert max_err(lse, ref_lse) <= 1e-2


@pytest.mark.parametrize("lengths", LENGTHS)
def test_varlen_f32(lengths):
    o, lse, ref_o, ref_lse = run(lengths, 4, 4, 64, 37, torch.float32, seed=len(lengths))
    assert max_err(o, ref_o) <= tol_for(torch.float32)
    assert max_err(lse, ref_lse) <= 1e-5


# windows of 256 keys or more run on the 128-key kernel: its tiles of a
# sequence start at the sequence's first row, the last one is written row
# by row, and units past a sequence's end do nothing
WIDE = [
    [700],
    [1, 130, 0, 257, 640, 5],
    [512, 512],
    [17, 1000, 3, 300],
]


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("lengths", WIDE)
@pytest.mark.parametrize("W", [256, 300])
def test_varlen_wide_window_bf16(d, lengths, W):
    o, lse, ref_o, ref_lse = run(lengths, 8, 2, d, W, torch.bfloat16, seed=len(lengths) + d + W)
    assert max_err(o, ref_o) <= tol_for(torch.bfloat16)
    assert max_err(lse, ref_lse) <= 1e-2


@pytest.mark.parametrize("Hq,Hkv", [(3, 3), (4, 4), (8, 1)])
def test_varlen_wide_window_group_sizes(Hq, Hkv):
    # odd group size: a CTA holds two row tiles of one head, the second
    # possibly past its sequence's end
    o, lse, ref_o, ref_lse = run([129, 300, 77, 600], Hq, Hkv, 64, 256, torch.bfloat16, seed=Hq + 7 * Hkv)
    assert max_err(o, ref_o) <= 2e-2
    assert max_err(lse, ref_lse) <= 1e-2


def test_odd_group_pairs_row_tiles():
    # group size 1: a CTA holds two row tiles of one head; the second may lie
    # past its sequence's end
    o, lse, ref_o, ref_lse = run([129, 300, 77], 3, 3, 64, 200, torch.bfloat16, seed=5)
    assert max_err(o, ref_o) <= 2e-2


def test_inconsistent_offsets_reported():
    total, Hq, Hkv, d = 100, 2, 1, 64
    q, k, v = (t[0].to(dev()) for t in wl.prefill_inputs(1, total, Hq, Hkv, d, torch.bfloat16, 7))
    cu = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device=dev())   # decreasing entry
    assert swa.swa_get_device_status() == 0
    swa.swa_prefill_varlen(q, k, v, cu, 16, 60)
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_get_device_status() == 0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("W", [1024, 1100])
def test_varlen_long_window_bf16(d, W):
    # a window of up to 1024 keys takes the persistent form of the 128-key
    # kernel, a longer one the one-unit-per-CTA form
    o, lse, ref_o, ref_lse = run([1300, 5, 1200, 129], 8, 2, d, W, torch.bfloat16, seed=d + W)
    assert max_err(o, ref_o) <= tol_for(torch.bfloat16)
    assert max_err(lse, ref_lse) <= 1e-2


def test_inconsistent_offsets_reported_wide_window():
    total, Hq, Hkv, d = 600, 2, 1, 64
    q, k, v = (t[0].to(dev()) for t in wl.prefill_inputs(1, total, Hq, Hkv, d, torch.bfloat16, 8))
    cu = torch.tensor([0, 300, 280, 600], dtype=torch.int32, device=dev())   # decreasing entry
    assert swa.swa_get_device_status() == 0
    swa.swa_prefill_varlen(q, k, v, cu, 256, 320)
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_get_device_status() == 0


# --------------------------------------------------- one window per sequence --

# with one window per sequence the longest sequence picks the kernel: the
# 128-key one from 256 rows (short windows there too), else the 64-key one
MIXED = [
    ([1, 130, 0, 257, 64, 5], [1, 64, 7, 100, 200, 3]),   # window 1, one wider than its sequence, an empty sequence
    ([300, 300, 300], [33, 129, 300]),                    # windows below, across and at a 128-row tile
    ([1, 130, 0, 200, 64, 5], [1, 64, 7, 100, 200, 3]),   # longest sequence below 256 rows
    ([700, 129, 450], [256, 1000, 2]),                    # 128-key tiles, a 2-key window among them
]


def run_mixed(lengths, windows, Hq, Hkv, d, dtype, seed, rows=None):
    total = sum(lengths)
    q, k, v = (t[0] for t in wl.prefill_inputs(1, total, Hq, Hkv, d, dtype, seed))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    win = torch.tensor(windows, dtype=torch.int32)
    lse = torch.zeros(Hq, total, dtype=torch.float32, device=dev())
    o = swa.swa_prefill_varlen(q.to(dev()), k.to(dev()), v.to(dev()), cu.to(dev()), win.to(dev()), max(lengths),
                               lse=lse)
    assert swa.swa_get_device_status() == 0
    ref_o, ref_lse = oracle.swa_prefill_varlen(q, k, v, cu, windows, rows=rows)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("lengths,windows", MIXED)
def test_per_sequence_windows_bf16(d, lengths, windows):
    o, lse, ref_o, ref_lse = run_mixed(lengths, windows, 8, 2, d, torch.bfloat16, seed=d + len(lengths))
    assert max_err(o, ref_o) <= tol_for(torch.bfloat16)
    assert max_err(lse, ref_lse) <= 1e-2


@pytest.mark.parametrize("lengths,windows", MIXED)
def test_per_sequence_windows_f32(lengths, windows):
    o, lse, ref_o, ref_lse = run_mixed(lengths, windows, 4, 4, 64, torch.float32, seed=len(lengths))
    assert max_err(o, ref_o) <= tol_for(torch.float32)
    assert max_err(lse, ref_lse) <= 1e-5


def test_gemma_like_local_windows_in_one_batch():
    # 1,024-token and 4,096-token windows side by side (the local-layer
    # windows of Gemma 3 and Gemma 2), Mistral-7B head shapes; every head,
    # rows at the sequences' edges, their window edges and a random sample
    lengths, windows, Hq, Hkv, d = [5000, 1900, 6000], [1024, 4096, 4096], 32, 8, 128
    cu = np.concatenate([[0], np.cumsum(lengths)])
    rng = np.random.default_rng(3)
    pick = set()
    for s, W in enumerate(windows):
        lo, hi = int(cu[s]), int(cu[s + 1])
        for c in (0, 1, 127, 128, W - 1, W, W + 1, W + 127, W + 128, hi - lo - 1):
            if 0 <= c < hi - lo:
                pick.add(lo + c)
        pick |= set(rng.integers(lo, hi, 40).tolist())
    r = np.array(sorted(pick))
    h = np.repeat(np.arange(Hq), len(r))
    rows = h * sum(lengths) + np.tile(r, Hq)
    o, lse, ref_o, ref_lse = run_mixed(lengths, windows, Hq, Hkv, d, torch.bfloat16, seed=17, rows=rows)
    got = o.cpu()[np.tile(r, Hq), h]
    assert max_err(got, ref_o) <= 2e-2
    assert max_err(lse.cpu()[h, np.tile(r, Hq)], ref_lse) <= 2e-2


@pytest.mark.parametrize("dtype,lengths", [(torch.bfloat16, [100, 60, 90]), (torch.float32, [100, 60, 90]),
                                           (torch.bfloat16, [300, 260, 290])])
def test_window_below_one_reported_and_rows_untouched(dtype, lengths):
    windows = [16, 0, 7] if lengths[0] < 256 else [300, 0, 17]
    total, Hq, Hkv, d = sum(lengths), 4, 2, 64
    q, k, v = (t[0].to(dev()) for t in wl.prefill_inputs(1, total, Hq, Hkv, d, dtype, 9))
    cu_list = [0] + np.cumsum(lengths).tolist()
    cu = torch.tensor(cu_list, dtype=torch.int32, device=dev())
    win = torch.tensor(windows, dtype=torch.int32, device=dev())
    o = torch.full((total, Hq, d), 7.0, dtype=dtype, device=dev())
    assert swa.swa_get_device_status() == 0
    swa.swa_prefill_varlen(q, k, v, cu, win, max(lengths), o=o)
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_get_device_status() == 0
    assert (o[cu_list[1]:cu_list[2]] == 7.0).all()           # the sequence with window 0
    ref, _ = oracle.swa_prefill_varlen(q.cpu(), k.cpu(), v.cpu(), cu_list, [windows[0], 1, windows[2]])
    keep = np.r_[0:cu_list[1], cu_list[2]:total]
    assert max_err(o[keep], ref[keep]) <= tol_for(dtype)
