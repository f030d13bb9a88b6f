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


# --------------------------------------------------- one window per sequence --

MIXED = [
    ([1, 130, 0, 257, 64, 5], [1, 64, 7, 100, 200, 3]),   # window 1, one wider than its sequence, an empty sequence
    ([300, 300, 300], [33, 129, 300]),                    # windows below, across and at a 128-row tile
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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_window_below_one_reported_and_rows_untouched(dtype):
    lengths, windows = [100, 60, 90], [16, 0, 7]
    total, Hq, Hkv, d = sum(lengths), 4, 2, 64
    q, k, v = (t[0].to(dev()) for t in wl.prefill_inputs(1, total, Hq, Hkv, d, dtype, 9))
    cu = torch.tensor([0, 100, 160, 250], dtype=torch.int32, device=dev())
    win = torch.tensor(windows, dtype=torch.int32, device=dev())
    o = torch.full((total, Hq, d), 7.0, dtype=dtype, device=dev())
    assert swa.swa_get_device_status() == 0
    swa.swa_prefill_varlen(q, k, v, cu, win, 100, o=o)
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert swa.swa_get_device_status() == 0
    assert (o[100:160] == 7.0).all()                          # the sequence with window 0
    ref, _ = oracle.swa_prefill_varlen(q.cpu(), k.cpu(), v.cpu(), [0, 100, 160, 250], [16, 1, 7])
    keep = np.r_[0:100, 160:250]
    assert max_err(o[keep], ref[keep]) <= tol_for(dtype)
