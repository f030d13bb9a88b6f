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
