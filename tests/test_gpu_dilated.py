"""Dilated windows on the GPU against the oracle, through the C ABI: causal
and symmetric, sequence lengths that do and do not divide by the dilation,
a dilation above T, and lse."""
import numpy as np
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, tol_for

pytestmark = pytest.mark.gpu

CASES = [
    (1, 300, 8, 2, 64, 3, False),    # T divisible by the dilation
    (2, 517, 4, 4, 100, 4, False),   # one residue class a row longer
    (1, 130, 4, 1, 50, 7, True),     # symmetric
    (1, 64, 2, 2, 16, 64, False),    # dilation = T: each row sees itself
    (1, 100, 8, 8, 8, 150, True),    # dilation above T
]


def run(case, d, dtype, seed):
    B, T, Hq, Hkv, W, dil, sym = case
    q, k, v = wl.prefill_inputs(B, T, Hq, Hkv, d, dtype, seed)
    lse = torch.zeros(B, Hq, T, dtype=torch.float32, device=dev())
    o = swa.swa_prefill_dilated(q.to(dev()), k.to(dev()), v.to(dev()), W, dil, symmetric=sym, lse=lse)
    assert swa.swa_get_device_status() == 0
    ref_o, ref_lse = oracle.swa_prefill_dilated(q, k, v, W, dil, oracle.SYMMETRIC if sym else oracle.CAUSAL)
    return o, lse, ref_o, ref_lse


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("case", CASES)
def test_dilated_bf16(d, case):
    o, lse, ref_o, ref_lse = run(case, d, torch.bfloat16, seed=sum(int(x) for x in case) + d)
    assert max_err(o, ref_o) <= tol_for(torch.bfloat16)
    assert max_err(lse, ref_lse) <= 1e-2


@pytest.mark.parametrize("case", CASES)
def test_dilated_f32(case):
    o, lse, ref_o, ref_lse = run(case, 64, torch.float32, seed=sum(int(x) for x in case))
    assert max_err(o, ref_o) <= tol_for(torch.float32)
    assert max_err(lse, ref_lse) <= 1e-5


def test_dilation_one_is_the_plain_window():
    q, k, v = (t.to(dev()) for t in wl.prefill_inputs(1, 300, 8, 2, 128, torch.bfloat16, 4))
    assert torch.equal(swa.swa_prefill_dilated(q, k, v, 70, 1), swa.swa_prefill(q, k, v, 70))
