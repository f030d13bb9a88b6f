"""swa_decode_noalloc (scratch in a static device array, for callers that
cannot allocate device memory) against swa_decode (caller workspace), both
through the C ABI, on two calls in a row with different inputs.  This file is
collected last."""
import pytest
import torch

import decode_swa_prefill_b200 as swa
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err

pytestmark = pytest.mark.gpu


def inputs(w, seed, B=None, W=None):
    B = B or w.B
    W = W or w.W
    q, kc, vc, kn, vn, pos = wl.decode_inputs(B, w.Hq, w.Hkv, w.d, W, w.dtype, seed, w.pos_lo, w.pos_hi)
    kcd, vcd = kc.to(dev()), vc.to(dev())
    swa.swa_cache_append(kcd, vcd, kn.to(dev()), vn.to(dev()), pos.to(dev()))
    return q.to(dev()), kcd, vcd, pos.to(dev())


@pytest.mark.parametrize("B,W", [(64, 4096), (5, 300)])
def test_noalloc_matches_workspace_decode_twice(B, W):
    w = wl.MISTRAL_DECODE
    for seed in (101, 202):   # two calls in a row; the scratch keeps the first call's data
        q, kc, vc, pos = inputs(w, seed, B=B, W=W)
        lse_ref = torch.empty(B, w.Hq, device=dev())
        lse_new = torch.full((B, w.Hq), float("nan"), device=dev())
        ref = swa.swa_decode(q, kc, vc, pos, lse=lse_ref)
        got = swa.swa_decode_noalloc(q, kc, vc, pos, lse=lse_new)
        torch.cuda.synchronize()
        assert max_err(got, ref.float().cpu().numpy()) <= 2e-2
        assert max_err(lse_new, lse_ref.cpu().numpy()) <= 2e-2


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # one sequence, 8 query heads on one kv head (a supported group), a
    # 2^20-slot ring: the split partials need 17 MB, above the 16 MiB array;
    # nothing is launched
    shape = (1, 8, 1, 128, 1 << 20)
    need = swa.swa_decode_workspace_bytes(*shape)
    assert need > swa.NOALLOC_SCRATCH_BYTES
    lib = swa.load()
    fake = 1 << 20
    st = lib.swa_decode_noalloc(fake, fake, fake, fake, None, fake, *shape, 0.088, 1, None)
    assert st == swa.SWA_ERR_UNSUPPORTED
    # the largest workload here fits
    assert swa.swa_decode_workspace_bytes(64, 32, 8, 128, 4096) <= swa.NOALLOC_SCRATCH_BYTES
