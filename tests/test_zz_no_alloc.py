"""swa_decode_noalloc keeps its split partials in a static device array
instead of a caller workspace, for callers that cannot allocate device memory
while they decode.  Checked through the C ABI on two calls in a row with
different inputs (the array keeps the first call's partials): against the
fp64 oracle within the decode tolerance, and bit for bit against swa_decode,
which runs the same kernels with the same split count on a workspace.  Every
shape here has more than one split, so the static array is really used.
This file is collected last, so that a failure here leaves every other test
already run."""
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err, poison_unfilled, tol_for

pytestmark = pytest.mark.gpu

# (B, W, dtype, positions drawn from [lo, hi)); 8, 64 and 128 splits
SHAPES = [
    (64, 4096, torch.bfloat16, 4096, 131072),   # the 64-sequence decode workload: every slot filled
    (3, 8192, torch.bfloat16, 0, 12000),        # partly filled rings, other partial offsets
    (1, 16384, torch.float32, 0, 20000),
]


@pytest.mark.parametrize("B,W,dtype,lo,hi", SHAPES)
def test_noalloc_matches_oracle_and_workspace_decode_twice(B, W, dtype, lo, hi):
    w = wl.MISTRAL_DECODE
    assert swa.swa_decode_workspace_bytes(B, w.Hq, w.Hkv, w.d, W) > 0    # the static array is used
    for seed in (101, 202):   # two calls in a row; the array still holds the first call's partials
        q, kc, vc, kn, vn, pos = wl.decode_inputs(B, w.Hq, w.Hkv, w.d, W, dtype, seed, lo, hi)
        poison_unfilled(kc, vc, [min(int(p) + 1, W) for p in pos])
        kcd, vcd, posd = kc.to(dev()), vc.to(dev()), pos.to(dev())
        swa.swa_cache_append(kcd, vcd, kn.to(dev()), vn.to(dev()), posd)
        qd = q.to(dev())
        lse_ref = torch.full((B, w.Hq), float("nan"), device=dev())
        lse_new = torch.full((B, w.Hq), float("nan"), device=dev())
        ref = swa.swa_decode(qd, kcd, vcd, posd, lse=lse_ref)
        got = swa.swa_decode_noalloc(qd, kcd, vcd, posd, lse=lse_new)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        assert torch.equal(lse_new, lse_ref)
        rk, rv, _ = oracle.ring_append(kc, vc, kn, vn, pos)
        ref_o, ref_lse = oracle.swa_decode(q, rk, rv, pos)
        assert max_err(got, ref_o) <= tol_for(dtype)
        assert max_err(lse_new, ref_lse) <= max(tol_for(dtype), 1e-5)


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
