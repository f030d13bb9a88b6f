"""Failure path without a GPU fault: a bounded device wait on a barrier that
nothing completes expires, the kernel records SWA_ERR_TIMEOUT in the status
word and returns, and the context keeps working."""
import pytest
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl
from gpu_util import dev, max_err

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives():
    assert swa.swa_get_device_status() == swa.SWA_OK
    swa.swa_debug_expire_wait(10_000)                   # 10 ms
    assert swa.swa_get_device_status() == swa.SWA_ERR_TIMEOUT
    assert swa.swa_get_device_status() == swa.SWA_OK    # read clears it
    # the context is still usable: a normal prefill after the expiry
    q, k, v = wl.prefill_inputs(1, 200, 2, 1, 64, torch.bfloat16, seed=3)
    o = swa.swa_prefill(q.to(dev()), k.to(dev()), v.to(dev()), 50)
    ref, _ = oracle.swa_prefill(q, k, v, 50)
    assert max_err(o, ref) <= 2e-2
    assert swa.swa_get_device_status() == swa.SWA_OK


def test_no_status_after_normal_work():
    w = wl.MISTRAL_DECODE
    q, kc, vc, kn, vn, pos = wl.decode_inputs(4, w.Hq, w.Hkv, w.d, 512, w.dtype, 1, 0, 2000)
    kcd, vcd = kc.to(dev()), vc.to(dev())
    swa.swa_cache_append(kcd, vcd, kn.to(dev()), vn.to(dev()), pos.to(dev()))
    swa.swa_decode(q.to(dev()), kcd, vcd, pos.to(dev()))
    assert swa.swa_get_device_status() == swa.SWA_OK
