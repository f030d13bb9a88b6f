"""Parity cases of every compute call, run by test_gpu_debug_build.py in a
subprocess with SWA_DEBUG=1, i.e. through libswa_debug.so, whose kernels check
their own tile, row and slot indices on the device.  Each case must match the
oracle and leave the status word clear (no check fired).  Not collected by
pytest on its own (no test_ prefix)."""
import numpy as np
import torch

import decode_swa_prefill_b200 as swa
import oracle
from decode_swa_prefill_b200 import workloads as wl

TOL = 2e-2


def check(name, got, ref):
    err = float(np.abs(got.float().cpu().double().numpy() - ref).max())
    st = swa.swa_get_device_status()
    assert st == swa.SWA_OK, "%s: status %d (%s)" % (name, st, swa.swa_status_string(st))
    assert err <= TOL, "%s: max abs err %g" % (name, err)
    print("%-24s ok  err %.2e" % (name, err))


def run_all():
    assert swa.library_path.endswith("libswa_debug.so"), swa.library_path
    dev = torch.device("cuda:0")
    d = lambda t: t.to(dev)
    q, k, v = wl.prefill_inputs(2, 300, 4, 2, 128, torch.bfloat16, seed=21)
    for W in (1, 40, 200, 400):
        check("prefill W=%d" % W, swa.swa_prefill(d(q), d(k), d(v), W), oracle.swa_prefill(q, k, v, W)[0])
    q6, k6, v6 = wl.prefill_inputs(2, 300, 4, 2, 64, torch.bfloat16, seed=22)
    check("prefill narrow d=64", swa.swa_prefill(d(q6), d(k6), d(v6), 40), oracle.swa_prefill(q6, k6, v6, 40)[0])
    gi = wl.global_positions(2, 300, 5, seed=23)
    check("prefill_global", swa.swa_prefill_global(d(q), d(k), d(v), d(gi), 64),
          oracle.swa_prefill_global(q, k, v, gi, 64)[0])
    check("prefill_sinks", swa.swa_prefill_sinks(d(q), d(k), d(v), 40, 4), oracle.swa_prefill_sinks(q, k, v, 40, 4)[0])
    check("prefill_dilated", swa.swa_prefill_dilated(d(q), d(k), d(v), 16, 3),
          oracle.swa_prefill_dilated(q, k, v, 16, 3)[0])
    qc, kc_, vc_, rk, rv = wl.chunk_inputs(2, 150, 8, 2, 128, 256, torch.bfloat16, seed=24)
    cpos = torch.tensor([0, 700], dtype=torch.int32)
    check("prefill_chunk", swa.swa_prefill_chunk(d(qc), d(kc_), d(vc_), d(rk), d(rv), d(cpos)),
          oracle.swa_prefill_chunk(qc, kc_, vc_, rk, rv, cpos)[0])
    qp, kp, vp = q.reshape(600, 4, 128), k.reshape(600, 2, 128), v.reshape(600, 2, 128)
    cu = torch.tensor([0, 129, 129, 600], dtype=torch.int32)
    win = torch.tensor([17, 5, 200], dtype=torch.int32)
    check("prefill_varlen", swa.swa_prefill_varlen(d(qp), d(kp), d(vp), d(cu), d(win), 471),
          oracle.swa_prefill_varlen(qp, kp, vp, cu, [17, 5, 200])[0])
    for B, W in ((3, 256), (2, 4096)):        # 2 and 32 splits
        qd, kc, vc, kn, vn, pos = wl.decode_inputs(B, 8, 2, 128, W, torch.bfloat16, seed=W, pos_lo=0, pos_hi=9000)
        kcd, vcd = d(kc), d(vc)
        swa.swa_cache_append(kcd, vcd, d(kn), d(vn), d(pos))
        rk2, rv2, _ = oracle.ring_append(kc, vc, kn, vn, pos)
        check("decode B=%d W=%d" % (B, W), swa.swa_decode(d(qd), kcd, vcd, d(pos)), oracle.swa_decode(qd, rk2, rv2, pos)[0])
    qd, kc, vc, kn, vn, pos = wl.decode_inputs(64, 32, 8, 128, 512, torch.bfloat16, seed=5, pos_lo=0, pos_hi=3000)
    kcd, vcd = d(kc), d(vc)
    swa.swa_cache_append(kcd, vcd, d(kn), d(vn), d(pos))
    rk2, rv2, _ = oracle.ring_append(kc, vc, kn, vn, pos)
    check("decode 64 sequences", swa.swa_decode(d(qd), kcd, vcd, d(pos)), oracle.swa_decode(qd, rk2, rv2, pos)[0])
    check("decode_noalloc", swa.swa_decode_noalloc(d(qd), kcd, vcd, d(pos)), oracle.swa_decode(qd, rk2, rv2, pos)[0])
    # paged ring: pages of 16 slots in a scrambled order
    B, W, P = 3, 128, 16
    table = torch.randperm(B * W // P + 2, generator=torch.Generator().manual_seed(3))[:B * W // P]
    table = table.reshape(B, W // P).to(torch.int32)
    pool_k = torch.zeros(B * W // P + 2, 2, P, 128, dtype=torch.bfloat16)
    pool_v = torch.zeros_like(pool_k)
    qd, _, _, kn, vn, pos = wl.decode_inputs(B, 8, 2, 128, W, torch.bfloat16, seed=7, pos_lo=0, pos_hi=400)
    pk, pv = d(pool_k), d(pool_v)
    swa.swa_cache_append_paged(pk, pv, d(kn), d(vn), d(pos), d(table))
    rk2, rv2, _ = oracle.paged_append(pool_k, pool_v, kn, vn, pos, table)
    check("decode_paged", swa.swa_decode_paged(d(qd), pk, pv, d(table), d(pos)),
          oracle.swa_decode_paged(qd, rk2, rv2, table, pos)[0])
    print("debug build: all cases ok")


if __name__ == "__main__":
    run_all()
