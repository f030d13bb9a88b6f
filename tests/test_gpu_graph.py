"""The hot path inside a CUDA graph: one step (causal prefill, ring append,
split-K decode with its combine) captured on a stream and replayed gives
the same bytes as the eager calls.  Every call is asynchronous and
allocates nothing, so it can be captured; the first (eager) call does the
per-device one-time setup."""
import pytest
import torch

from decode_swa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs():
    q, k, v = wl.prefill_inputs(1, 700, 8, 2, 128, torch.bfloat16, 11)
    names = ("q", "k_cache", "v_cache", "k_new", "v_new", "pos")
    d = wl.decode_inputs(16, 8, 2, 128, 1024, torch.bfloat16, 12, 1024, 5000)
    return [t.cuda() for t in (q, k, v)], {n: t.cuda() for n, t in zip(names, d)}


def _step(swa, pre, dec, o, lse, od, ws):
    q, k, v = pre
    swa.swa_prefill(q, k, v, 300, o=o, lse=lse)
    swa.swa_cache_append(dec["k_cache"], dec["v_cache"], dec["k_new"], dec["v_new"], dec["pos"])
    swa.swa_decode(dec["q"], dec["k_cache"], dec["v_cache"], dec["pos"], o=od, workspace=ws)


def test_captured_step_matches_eager():
    import decode_swa_prefill_b200 as swa
    pre, dec = _inputs()
    B, Hq, d, W = dec["q"].shape[0], dec["q"].shape[1], dec["q"].shape[2], dec["k_cache"].shape[2]
    Hkv = dec["k_cache"].shape[1]
    assert swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W) > 0      # the combine runs
    ws = torch.empty(swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W), dtype=torch.uint8, device="cuda")
    o, od = torch.empty_like(pre[0]), torch.empty_like(dec["q"])
    lse = torch.empty(1, 8, 700, dtype=torch.float32, device="cuda")
    caches = (dec["k_cache"].clone(), dec["v_cache"].clone())

    _step(swa, pre, dec, o, lse, od, ws)                 # eager (and one-time setup)
    torch.cuda.synchronize()
    ref = (o.clone(), lse.clone(), od.clone(), dec["k_cache"].clone(), dec["v_cache"].clone())

    dec["k_cache"].copy_(caches[0]); dec["v_cache"].copy_(caches[1])
    o.zero_(); lse.zero_(); od.zero_()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        _step(swa, pre, dec, o, lse, od, ws)
    for _ in range(3):                                   # replays start from the same caches
        dec["k_cache"].copy_(caches[0]); dec["v_cache"].copy_(caches[1])
        o.zero_(); od.zero_()
        g.replay()
        torch.cuda.synchronize()
        got = (o, lse, od, dec["k_cache"], dec["v_cache"])
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    assert swa.swa_get_device_status() == 0
