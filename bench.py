"""Benchmark of the sliding-window attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic inputs:
  1. causal prefill, Mistral-7B shapes (B=1, T=32768, 32/8 heads, d=128, W=4096)
  2. Longformer-style prefill (B=8, T=4096, 12 heads, d=64, symmetric W=512,
     16 global tokens)
  3. ring append of one new token per sequence and
  4. one decode step over the W=4096-slot ring (64 sequences, 32/8 heads,
     d=128)
`value` is the whole step's in-window attention throughput: 4*d FLOPs per
visible (query, key) pair, summed over the four calls, divided by the step's
device time.  The components are also timed one by one (CUDA events on the
launching stream) and reported against their own rooflines: prefill against
the dense bf16 tensor peak, decode against HBM bandwidth (bytes = the K/V rows
actually read).  Every input is larger than L2, so no flush is needed between
steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun): each rank runs its own replica (weak scaling, no
collective on the data path); ranks are timed on the device and the slowest
rank's time is reported.
"""
import argparse
import itertools
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_swa_prefill_b200 import workloads as wl  # noqa: E402

METRIC = ("prefill in-window TFLOP/s + % BF16 peak; decode HBM GB/s + % of peak (1 B200)")
WORKLOAD = "mistral7b_prefill + longformer_prefill_global + ring_append + mistral7b_decode"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------ accounting --

def causal_pairs(T, W):
    return W * T - W * (W - 1) // 2 if T >= W else T * (T + 1) // 2


def global_pairs(T, W, gidx_row):
    """Visible pairs of one (batch row, head) with a symmetric window and
    global tokens: band rows see band U G, global rows see all T keys."""
    h = W // 2
    i = np.arange(T)
    band = np.minimum(T - 1, i + h) - np.maximum(0, i - h) + 1
    g = np.asarray(gidx_row, dtype=np.int64)
    is_g = np.zeros(T, dtype=bool)
    is_g[g] = True
    # globals outside row i's band
    in_band = (np.abs(i[:, None] - g[None, :]) <= h).sum(axis=1)
    rows = np.where(is_g, T, band + len(g) - in_band)
    return int(rows.sum())


def step_accounting(inp_lf):
    P, L, D = wl.MISTRAL_PREFILL, wl.LONGFORMER, wl.MISTRAL_DECODE
    f_prefill = causal_pairs(P.T, P.W) * P.B * P.Hq * 4 * P.d
    lf_pairs = sum(global_pairs(L.T, L.W, inp_lf["global_idx"][b].numpy()) for b in range(L.B)) * L.Hq
    f_lf = lf_pairs * 4 * L.d
    # decode positions are >= W: every slot is visible
    f_dec = D.B * D.Hq * D.W * 4 * D.d
    bytes_dec = D.B * D.Hkv * D.W * D.d * 2 * 2
    bytes_prefill = (P.B * P.T * (2 * P.Hq + 2 * P.Hkv) * P.d) * 2
    bytes_lf = (L.B * L.T * (2 * L.Hq + 2 * L.Hkv) * L.d) * 2
    bytes_append = D.B * D.Hkv * D.d * 2 * 2 * 2
    return dict(f_prefill=f_prefill, f_lf=f_lf, f_dec=f_dec, bytes_dec=bytes_dec,
                bytes_prefill=bytes_prefill, bytes_lf=bytes_lf, bytes_append=bytes_append,
                lf_pairs=lf_pairs)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the sources each recorded kernel is built from
KERNEL_SOURCES = {
    "prefill_mistral": ("prefill_pp.cu", "ptx.cuh", "swa_internal.h", "tma_map.h"),
    "longformer": ("prefill_tc.cu", "ptx.cuh", "swa_internal.h", "tma_map.h"),
    "tinymistral": ("narrow_tc.cu", "ptx.cuh", "swa_internal.h", "tma_map.h"),
    "decode_mistral": ("simt_kernels.cu", "ptx.cuh", "swa_internal.h"),
}


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "decode_swa_prefill_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, only if it was taken
    on the kernel's current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """NVML samples of SM clock and throttle reasons while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.02):
        self.index, self.period = index, period
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def report(self):
        if not self.nv or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------ distributed --

def relaunch_command(gpus, argv, port):
    """The torchrun command line that runs this script as `gpus` ranks (one
    process per GPU) with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(gpus),
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else None
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------- GPU arm --

def rank_workload(w, rank):
    """Each rank of a multi-GPU run processes its own batch: same shapes,
    seed offset by the rank (weak scaling)."""
    import dataclasses
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 1000 * rank)


class Step:
    """Device-resident inputs/outputs of one step and the calls that run it."""

    def __init__(self, swa, dev, rank=0):
        self.swa = swa
        P, L, D = (rank_workload(w, rank) for w in (wl.MISTRAL_PREFILL, wl.LONGFORMER, wl.MISTRAL_DECODE))
        self.host = {"prefill": wl.make(P), "lf": wl.make(L), "dec": wl.make(D)}
        hp, hl, hd = self.host["prefill"], self.host["lf"], self.host["dec"]
        self.q, self.k, self.v = (hp[n].to(dev) for n in ("q", "k", "v"))
        self.o = torch.empty_like(self.q)
        self.lq, self.lk, self.lv = (hl[n].to(dev) for n in ("q", "k", "v"))
        self.lg = hl["global_idx"].to(dev)
        self.lo = torch.empty_like(self.lq)
        self.dq = hd["q"].to(dev)
        self.kc, self.vc = hd["k_cache"].to(dev), hd["v_cache"].to(dev)
        self.kn, self.vn = hd["k_new"].to(dev), hd["v_new"].to(dev)
        self.pos = hd["pos"].to(dev)
        self.do = torch.empty_like(self.dq)
        self.ws = torch.empty(max(1, swa.swa_decode_workspace_bytes(D.B, D.Hq, D.Hkv, D.d, D.W)),
                              dtype=torch.uint8, device=dev)
        self.launches_per_step = 1 + 1 + 1 + (2 if self.ws.numel() > 1 else 1)

    def run(self, ev=None):
        """One step; ev: optional list of 8 events bracketing the 4 calls."""
        swa, P, L = self.swa, wl.MISTRAL_PREFILL, wl.LONGFORMER
        if ev: ev[0].record()
        swa.swa_prefill(self.q, self.k, self.v, P.W, o=self.o)
        if ev: ev[1].record(); ev[2].record()
        swa.swa_prefill_global(self.lq, self.lk, self.lv, self.lg, L.W, o=self.lo)
        if ev: ev[3].record(); ev[4].record()
        swa.swa_cache_append(self.kc, self.vc, self.kn, self.vn, self.pos)
        if ev: ev[5].record(); ev[6].record()
        swa.swa_decode(self.dq, self.kc, self.vc, self.pos, o=self.do, workspace=self.ws)
        if ev: ev[7].record()


def gpu_arm(args, world, rank, local):
    import decode_swa_prefill_b200 as swa
    swa.load()
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    st = Step(swa, dev, rank)
    acc = step_accounting(st.host["lf"])
    step_flops = acc["f_prefill"] + acc["f_lf"] + acc["f_dec"]

    for _ in range(args.warmup):
        st.run()
    torch.cuda.synchronize()
    assert swa.swa_get_device_status() == 0, "device status after warm-up"

    # ---- device-timed region: exactly K steps ----
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record()
        for s in range(args.steps):
            st.run(evs[s])
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world)
    status = swa.swa_get_device_status()
    assert status == 0, "device status %d after timed region" % status
    comp = {n: [evs[s][2 * c].elapsed_time(evs[s][2 * c + 1]) for s in range(args.steps)]
            for c, n in enumerate(("prefill", "longformer", "append", "decode"))}
    avg = {n: sum(v) / len(v) for n, v in comp.items()}

    ms_per_step = elapsed_ms / args.steps
    value = world * step_flops / (ms_per_step * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers ----
    e2e = e2e_arm(st, args, world, dev, step_flops)
    extra, tiny_o = tinymistral_arm(swa, dev, args)
    toy, toy_o = toy_arm(swa, dev, args)
    chunk = chunk_arm(swa, dev, args)
    backward = backward_arm(swa, dev, args, peaks)
    sinks = sinks_arm(swa, dev, args, load_peaks()[0])
    dilated = dilated_arm(swa, dev, args, load_peaks()[0])
    varlen = varlen_arm(swa, dev, args, load_peaks()[0])
    paged = paged_arm(swa, st, dev, args, load_peaks()[0])

    peak_t = peaks["bf16_tflops"]
    peak_h = peaks["hbm_gbs"]
    pre_tf = acc["f_prefill"] / (avg["prefill"] * 1e-3) / 1e12
    lf_tf = acc["f_lf"] / (avg["longformer"] * 1e-3) / 1e12
    dec_gbs = acc["bytes_dec"] / (avg["decode"] * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs; no weights)",
        "config": {"workload": WORKLOAD,
                   "prefill": wl.MISTRAL_PREFILL.name, "longformer": wl.LONGFORMER.name,
                   "decode": wl.MISTRAL_DECODE.name, "parallelism": "replica per GPU" if world > 1 else "1 GPU",
                   "l2": "inputs larger than L2 (126 MB) for every kernel; no flush"},
        "components": {
            "prefill": {"tflops": round(pre_tf, 2), "ms": round(avg["prefill"], 4),
                        "frac_of_bf16_peak": round(pre_tf / peak_t, 4), "flops": acc["f_prefill"]},
            "longformer": {"tflops": round(lf_tf, 2), "ms": round(avg["longformer"], 4),
                           "frac_of_bf16_peak": round(lf_tf / peak_t, 4),
                           "gbs": round(acc["bytes_lf"] / (avg["longformer"] * 1e-3) / 1e9, 1),
                           # at the ridge: the slower of the two floors over the time taken
                           "frac_of_min_roofline": round(max(acc["f_lf"] / (peak_t * 1e12),
                                                             acc["bytes_lf"] / (peak_h * 1e9))
                                                         / (avg["longformer"] * 1e-3), 4),
                           "flops": acc["f_lf"]},
            "append": {"us": round(avg["append"] * 1e3, 2)},
            "tinymistral_prefill": extra,
            "toy_f32": toy,
            "chunk_prefill": chunk,
            "prefill_backward": backward,
            "sinks": sinks,
            "dilated": dilated,
            "varlen": varlen,
            "paged_decode": paged,
            "decode": {"gbs": round(dec_gbs, 1), "us": round(avg["decode"] * 1e3, 2),
                       "frac_of_hbm_peak": round(dec_gbs / peak_h, 4),
                       "frac_of_8tbs": round(dec_gbs / 8000.0, 4), "bytes": acc["bytes_dec"]},
        },
        "roofline": {"kernel": "swa_prefill_pp_kernel<128> (Mistral-7B prefill)", "bound": "tensor",
                     "achieved": round(pre_tf, 2), "peak": peak_t, "unit": "TFLOP/s",
                     "frac": round(pre_tf / peak_t, 4), "peak_source": peak_src + " bf16 burst",
                     "traffic": recorded_traffic("prefill_mistral")},
        "roofline_decode": {"kernel": "decode_bulk_kernel<128,4> + decode_combine_kernel", "bound": "hbm",
                            "achieved": round(dec_gbs, 1), "peak": peak_h, "unit": "GB/s",
                            "frac": round(dec_gbs / peak_h, 4), "peak_source": peak_src + " copy",
                            "traffic": recorded_traffic("decode_mistral")},
        "clocks": clk.report(),
        "e2e": e2e,
        "gpu_launches": st.launches_per_step * args.steps,
    }
    if rank == 0 and not args.no_cpu_baseline:
        # the GPU outputs of the five configurations, for the parity check
        # the CPU-baseline leg runs next to its timing
        outs = {"prefill": st.o.cpu(), "longformer": st.lo.cpu(), "decode": st.do.cpu(),
                "tinymistral": tiny_o.cpu(), "toy": toy_o.cpu()}
        line["cpu_baseline"], line["max_abs_err"] = cpu_baseline(args, world, st.host, outs)
    return line


def tinymistral_arm(swa, dev, args):
    """TinyMistral-shaped prefill (B=4, T=2048, 32/8 heads, d=32, W=32): HBM
    bound (25 FLOP per byte), not part of the step.  Its 42 MB fit in L2, so
    L2 is flushed before every timed launch by READING a 256 MB buffer: a
    written flush buffer would leave ~126 MB of dirty lines whose write-back
    then competes with the timed launch."""
    w = wl.TINYMISTRAL
    inp = {k: v.to(dev) for k, v in wl.make(w).items()}
    o = torch.empty_like(inp["q"])
    flush = torch.zeros(32 << 20, dtype=torch.float64, device=dev)   # 256 MB, written once
    sink = torch.empty((), dtype=torch.float64, device=dev)
    torch.cuda.synchronize()
    peaks, _ = load_peaks()
    flops = causal_pairs(w.T, w.W) * w.B * w.Hq * 4 * w.d
    nbytes = w.B * w.T * (2 * w.Hq + 2 * w.Hkv) * w.d * 2
    times = []
    for i in range(args.warmup + max(10, args.steps // 2)):
        torch.sum(flush, dim=0, out=sink)   # read sweep: evicts L2, leaves clean lines
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_prefill(inp["q"], inp["k"], inp["v"], w.W, o=o)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"us": round(ms * 1e3, 2), "gbs": round(gbs, 1), "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4),
            "tflops": round(flops / (ms * 1e-3) / 1e12, 2), "bytes": nbytes, "flops": flops,
            "l2": "flushed before each launch by a 256 MB read sweep", "kernel": "swa_prefill_narrow_kernel",
            "traffic": recorded_traffic("tinymistral")}, o


def toy_arm(swa, dev, args):
    """The fp32 toy configuration (B=1, T=16, W=4, d=64): launch-latency
    bound, reported in microseconds only."""
    w = wl.TOY
    inp = {k: v.to(dev) for k, v in wl.make(w).items()}
    o = torch.empty_like(inp["q"])
    times = []
    for i in range(args.warmup + max(10, args.steps // 2)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_prefill(inp["q"], inp["k"], inp["v"], w.W, o=o)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    return {"us": round(sum(times) / len(times) * 1e3, 2), "workload": w.name, "dtype": "f32",
            "kernel": "prefill_f32_kernel"}, o


def chunk_pairs(n, W, p0):
    """In-window pairs of a chunk of n queries at positions p0.. (each sees
    min(P+1, W) keys)."""
    full = max(0, min(n, n - (W - 1 - p0)))          # rows with P >= W-1
    short = n - full                                # rows with P+1 < W: keys p0+t+1
    return full * W + short * p0 + short * (short + 1) // 2


def chunk_arm(swa, dev, args):
    """Chunked prefill from full rings (4 sequences, 4096-token chunks,
    Mistral-7B shapes): not part of the step.  Its 336 MB of inputs and
    outputs exceed L2, so nothing is flushed."""
    w = wl.MISTRAL_CHUNK
    inp = {k: v.to(dev) for k, v in wl.make(w).items()}
    o = torch.empty_like(inp["q"])
    peaks, _ = load_peaks()
    pairs = sum(chunk_pairs(w.T, w.W, int(p)) for p in inp["pos"].cpu())
    flops = pairs * w.Hq * 4 * w.d
    times = []
    for i in range(args.warmup + max(10, args.steps // 2)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_prefill_chunk(inp["q"], inp["k"], inp["v"], inp["k_cache"], inp["v_cache"], inp["pos"], o=o)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    tf = flops / (ms * 1e-3) / 1e12
    return {"tflops": round(tf, 2), "ms": round(ms, 4), "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
            "flops": flops, "workload": w.name}


def backward_arm(swa, dev, args, peaks):
    """Backward pass of the Mistral-7B prefill (dq, dk, dv for a seeded
    upstream gradient): not part of the step.  FLOPs: 5 matmuls of 2*d per
    in-window pair (the recomputed Q K^T, dO V^T, P^T dO, dS^T Q, dS K), the
    usual 2.5x of the forward's 4*d.  Inputs and outputs (1.3 GB) exceed L2."""
    w = wl.MISTRAL_PREFILL
    q, k, v = (t.to(dev) for t in wl.prefill_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.dtype, w.seed))
    g = torch.Generator().manual_seed(w.seed + 500)
    dout = torch.randn(w.B, w.T, w.Hq, w.d, generator=g).to(w.dtype).to(dev)
    lse = torch.empty(w.B, w.Hq, w.T, dtype=torch.float32, device=dev)
    o = swa.swa_prefill(q, k, v, w.W, lse=lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(swa.swa_prefill_backward_workspace_bytes(w.B, w.T, w.Hq), dtype=torch.uint8, device=dev)
    flops = causal_pairs(w.T, w.W) * w.B * w.Hq * 10 * w.d
    times = []
    for i in range(args.warmup + max(5, args.steps // 4)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_prefill_backward(q, k, v, o, lse, dout, w.W, dq=dq, dk=dk, dv=dv, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    assert swa.swa_get_device_status() == 0, "device status after the backward pass"
    ms = sum(times) / len(times)
    tf = flops / (ms * 1e-3) / 1e12
    return {"tflops": round(tf, 2), "ms": round(ms, 4), "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
            "flops": flops, "workload": w.name + "_backward",
            "kernels": "bwd_delta_kernel + bwd_dq_kernel<128> + bwd_dkdv_kernel<128>"}


def dilated_pairs(T, W, dil, symmetric):
    """In-window pairs of a dilated window (W keys with stride dil, or W//2
    per side)."""
    if not symmetric:
        return sum(min(W, i // dil + 1) for i in range(T))
    h = W // 2
    return sum(min(h, i // dil) + min(h, (T - 1 - i) // dil) + 1 for i in range(T))


def dilated_arm(swa, dev, args, peaks):
    """Dilated symmetric window (Longformer shapes without global tokens,
    dilation 2), timed with its two permutations: not part of the step."""
    w, dil = wl.LONGFORMER, 2
    q, k, v = (t.to(dev) for t in wl.prefill_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.dtype, w.seed))
    o = torch.empty_like(q)
    ws = torch.empty(swa.swa_prefill_dilated_workspace_bytes(w.B, w.T, w.Hq, w.Hkv, w.d, dil), dtype=torch.uint8,
                     device=dev)
    flops = dilated_pairs(w.T, w.W, dil, True) * w.B * w.Hq * 4 * w.d
    times = []
    for i in range(args.warmup + max(10, args.steps // 2)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_prefill_dilated(q, k, v, w.W, dil, symmetric=True, o=o, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    tf = flops / (ms * 1e-3) / 1e12
    return {"tflops": round(tf, 2), "ms": round(ms, 4), "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
            "flops": flops, "dil": dil, "workload": "longformer_B8_T4096_h12_d64_W512_dil2_symmetric"}


def varlen_arm(swa, dev, args, peaks):
    """Packed variable-length prefill: 8 sequences of seeded lengths summing
    to 32768 tokens, Mistral-7B heads and window: not part of the step."""
    w = wl.MISTRAL_PREFILL
    lengths = wl.varlen_lengths(8, w.T, seed=6)
    q, k, v = (t[0].to(dev) for t in wl.prefill_inputs(1, w.T, w.Hq, w.Hkv, w.d, w.dtype, w.seed))
    cu = torch.tensor([0] + list(itertools.accumulate(lengths)), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    flops = sum(causal_pairs(n, w.W) for n in lengths) * w.Hq * 4 * w.d
    times = []
    for i in range(args.warmup + max(10, args.steps // 2)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_prefill_varlen(q, k, v, cu, w.W, max_seqlen=max(lengths), o=o)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    tf = flops / (ms * 1e-3) / 1e12
    res = {"tflops": round(tf, 2), "ms": round(ms, 4), "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
           "flops": flops, "lengths": lengths}
    # the same batch with one window per sequence: 1,024 and 4,096 tokens
    # alternating (the local-layer windows of Gemma 3 and Gemma 2)
    windows = [1024 if s % 2 == 0 else 4096 for s in range(len(lengths))]
    win = torch.tensor(windows, dtype=torch.int32, device=dev)
    flops_m = sum(causal_pairs(n, W) for n, W in zip(lengths, windows)) * w.Hq * 4 * w.d
    times = []
    for i in range(args.warmup + max(10, args.steps // 2)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_prefill_varlen(q, k, v, cu, win, max(lengths), o=o)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    tf = flops_m / (ms * 1e-3) / 1e12
    res["mixed_windows"] = {"windows": windows, "tflops": round(tf, 2), "ms": round(ms, 4),
                            "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4), "flops": flops_m}
    return res


def paged_arm(swa, st, dev, args, peaks):
    """Decode over a paged ring: the 64-sequence decode workload with each
    ring split into pages of 16 slots scattered over a shared pool in a
    seeded random order; not part of the step.  Bytes are the K/V rows read,
    as for the dense decode."""
    D, P = wl.MISTRAL_DECODE, 16
    npg = D.W // P
    g = torch.Generator().manual_seed(77)
    table = torch.randperm(D.B * npg, generator=g).reshape(D.B, npg).to(torch.int32).to(dev)
    kp = torch.empty(D.B * npg, D.Hkv, P, D.d, dtype=D.dtype, device=dev)
    vp = torch.empty_like(kp)
    s = torch.arange(D.W, device=dev)
    for b in range(D.B):
        kp[table[b, s // P].long(), :, s % P] = st.kc[b].permute(1, 0, 2)
        vp[table[b, s // P].long(), :, s % P] = st.vc[b].permute(1, 0, 2)
    o = torch.empty_like(st.dq)
    nbytes = D.B * D.Hkv * D.W * D.d * 2 * 2
    times = []
    for i in range(args.warmup + max(10, args.steps // 2)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        swa.swa_decode_paged(st.dq, kp, vp, table, st.pos, o=o, workspace=st.ws)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    gbs = nbytes / (ms * 1e-3) / 1e9
    same = bool(torch.equal(o, st.do))
    del kp, vp
    return {"page_size": P, "us": round(ms * 1e3, 2), "gbs": round(gbs, 1),
            "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4), "frac_of_8tbs": round(gbs / 8000.0, 4),
            "equal_to_dense_decode": same}


def sink_pairs(T, W, s):
    """In-window pairs of a causal window W plus s sinks: each row's window,
    plus the sinks older than it."""
    return causal_pairs(T, W) + sum(max(0, min(s, i - W + 1)) for i in range(T))


def sinks_arm(swa, dev, args, peaks):
    """Attention sinks (4 per sequence) beside the window: the Mistral-7B
    prefill and decode configurations with sinks, not part of the step."""
    n_sink = 4
    w = wl.MISTRAL_PREFILL
    q, k, v = (t.to(dev) for t in wl.prefill_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.dtype, w.seed))
    o = torch.empty_like(q)
    pf = sink_pairs(w.T, w.W, n_sink) * w.B * w.Hq * 4 * w.d
    wd = wl.MISTRAL_DECODE
    dq, kc, vc, _, _, pos = wl.decode_inputs(wd.B, wd.Hq, wd.Hkv, wd.d, wd.W, wd.dtype, wd.seed, wd.pos_lo,
                                             wd.pos_hi)
    _, ks, vs, _, _, _ = wl.decode_inputs(wd.B, wd.Hq, wd.Hkv, wd.d, n_sink, wd.dtype, wd.seed + 1, 0, 1)
    dq, kc, vc, ks, vs, pos = (t.to(dev) for t in (dq, kc, vc, ks, vs, pos))
    do = torch.empty_like(dq)
    ws = torch.empty(max(1, swa.swa_decode_workspace_bytes(wd.B, wd.Hq, wd.Hkv, wd.d, wd.W)), dtype=torch.uint8,
                     device=dev)
    dbytes = wd.B * wd.Hkv * (wd.W + n_sink) * wd.d * 2 * 2
    res = {}
    for name, fn, work in (
            ("prefill", lambda: swa.swa_prefill_sinks(q, k, v, w.W, n_sink, o=o), pf),
            ("decode", lambda: swa.swa_decode_sinks(dq, kc, vc, ks, vs, pos, o=do, workspace=ws), dbytes)):
        times = []
        for i in range(args.warmup + max(10, args.steps // 2)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                times.append(e0.elapsed_time(e1))
        ms = sum(times) / len(times)
        if name == "prefill":
            tf = work / (ms * 1e-3) / 1e12
            res[name] = {"tflops": round(tf, 2), "ms": round(ms, 4),
                         "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4)}
        else:
            gbs = work / (ms * 1e-3) / 1e9
            res[name] = {"gbs": round(gbs, 1), "us": round(ms * 1e3, 2),
                         "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4)}
    res["n_sink"] = n_sink
    return res


def e2e_arm(st, args, world, dev, step_flops):
    """Per step: pinned host -> device copies of the step's inputs, the four
    calls, device -> host copies of the outputs.  The decode ring is resident
    model state (like weights); the new token's k/v, q and positions are
    inputs.  Steps are pipelined over three streams and two device buffer
    sets: step i+1's inputs are copied in and step i-1's outputs copied out
    while step i computes, each step waiting for exactly the copies it
    needs."""
    import copy

    hp, hl, hd = st.host["prefill"], st.host["lf"], st.host["dec"]
    in_names = ["q", "k", "v", "lq", "lk", "lv", "lg", "dq", "kn", "vn", "pos"]
    out_names = ["o", "lo", "do"]
    host_in = [hp["q"], hp["k"], hp["v"], hl["q"], hl["k"], hl["v"], hl["global_idx"], hd["q"], hd["k_new"],
               hd["v_new"], hd["pos"]]
    host_in = [h.pin_memory() for h in host_in]
    host_out = [torch.empty(getattr(st, n).shape, dtype=getattr(st, n).dtype, pin_memory=True) for n in out_names]
    # a second set of per-step buffers; the ring and the decode workspace are shared
    alt = copy.copy(st)
    for n in in_names + out_names:
        setattr(alt, n, torch.empty_like(getattr(st, n)))
    sets = [st, alt]
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = sum(h.numel() * h.element_size() for h in host_out)
    steps = max(4, args.steps // 4)
    s_in, s_cp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def pipeline(n):
        ev = {k: [torch.cuda.Event() for _ in range(n)] for k in ("in", "cp", "out")}
        for i in range(n):
            bs = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev["cp"][i - 2])      # set no longer read by compute i-2
                for h, name in zip(host_in, in_names):
                    getattr(bs, name).copy_(h, non_blocking=True)
                ev["in"][i].record(s_in)
            with torch.cuda.stream(s_cp):
                s_cp.wait_event(ev["in"][i])
                if i >= 2:
                    s_cp.wait_event(ev["out"][i - 2])     # outputs of step i-2 copied out
                bs.run()
                ev["cp"][i].record(s_cp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["cp"][i])
                for name, h in zip(out_names, host_out):
                    h.copy_(getattr(bs, name), non_blocking=True)
                ev["out"][i].record(s_out)
        return ev

    pipeline(2)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record()
    for s_ in (s_in, s_cp, s_out):
        s_.wait_event(a)
    ev = pipeline(steps)
    cur = torch.cuda.current_stream()
    for k in ("in", "cp", "out"):
        cur.wait_event(ev[k][-1])
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world) / steps
    return {"value": round(world * step_flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "copies": "pipelined: inputs of step i+1 and outputs of step i-1 move while step i computes"}


# ------------------------------------------------------- oracle (CPU) --

def f64_inputs():
    """The step's inputs as fp64 numpy arrays (the oracle's own input type),
    converted once so that the timed oracle calls do not convert them."""
    P, L, D = wl.MISTRAL_PREFILL, wl.LONGFORMER, wl.MISTRAL_DECODE
    f = lambda d: {k: (v.double().numpy() if v.is_floating_point() else v.numpy()) for k, v in d.items()}
    return f(wl.make(P)), f(wl.make(L)), f(wl.make(D))


def oracle_sample(budget_s, seed=0, inputs=None):
    """Run the fp64 oracle on a seeded row sample of every component of the
    step; returns (in-window FLOPs computed, seconds, threads)."""
    import oracle
    rng = np.random.default_rng(seed)
    P, L, D = wl.MISTRAL_PREFILL, wl.LONGFORMER, wl.MISTRAL_DECODE
    threads = oracle.default_threads()
    flops, secs = 0, 0.0
    hp, hl, hd = inputs if inputs is not None else f64_inputs()
    # rows per component in proportion to their share of a step's FLOPs
    plan = [("prefill", 0.80), ("longformer", 0.15), ("decode", 0.05)]
    for name, share in plan:
        t_budget = budget_s * share
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < t_budget:
            if name == "prefill":
                i = rng.integers(P.W, P.T, 64)
                h = rng.integers(0, P.Hq, 64)
                oracle.swa_prefill(hp["q"], hp["k"], hp["v"], P.W,
                                   rows=oracle.row_ids(np.zeros(64, np.int64), h, i, P.Hq, P.T))
                n += 64 * P.W * 4 * P.d
            elif name == "longformer":
                b = rng.integers(0, L.B, 64)
                h = rng.integers(0, L.Hq, 64)
                i = rng.integers(0, L.T, 64)
                oracle.swa_prefill_global(hl["q"], hl["k"], hl["v"], hl["global_idx"], L.W,
                                          rows=oracle.row_ids(b, h, i, L.Hq, L.T))
                gi = hl["global_idx"]
                for bb, ii in zip(b, i):
                    row = gi[bb]
                    if ii in row:
                        n += L.T * 4 * L.d
                    else:
                        hw = L.W // 2
                        band = min(L.T - 1, ii + hw) - max(0, ii - hw) + 1
                        n += (band + int((np.abs(row - ii) > hw).sum())) * 4 * L.d
            else:
                bsel = rng.integers(0, D.B, 2)
                oracle.swa_decode(hd["q"][bsel], hd["k_cache"][bsel], hd["v_cache"][bsel],
                                  hd["pos"][bsel])
                n += 2 * D.Hq * D.W * 4 * D.d
        secs += time.perf_counter() - t0
        flops += n
    return flops, secs, threads


def parity_errors(host, outs, seed=7):
    """Max abs error of the bench's own GPU outputs against the fp64 oracle:
    every row of the TinyMistral, toy and decode configurations, and for the
    Mistral and Longformer prefills a seeded sample of rows of every head
    (the last row of each head, 64 random rows, and every global row)."""
    import oracle
    rng = np.random.default_rng(seed)
    hp, hl, hd = host
    P, L = wl.MISTRAL_PREFILL, wl.LONGFORMER
    err = {}

    def mx(got, ref):
        return float(np.abs(np.asarray(got, dtype=np.float64) - ref).max())

    b, h, i = [], [], []
    for hh in range(P.Hq):
        rows = np.concatenate([[P.T - 1], rng.integers(0, P.T, 64)])
        b += [0] * len(rows); h += [hh] * len(rows); i += rows.tolist()
    b, h, i = map(np.array, (b, h, i))
    ref, _ = oracle.swa_prefill(hp["q"], hp["k"], hp["v"], P.W, rows=oracle.row_ids(b, h, i, P.Hq, P.T))
    err["mistral7b_prefill"] = mx(outs["prefill"][b, i, h].float().numpy(), ref)
    b, h, i = [], [], []
    for bb in range(L.B):
        for hh in range(L.Hq):
            rows = np.concatenate([[L.T - 1], rng.integers(0, L.T, 64), hl["global_idx"][bb]])
            b += [bb] * len(rows); h += [hh] * len(rows); i += rows.tolist()
    b, h, i = map(np.array, (b, h, i))
    ref, _ = oracle.swa_prefill_global(hl["q"], hl["k"], hl["v"], hl["global_idx"], L.W,
                                       rows=oracle.row_ids(b, h, i, L.Hq, L.T))
    err["longformer_prefill"] = mx(outs["longformer"][b, i, h].float().numpy(), ref)
    # decode: the bench appended the new token at pos before every decode
    kc, vc, _ = oracle.ring_append(hd["k_cache"], hd["v_cache"], hd["k_new"], hd["v_new"], hd["pos"])
    ref, _ = oracle.swa_decode(hd["q"], kc, vc, hd["pos"])
    err["mistral7b_decode"] = mx(outs["decode"].float().numpy(), ref)
    for name, w in (("tinymistral", wl.TINYMISTRAL), ("toy", wl.TOY)):
        t = wl.make(w)
        ref, _ = oracle.swa_prefill(t["q"], t["k"], t["v"], w.W)
        err[w.name] = mx(outs[name].float().numpy(), ref)
    err["tolerance"] = {"bf16": 2e-2, "f32": 1e-5}
    return err


def cpu_baseline(args, world, host=None, outs=None):
    """The fp64 oracle timed on the host cores on a bounded sample of the
    step; with the bench's GPU outputs it also reports their max abs error
    against the oracle per configuration (not timed)."""
    inputs = f64_inputs()
    flops, secs, threads = oracle_sample(args.cpu_seconds, inputs=inputs)
    base = {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": "fp64 oracle on seeded row samples of the same step (about %.0f s: "
                      "Mistral prefill rows past W, Longformer rows, decode sequences), scaled by "
                      "their in-window FLOPs; inputs converted to fp64 once, before the timing"
                      % args.cpu_seconds}
    if outs is None:
        return base
    return base, parity_errors(inputs, outs)


def reference_arm(args, world, rank):
    """The oracle as the reference arm: same metric, unit and config, each
    step a bounded row sample of the step's workload on the host cores."""
    if rank != 0:
        return None
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    flops_total, secs_total, threads = 0, 0.0, 1
    inputs = f64_inputs()
    for s in range(args.warmup):
        oracle_sample(min(per_step, 1.0), seed=1000 + s, inputs=inputs)
    for s in range(args.steps):
        f, t, threads = oracle_sample(per_step, seed=s, inputs=inputs)
        flops_total += f
        secs_total += t
    v = flops_total / secs_total / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs_total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "prefill": wl.MISTRAL_PREFILL.name,
                   "longformer": wl.LONGFORMER.name, "decode": wl.MISTRAL_DECODE.name},
        "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": "each step: fp64 oracle on a seeded row sample (~%.1f s) of the "
                                   "step's workload" % per_step},
        "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


PROFILE_CASES = {
    # name: (workload, shape overrides); sizes stay above L2 (126 MB) and a
    # few GB at most so that an ncu capture of one launch ends quickly
    "prefill_small": (wl.MISTRAL_PREFILL, {"T": 8192}),
    "prefill": (wl.MISTRAL_PREFILL, {}),
    "prefill_w512": (wl.MISTRAL_PREFILL, {"T": 16384, "W": 512}),   # the persistent form
    "longformer": (wl.LONGFORMER, {}),
    "tinymistral": (wl.TINYMISTRAL, {}),
    "chunk": (wl.MISTRAL_CHUNK, {}),
    "decode": (wl.MISTRAL_DECODE, {}),
    "backward": (wl.MISTRAL_PREFILL, {"T": 8192}),
}


def profile_case(name, launches):
    """Run one kernel of the path `launches` times (for ncu captures)."""
    import dataclasses

    import decode_swa_prefill_b200 as swa
    w, over = PROFILE_CASES[name]
    w = dataclasses.replace(w, **over)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = {k: v.to(dev) for k, v in wl.make(w).items()}
    if name == "backward":
        lse = torch.empty(w.B, w.Hq, w.T, dtype=torch.float32, device=dev)
        o = swa.swa_prefill(inp["q"], inp["k"], inp["v"], w.W, lse=lse)
        dout = torch.randn(w.B, w.T, w.Hq, w.d, generator=torch.Generator().manual_seed(w.seed + 500)).to(w.dtype)
        dout = dout.to(dev)
    for _ in range(launches):
        if name == "backward":
            swa.swa_prefill_backward(inp["q"], inp["k"], inp["v"], o, lse, dout, w.W)
        elif w.kind == "prefill":
            swa.swa_prefill(inp["q"], inp["k"], inp["v"], w.W)
        elif w.kind == "prefill_global":
            swa.swa_prefill_global(inp["q"], inp["k"], inp["v"], inp["global_idx"], w.W)
        elif w.kind == "prefill_chunk":
            swa.swa_prefill_chunk(inp["q"], inp["k"], inp["v"], inp["k_cache"], inp["v_cache"], inp["pos"])
        else:
            swa.swa_cache_append(inp["k_cache"], inp["v_cache"], inp["k_new"], inp["v_new"], inp["pos"])
            swa.swa_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["pos"])
    torch.cuda.synchronize()
    assert swa.swa_get_device_status() == 0
    print("profile case %s: %d launches ok" % (name, launches))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES))
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case, args.launches)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not under torchrun yet: become `gpus` ranks, one process per GPU
        sys.stdout.flush()
        os.execv(sys.executable, relaunch_command(args.gpus, sys.argv[1:], free_port()))
    if int(os.environ.get("WORLD_SIZE", "1")) != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE is %s" % (args.gpus, os.environ.get("WORLD_SIZE", "1")))
    if args.impl == "reference":
        # rank 0 alone runs the oracle; other ranks exit without work
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = reference_arm(args, world, rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup()
    line = gpu_arm(args, world, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
