"""Host-side logic of bench.py, CPU only: the in-window FLOP accounting (pinned
to the oracle's pair counts), per-rank workloads, and the multi-rank timing
path (barrier + max over ranks) run as two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
import oracle
from decode_swa_prefill_b200 import workloads as wl


@pytest.mark.parametrize("T,W", [(16, 4), (100, 7), (64, 64), (50, 200)])
def test_causal_pairs_match_oracle(T, W):
    assert bench.causal_pairs(T, W) == oracle.count_pairs(T, W)


@pytest.mark.parametrize("T,W,g", [(60, 8, 0), (60, 8, 3), (100, 20, 7), (40, 100, 5)])
def test_global_pairs_match_oracle(T, W, g):
    gi = wl.global_positions(1, T, g, seed=T + g)[0].numpy()
    assert bench.global_pairs(T, W, gi) == oracle.count_pairs(T, W, oracle.SYMMETRIC, gi if g else None)


@pytest.mark.parametrize("n,W,p0", [(10, 4, 0), (10, 4, 2), (5, 100, 3), (7, 3, 50), (1, 1, 0), (300, 256, 0),
                                     (4096, 4096, 5000)])
def test_chunk_pairs_match_oracle(n, W, p0):
    # rows p0..p0+n-1 of a causal prefill over p0+n tokens
    assert bench.chunk_pairs(n, W, p0) == oracle.count_pairs(p0 + n, W) - oracle.count_pairs(p0, W)


@pytest.mark.parametrize("T,W,s", [(16, 4, 2), (30, 7, 0), (9, 20, 4), (100, 10, 100), (64, 1, 3)])
def test_sink_pairs_match_oracle(T, W, s):
    assert bench.sink_pairs(T, W, s) == oracle.count_pairs_sinks(T, W, s)


@pytest.mark.parametrize("T,W,dil,sym", [(16, 4, 2, False), (30, 6, 3, True), (9, 20, 4, False), (40, 2, 7, True)])
def test_dilated_pairs_match_oracle(T, W, dil, sym):
    mode = oracle.SYMMETRIC if sym else oracle.CAUSAL
    assert bench.dilated_pairs(T, W, dil, sym) == oracle.count_pairs_dilated(T, W, dil, mode)


def test_step_accounting_totals():
    acc = bench.step_accounting(wl.make(wl.LONGFORMER))
    assert acc["f_prefill"] == 125_831_168 * 32 * 4 * 128
    assert acc["bytes_dec"] == 1_073_741_824
    assert acc["f_dec"] == 64 * 32 * 4096 * 4 * 128
    assert acc["f_lf"] == acc["lf_pairs"] * 4 * 64


def test_rank_workloads_differ_only_in_seed():
    w0 = bench.rank_workload(wl.MISTRAL_DECODE, 0)
    w1 = bench.rank_workload(wl.MISTRAL_DECODE, 1)
    assert w0 == wl.MISTRAL_DECODE
    assert (w1.B, w1.Hq, w1.Hkv, w1.d, w1.W) == (w0.B, w0.Hq, w0.Hkv, w0.d, w0.W)
    assert w1.seed != w0.seed


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_setup()
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # each rank reports its own elapsed time; every rank gets the slowest
    out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def _ref_rank(rank, world, port, out):
    import argparse
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world))
    args = argparse.Namespace(steps=1, warmup=0, cpu_seconds=0.5)
    line = bench.reference_arm(args, world, rank) if rank != 0 else "rank0-skipped"
    out[rank] = line


def test_reference_arm_only_rank0_works():
    out = mp.Manager().dict()
    mp.spawn(_ref_rank, args=(2, 0, out), nprocs=2, join=True)
    assert out[1] is None


def _bench_env():
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["PYTHONPATH"] = bench.ROOT
    return env


def test_relaunch_command_is_one_rank_per_gpu():
    cmd = bench.relaunch_command(4, ["--gpus", "4", "--steps", "2"], 12345)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert cmd[cmd.index("--nproc-per-node") + 1] == "4"
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "2"]


def test_gpus_flag_launches_that_many_ranks():
    # --gpus 2 outside torchrun re-executes the script as two ranks; the
    # reference arm (CPU only) then prints one line, from rank 0, that counts
    # both ranks
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2", "--impl",
                          "reference", "--steps", "1", "--warmup", "3", "--cpu-seconds", "1"],
                         capture_output=True, text=True, timeout=900, env=_bench_env())
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_gpus_flag_must_match_the_launcher():
    import subprocess
    import sys
    env = _bench_env()
    env.update(WORLD_SIZE="3", RANK="0")
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2"],
                         capture_output=True, text=True, timeout=300, env=env)
    assert out.returncode != 0 and "WORLD_SIZE" in out.stderr
