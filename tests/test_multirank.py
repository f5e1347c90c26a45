"""Multi-rank host logic of bench.py, on CPU with the gloo backend.

Frames are sharded over ranks (each rank draws its own frames with its own
seed and renders them alone); the only cross-rank steps are the timing
barrier and the aggregation of the per-rank figures: evals summed, times
max-reduced.  These tests run that aggregation on two gloo ranks, and the
reference arm under torchrun with two ranks (rank 0 times the oracle, the
other rank exits 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from differentiable_gaussian_splatting_pdr_b200.inputs import (  # noqa: E402
    WORKLOADS, make_inputs, rank_seed)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["mono64"]
        p, _ = make_inputs(w, rank_seed(w, rank))
        evals = bench.in_grid_evals(p, w.H, w.W, w.k)
        step_ms = 10.0 + 5.0 * rank          # rank 1 is the slower one
        extra = (3.0 * (world - rank), 7.0)  # rank 0 is slower here
        out = bench.aggregate_over_ranks(torch, dist, world, torch.device("cpu"), evals,
                                         step_ms, extra)
        q.put((rank, evals, out))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    evals = [e for _, e, _ in res]
    assert evals[0] != evals[1]  # different seeds, different frames
    for _, _, (ev_all, times) in res:
        assert ev_all == sum(evals)
        assert times == [15.0, 6.0, 7.0]  # max over ranks, element by element
    ev_all, times = res[0][2]
    assert bench.throughput(ev_all, 10, times[0]) == pytest.approx(sum(evals) * 10 / 15e-3)


def test_rank_seeds_shard_distinct_frames():
    w = WORKLOADS["tiny"]
    a, _ = make_inputs(w, rank_seed(w, 0))
    b, _ = make_inputs(w, rank_seed(w, 1))
    assert rank_seed(w, 0) == w.seed
    assert not np.array_equal(a, b)


def test_single_rank_aggregate_is_identity():
    ev, t = bench.aggregate_over_ranks(torch, dist, 1, torch.device("cpu"), 123, 4.5, (1.0,))
    assert ev == 123 and t == [4.5, 1.0]


def test_forward_kernel_attribution():
    assert bench.forward_kernel(WORKLOADS["mono64"]) == "k_fwd_cluster"   # 16 tiles
    assert bench.forward_kernel(WORKLOADS["rgb128"]) == "k_fwd"           # 64 tiles
    assert bench.forward_kernel(WORKLOADS["field32x64"]) == "k_fwd"            # 2560 blocks
    assert bench.forward_kernel(WORKLOADS["tiny"]) == "k_fwd_cluster"


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "tiny", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]


def test_oracle_sample_on_one_core_and_on_all():
    """The CPU baseline's two figures: the oracle on every host core and on one."""
    w = WORKLOADS["tiny"]
    v1, f1, c1, s1, _ = bench.oracle_sample(w, 0.05, threads=1)
    va, fa, ca, sa, _ = bench.oracle_sample(w, 0.05)
    assert c1 == 1 and ca >= 1
    assert v1 > 0 and va > 0 and f1 > 0 and fa > 0
    assert "frames of tiny" in s1 and "frames of tiny" in sa
