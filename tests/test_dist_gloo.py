"""Multi-rank host logic of bench.py, on CPU with the gloo backend and world size 2.

The benchmark shards by sequence: each rank draws its own batch (distinct seeds, same shapes), runs the
whole hot path on it with no data-path collective, and the job's time is the slowest rank's. These
tests run the same Dist / aggregation code the GPU launch uses, as two local processes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from chunk_wise_hierarchical_summary_b200 import workloads as W

    d = bench.Dist(world)
    try:
        d.barrier()
        # rank r pretends its step took 10 + 2r ms: the job time is the slowest rank's
        ms, value = bench.weak_scaling_value(d, 10.0 + 2.0 * rank, 4 * 8192)
        # a second collective in the same order on every rank
        m2 = d.max(float(rank))
        w = W.TINY_FP32
        x = W.prefill_inputs(w, seed=bench.rank_seed(1000, rank), device="cpu")
        out_q.put((rank, ms, value, m2, float(x["q"].double().sum()), tuple(x["q"].shape)))
        d.barrier()
    finally:
        d.close()


def test_weak_scaling_aggregation_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, ms0, v0, m20, s0, sh0), (r1, ms1, v1, m21, s1, sh1) = res
    assert ms0 == ms1 == 12.0  # max over ranks, identical everywhere
    assert v0 == v1 == pytest.approx(2 * 4 * 8192 / 0.012)  # whole-job units / slowest time
    assert m20 == m21 == 1.0
    assert sh0 == sh1  # same shapes ...
    assert s0 != s1  # ... different sequences on each rank


def test_single_rank_dist_is_local():
    sys.path.insert(0, ROOT)
    import bench

    os.environ.pop("WORLD_SIZE", None)
    d = bench.Dist(1)
    assert d.world == 1 and d.pg is None
    ms, value = bench.weak_scaling_value(d, 5.0, 1000)
    assert ms == 5.0 and value == pytest.approx(1000 / 0.005)
    d.barrier()
    d.close()


def test_reference_arm_under_torchrun_rank0_only():
    """`bench.py --impl reference` launched by torchrun with two ranks: rank 0 alone runs the oracle
    sample and prints one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
