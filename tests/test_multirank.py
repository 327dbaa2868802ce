"""The multi-GPU path of bench.py on CPU: two gloo ranks (world size 2).

The path shards into independent problems (one seeded batch per rank), so the
only collectives are the barrier and the max over ranks of the timings; these
tests run exactly that host logic with gloo instead of NCCL.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from polar_attention_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        cpu = torch.device("cpu")
        t = 1.0 + 0.5 * r                      # per-rank "elapsed seconds"
        bench.barrier(w, cpu)
        m = bench.max_over_ranks(t, w, cpu)
        seed = bench.rank_seed(0, r)
        x = W.prefill_inputs(W.small_prefill(B=1, T=64, Hq=4, Hkv=2, dtype="bf16"), "cpu", seed=seed)
        xg = W.gdelta_inputs(W.small_gdelta(B=1, T=64, H=2), "cpu", seed=seed + 2)
        q.put((r, w, local, seed, m, bench.aggregate_throughput(10.0, w, m),
               float(x["q"].float().sum()), float(xg["k"].float().sum() + xg["alpha"].sum())))
        bench.barrier(w, cpu)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, s0, m0, v0, q0, g0), (r1, w1, l1, s1, m1, v1, q1, g1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == 2 and (l0, l1) == (0, 1)
    assert s0 != s1, "each rank must draw its own batch"
    assert q0 != q1, "the two ranks' inputs must differ"
    assert g0 != g1, "the two ranks' memory-channel inputs must differ"
    assert m0 == m1 == 1.5, "every rank sees the slowest rank's time"
    assert v0 == v1 == pytest.approx(10.0 * 2 / 1.5), "whole-job work over the max time"


def test_reference_arm_only_rank0_reports(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1"])) is None
