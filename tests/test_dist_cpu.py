"""bench.py's multi-process path on CPU: two ranks over gloo (no GPU).

One process per GPU is the deployment; every (sequence, v-head) chain is
independent, so the ranks run replicas on their own sequences with no
data-path collective.  What the ranks share is the timing plumbing: the
process group, the barriers around the timed region, the max over ranks of
the device time, and the whole-job throughput computed from it.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import types

    import torch.distributed as dist

    import bench
    import workloads as W
    try:
        w_, r_, l_ = bench.dist_setup(types.SimpleNamespace(impl="ours"), backend="gloo")
        assert (w_, r_, l_) == (world, rank, rank) and dist.is_initialized()
        bench.barrier(world)
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")  # rank 1 is the slower one
        value = bench.job_throughput(1000, world, 4, slowest)
        # weak scaling: each rank draws its own sequences (seed 2 + rank, as bench.py does)
        w = W.make_prefill(num_seqs=2, seq_len=64, nqk=1, nv=2, d=64, io="bf16", seed=2 + rank)
        bench.barrier(world)
        q.put((rank, slowest, value, float(w["q"].float().sum())))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_ranks_over_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, m0, v0, s0), (_, m1, v1, s1) = res
    assert m0 == m1 == 15.0                      # both ranks see the slowest rank's time
    assert v0 == v1 == 1000 * 2 * 4 / 0.015      # all ranks' units over that time
    assert s0 != s1                              # the replicas work on different sequences


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import types

    import bench
    args = types.SimpleNamespace(impl="reference", warmup=3, steps=1, ref_sample_tokens=8)
    assert bench.run_reference(args, 2, 1) is None
