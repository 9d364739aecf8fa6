"""Host-side logic of the multi-GPU path (replicas / weak scaling), on CPU with gloo.

Every rank owns its own sequences (rank-specific seed), there is no data-path
collective, the step time is the max over ranks, and the whole-job throughput
counts every rank's tokens.  The reference arm runs on rank 0 only.
"""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_10_b200 import configs, synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(configs.TINY, rank)
        q_, qi, _ = synth.queries(w, [0])
        first = synth.kv_tokens(w, synth.TID_IK, 0, 1, w.DI, 0, 4)
        t = bench.max_over_ranks(1.0 + rank)  # rank r "took" 1 + r ms
        # gather what each rank saw, for the parent to check
        out = [None] * world
        dist.all_gather_object(out, (w.seed, float(qi.float().sum()), float(first.sum()), t))
        if rank == 0:
            q.put(out)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_own_sequences_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    res = q.get()
    (s0, a0, b0, t0), (s1, a1, b1, t1) = res
    assert s0 != s1 and a0 != a1 and b0 != b1  # different sequences per rank
    assert t0 == t1 == 2.0                     # both ranks report the slowest time
    import bench
    assert bench.aggregate_throughput(32, 2, 1e-3) == 64000.0


def test_max_over_ranks_without_process_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
