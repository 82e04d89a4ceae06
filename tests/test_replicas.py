"""The N > 1 host path on the CPU: two gloo ranks run the replica plumbing the
benchmark uses on GPUs (rank environment, per-replica seeds, barriers, the max
over ranks of a timed region, whole-job throughput, rank-0-only reporting),
plus the reference arm under a multi-rank environment."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

from linear_rnn_mlstm_b200 import replicas
from linear_rnn_mlstm_b200 import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    env = {"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
           "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)}
    os.environ.update(env)
    e = replicas.rank_env()
    replicas.init(e, "gloo", timeout_s=60)
    try:
        replicas.barrier(e)
        # each rank "measured" a different duration; all must agree on the slowest
        slowest = replicas.max_over_ranks(10.0 + 5.0 * rank, e)
        # each replica draws its own shard of heads
        w = syn.custom("r", 1, 2, 8, 16, syn.SMALL, dtype="f32")
        q = syn.fwd_inputs(w, seed=replicas.replica_seed(w.seed, rank))["q"]
        gathered = [torch.zeros_like(q) for _ in range(world)]
        torch.distributed.all_gather(gathered, q)
        distinct = not torch.equal(gathered[0], gathered[1])
        out[rank] = (slowest, replicas.job_throughput(100.0, e, slowest * 1e-3), e.reports, distinct)
        replicas.barrier(e)
    finally:
        replicas.shutdown(e)


def test_two_gloo_ranks_agree_on_the_slowest_replica():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        slowest, thr, reports, distinct = out[r]
        assert slowest == 15.0                       # max over ranks, seen by every rank
        assert thr == pytest.approx(100.0 * world / 15e-3)
        assert reports == (r == 0)                   # only rank 0 prints
        assert distinct                              # different synthetic shards per replica


def test_rank_env_defaults_and_validation():
    e = replicas.rank_env({})
    assert (e.world, e.rank, e.local_rank, e.distributed, e.reports) == (1, 0, 0, False, True)
    e = replicas.rank_env({"WORLD_SIZE": "4", "RANK": "3", "LOCAL_RANK": "3"})
    assert e.distributed and not e.reports
    with pytest.raises(ValueError):
        replicas.rank_env({"WORLD_SIZE": "2", "RANK": "2"})
    # one process: no collective is needed for the max or the barrier
    assert replicas.max_over_ranks(3.5, replicas.rank_env({})) == 3.5
    replicas.barrier(replicas.rank_env({}))


def test_reference_arm_on_a_non_zero_rank_exits_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
