"""Multi-rank host logic of bench.py on CPU (gloo, world size 2; no GPU).

The forward shards over independent heads: each rank draws its own batch
(distinct seeds, so no two ranks duplicate work), times it, and the job time
is the max over ranks; the whole-job throughput counts every rank's tokens.
The only collective is that timing reduction.  Also checks that the
reference arm under several ranks runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    from kernelized_linear_attention_fwd_b200 import inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seed = bench.rank_seed(0, rank)
        q, _, _ = inputs.make_qkv(1, 2, 32, 16, 16, "bf16", seed=seed)
        my_ms = 10.0 + 5.0 * rank                    # rank 1 is the slow one
        ms_max = bench.max_over_ranks(my_ms, world, device="cpu")
        value = bench.job_throughput(world, 1000, ms_max)
        results[rank] = (seed, int(q.astype("int64").sum()), ms_max, value)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_distinct_heads_and_share_the_max_time():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    assert set(res) == {0, 1}
    (s0, sum0, m0, v0), (s1, sum1, m1, v1) = res[0], res[1]
    assert s0 != s1 and sum0 != sum1          # independent batches of heads
    assert m0 == m1 == 15.0                   # every rank sees the slowest time
    assert v0 == v1 == pytest.approx(2 * 1000 / 0.015)


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1, 131072, 1.0) == pytest.approx(131072 / 1e-3)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
