"""The N > 1 path of bench.py, on CPU with two gloo ranks.

Several GPUs run as replicas: every rank serves its own batch of independent
sequences (no collective on the data path), the job's step time is the
slowest rank's, and the job's throughput counts the queries of all ranks.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_of_rank, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    from compressed_sparse_attention_15_b200 import workloads as WL

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(ms_of_rank[rank], True, torch.device("cpu"))
        w = WL.shard(WL.WORKLOADS["csa_decode_64k"], rank)
        # a slice of this rank's inputs, gathered to compare across ranks
        q_head = WL.make(WL.small(w, Q=2, H=2, D=8), "q").float().flatten()
        got = [torch.empty_like(q_head) for _ in range(world)]
        dist.all_gather(got, q_head)
        results[rank] = (ms_max, bench.job_value(world, w.Q, ms_max), w.seed, [g.tolist() for g in got])
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_step_and_serve_distinct_batches():
    world, port = 2, _free_port()
    ms_of_rank = [0.75, 1.25]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, ms_of_rank, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    for r in range(world):
        ms_max, value, seed, gathered = res[r]
        assert ms_max == max(ms_of_rank)                       # every rank sees the slowest rank's time
        assert value == pytest.approx(world * 32 / 1.25e-3)    # 32 queries per rank per step
    assert res[0][2] != res[1][2]                              # each rank draws its own sequences
    g = res[0][3]
    assert g == res[1][3] and g[0] != g[1]


def test_shard_keeps_shapes_and_rank0_is_the_single_gpu_batch():
    from compressed_sparse_attention_15_b200 import workloads as WL

    w = WL.WORKLOADS["hca_decode_1m"]
    assert WL.shard(w, 0) == w
    s3 = WL.shard(w, 3)
    assert (s3.B, s3.Q, s3.N, s3.T_raw, s3.dtype) == (w.B, w.Q, w.N, w.T_raw, w.dtype)
    with pytest.raises(ValueError):
        WL.shard(w, -1)


def test_reference_arm_runs_on_rank0_only():
    # Under torchrun every rank starts bench.py --impl reference; ranks other
    # than 0 leave at once, without work and without output.
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
