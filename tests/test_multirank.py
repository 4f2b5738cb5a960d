"""Host logic of the multi-GPU bench path, run as two gloo ranks on the CPU.

The block-attention step shards by example with no exchange (each rank runs
its own seeded batch); the only collective is the final report, which sums
useful FLOPs and tokens over ranks and takes the slowest rank's time.
"""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        class Args:
            config, examples, swa, block, window = 2, 2, 0, 0, 0
        w, inp = bench.workload(Args(), rank)
        # per-rank numbers: rank r pretends to run 10 * (r + 1) GFLOP in 2 + r ms
        got = bench.job_totals(1e10 * (rank + 1), 100 * (rank + 1), 2.0 + rank, dist)
        results[rank] = (got, float(inp["q"].float().sum()), int(inp["q"].shape[0]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_batches_and_reduce_job_totals():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), results), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(results)
    (t0, s0, n0), (t1, s1, n1) = res[0], res[1]
    assert t0 == t1 == (3e10, 300.0, 3.0)    # FLOPs and tokens summed, time = max
    assert n0 == n1 > 0 and s0 != s1          # same shapes, different seeded data per rank


def test_bench_gpus_n_launches_ranks_and_prints_one_line():
    """bench.py --gpus 2 without torchrun starts two ranks itself
    (bench.spawn_ranks); with the GPU step replaced by a stand-in that runs on
    gloo ranks, exactly one JSON line comes back, from rank 0, with n_gpus 2,
    FLOPs and tokens summed over the ranks and the slowest rank's time."""
    import json
    import subprocess
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_kunlun_b200 import flops as F
    argv = ["--gpus", "2", "--config", "2", "--examples", "2", "--steps", "3", "--warmup", "1", "--no-e2e",
            "--no-cpu-baseline"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = bench.spawn_ranks(2, argv, script=os.path.join(ROOT, "tests", "multirank_stub.py"),
                          capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["steps"] == 3 and d["scaling"] == "weak"
    # per rank: 2 examples of 1024 tokens, H4 D64, block 128, window 2; rank r takes 2 + r ms per step
    pairs = F.visible_pairs([1024, 1024], 128, 2)
    step_flops = F.step_flops(pairs, 4, 64)["step"]
    assert abs(d["ms_per_step"] - 3.0) < 1e-9
    assert abs(d["value"] - 2 * step_flops / 3e-3 / 1e12) < 1e-6 * d["value"]
    assert abs(d["tokens_per_s"] - 2 * 2048 / 3e-3) < 1e-6 * d["tokens_per_s"]
    assert d["config"]["parallelism"].startswith("dp2")
