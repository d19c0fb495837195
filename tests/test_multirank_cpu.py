"""The N > 1 host logic of bench.py on world_size-2 gloo ranks (CPU only).

Each rank attends its own independent decode batch (no data-path collective);
ranks meet only in the MAX reduction of the elapsed time, and the reported
throughput counts every rank's bytes over the slowest rank's time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads

        case = workloads.decode_batch(num_seqs=4, lo=16, hi=64, seed=bench.shard_seed(rank),
                                      num_q_heads=4, num_kv_heads=2, head_dim=64)
        elapsed = 10.0 + 5.0 * rank                      # the slower rank sets the time
        mx = bench.max_over_ranks(elapsed, world, "cpu")
        bytes_step = bench.scatter_bytes(case) + bench.attention_bytes(case)
        total = torch.tensor([bytes_step], dtype=torch.float64)
        dist.all_reduce(total)                           # only to check the test's own sum
        results[rank] = {
            "max_ms": mx,
            "value": bench.whole_job_gbs(bytes_step, 7, world, mx),
            "lens": case.seq_lens.tolist(),
            "bytes": bytes_step,
            "sum_bytes": float(total.item()),
        }
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_the_max():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    r0, r1 = results[0], results[1]
    assert r0["max_ms"] == r1["max_ms"] == 15.0
    assert r0["lens"] != r1["lens"]                      # independent batches per rank
    # every rank reports bytes_per_step * steps * world / max time
    assert r0["value"] == pytest.approx(r0["bytes"] * 7 * 2 / 15e-3 / 1e9)


def test_reference_arm_prints_on_rank_zero_only():
    import argparse

    import bench

    args = argparse.Namespace(steps=1, warmup=0)
    assert bench.run_reference(args, rank=1, world=2) is None
