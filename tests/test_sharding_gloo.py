"""The multi-rank path on CPU: two gloo ranks each verify their block of
rows (oracle as the per-rank engine, rows keyed by their global id through
row_base), gather, and reproduce the single-process result; the timing
reduction takes the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verification_93_b200.sharding import max_over_ranks, shard_rows


def test_shard_rows_partition():
    for total in (1, 7, 256, 1025):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from speculative_decoding_verification_93_b200 import workloads
        from speculative_decoding_verification_93_b200.workloads import to_host_logits
        b = workloads.random_small(24, 4, 300, dtype=torch.bfloat16, seed=5,
                                   temps=(0.0, 0.6, 1.0))
        s0, s1 = shard_rows(24, world, rank)
        out, acc, _, st = oracle.verify(to_host_logits(b.zt[s0:s1]), to_host_logits(b.zd[s0:s1]),
                                        b.tokens[s0:s1].numpy(), b.lengths[s0:s1].numpy(),
                                        b.temperature[s0:s1].numpy(), seed=77, row_base=s0,
                                        nthreads=1)
        parts = [None] * world
        dist.all_gather_object(parts, (s0, out, acc))
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            parts.sort(key=lambda p: p[0])
            full_out, full_acc, _, _ = oracle.verify(
                to_host_logits(b.zt), to_host_logits(b.zd), b.tokens.numpy(), b.lengths.numpy(),
                b.temperature.numpy(), seed=77, nthreads=1)
            ok = (np.array_equal(np.concatenate([p[1] for p in parts]), full_out)
                  and np.array_equal(np.concatenate([p[2] for p in parts]), full_acc)
                  and t == float(world))
            with open(result_path, "w") as f:
                f.write("ok" if ok else "mismatch")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_unsharded_batch(tmp_path):
    world = 2
    path = str(tmp_path / "result.txt")
    mp.start_processes(_worker, args=(world, _free_port(), path), nprocs=world, join=True,
                       start_method="spawn")
    assert open(path).read() == "ok"


def test_max_over_ranks_without_group():
    assert max_over_ranks(3.5) == 3.5
