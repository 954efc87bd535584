"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

The fused sconv step shards by request with no exchange, so N GPUs run N
independent batches; the only cross-rank operations are the timing
barrier, the maximum of the elapsed times and the sum of the token counts.
"""
from __future__ import annotations

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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads
        bench.barrier(world)
        t_max = bench.max_over_ranks(1.0 + rank, world)        # elapsed seconds per rank
        n_sum = bench.sum_over_ranks(256.0 * (rank + 1), world)  # tokens per rank
        wl = workloads.decode_bf16(seed=bench.rank_seed(1002, rank))
        digest = torch.tensor([float(wl.positions.sum()), float(wl.block_table[:, 0].sum())],
                              dtype=torch.float64)
        all_d = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(all_d, digest)
        q.put((rank, t_max, n_sum, [d.tolist() for d in all_d]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_reduce_time_and_tokens():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(world, _free_port(), q), nprocs=world, join=True,
                       start_method="spawn")
    results = sorted(q.get() for _ in range(world))
    for rank, t_max, n_sum, digests in results:
        assert t_max == 2.0            # the slowest rank's time
        assert n_sum == 256.0 * 3      # whole-job tokens
        assert digests[0] != digests[1]  # each rank decodes its own requests
