"""The multi-rank host path with world size 2 on gloo (CPU, no GPU).

The op partitions over 128-aligned token ranges with no exchange: each rank's
result on its shard must equal the global result restricted to that shard.
The oracle stands in for the kernel here (the host logic is what is tested);
the only collective, the max-over-ranks of a timing, runs on gloo."""
from __future__ import annotations

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, M: int, K: int) -> None:
    import oracle
    import workloads as W
    from swiglu_backward_int8_b200 import parallel
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = W.small_workload(M, K, seed=11)
        x, gy = W.make_inputs(w)
        m0, m1 = parallel.shard_rows(M, world, rank)
        i0, i1 = parallel.group_range(m0, m1)
        full = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
        mine = oracle.silu_dot_fwd_bwd_quant_fuse(x[m0:m1], gy[m0:m1])
        ok = (np.array_equal(mine[0], full[0][m0:m1]) and np.array_equal(mine[1], full[1][m0:m1])
              and np.array_equal(mine[2], full[2][:, m0:m1]) and np.array_equal(mine[3], full[3][:, i0:i1]))
        # the same with grad_y handed over as INT8 codes + scales (their rows shard with the tokens)
        q, sc = W.quantized_grad_y(w)
        qfull = oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(x, q, sc)
        qmine = oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(x[m0:m1], q[m0:m1], sc[m0:m1])
        ok = ok and (np.array_equal(qmine[0], qfull[0][m0:m1]) and np.array_equal(qmine[1], qfull[1][m0:m1])
                     and np.array_equal(qmine[2], qfull[2][:, m0:m1])
                     and np.array_equal(qmine[3], qfull[3][:, i0:i1]))
        flag = torch.tensor([1 if ok else 0], dtype=torch.int32)
        dist.all_reduce(flag, op=dist.ReduceOp.MIN)
        assert flag.item() == 1, f"rank {rank}: shard result differs from the global result"
        # shard sizes add up to M with no overlap
        sizes = torch.tensor([m1 - m0], dtype=torch.int64)
        dist.all_reduce(sizes)
        assert sizes.item() == M
        # the slowest rank's time and the whole-job throughput
        worst = parallel.max_over_ranks(10.0 + rank)
        assert worst == 10.0 + world - 1
        assert parallel.aggregate_gbs(1_000_000, world, worst) == pytest.approx(world * 1e6 / (worst * 1e-3) / 1e9)
        parallel.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,K", [(300, 256), (1000, 128)])
def test_two_ranks_shards_equal_global_result(M, K):
    mp.spawn(_worker, args=(2, _free_port(), M, K), nprocs=2, join=True)


def test_shard_rows_cover_and_align():
    from swiglu_backward_int8_b200 import parallel
    for M in (1, 127, 128, 129, 300, 4000, 16384):
        for world in (1, 2, 3, 8):
            prev = 0
            for r in range(world):
                m0, m1 = parallel.shard_rows(M, world, r)
                assert m0 == prev and m1 >= m0 and (m0 % 128 == 0 or m0 == m1 == M)
                prev = m1
            assert prev == M
    with pytest.raises(ValueError):
        parallel.shard_rows(100, 2, 2)
