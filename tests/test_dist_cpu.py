"""Host side of the N > 1 path, as two gloo ranks on CPU (no GPU).

bench.py runs one replica per GPU: each rank times its own batch, the job's time
is the max over ranks and its value the operations of all ranks over that time.
These tests drive the same helpers through a real two-process group, and check
the one exchange a token-sharded batch would need: an all-reduce MAX of the
runtime group maxima s, which must equal the single-process s bit for bit
because max is exact (the method computes s over all tokens of the batch at
inference: Rotated Runtime Smooth summary page, "Approach").
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from activation_smoothing_b200 import workloads as wl

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # max over ranks and the whole-job value
        my_ms = 10.0 + 7.5 * rank
        ms = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        assert ms == 10.0 + 7.5 * (world - 1)
        ops = 2 * 2048 * 4096 * 4096
        assert bench.whole_job_tops(ops, 100, world, ms) == pytest.approx(ops * 100 * world / (ms * 1e-3) / 1e12)

        # replicas draw distinct batches
        mine = torch.tensor([bench.activation_sample(i, rank) for i in range(bench.N_XSETS)])
        gathered = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)
        seen = torch.cat(gathered).tolist()
        assert len(set(seen)) == len(seen)

        # token-sharded batch: s from each shard, all-reduce MAX == s of the whole batch
        L = wl.LAYERS["tiny"]
        X = wl.make_activations(L, M=32)
        perm = wl.random_perm(L.K, 4).numpy()
        rows = np.array_split(np.arange(X.shape[0]), world)[rank]
        Xp = oracle.reorder(oracle.rotate(X[torch.from_numpy(rows)], L.had_block), perm)
        s_local = torch.from_numpy(oracle.group_max(Xp, L.G).copy())
        dist.all_reduce(s_local, op=dist.ReduceOp.MAX)
        s_full = oracle.group_max(oracle.reorder(oracle.rotate(X, L.had_block), perm), L.G)
        assert np.array_equal(s_local.numpy().view(np.uint32), np.asarray(s_full, np.float32).view(np.uint32))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_timing_value_and_sharded_group_max():
    mp.spawn(_rank_main, args=(WORLD, _free_port()), nprocs=WORLD, join=True)


def test_single_process_helpers():
    assert bench.max_over_ranks(3.25, None, torch.device("cpu")) == 3.25
    assert bench.whole_job_tops(10 ** 12, 1, 1, 1000.0) == pytest.approx(1.0)
