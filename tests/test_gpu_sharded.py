"""Token-sharded activation path on the CUDA kernels (needs a GPU).

One batch is split by tokens; each shard runs pass A (rrs_group_max), the
shards' group maxima are combined with an elementwise MAX, and each shard runs
pass B (rrs_smooth_quant_scaled) with the combined scales.  The runtime scale
of a group is the maximum over all tokens of the batch (Rotated Runtime Smooth
summary page, "Approach") and a maximum of maxima is exact, so the result must
be bit-identical to one rrs_smooth_quant over the whole batch, and to the
oracle.  The combine runs on the device, and across two processes with a gloo
all-reduce (MAX) of host copies, as a multi-GPU job would do it over NCCL.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from activation_smoothing_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module")
def rrs():
    import activation_smoothing_b200 as m
    m.lib()
    return m


def _bits(t):
    return t.detach().cpu().numpy().view(np.uint8)


def _same(a, b):
    a = a.detach().cpu().numpy() if isinstance(a, torch.Tensor) else np.asarray(a)
    b = b.detach().cpu().numpy() if isinstance(b, torch.Tensor) else np.asarray(b)
    return a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8))


CASES = [("tiny", 16, (5, 11), 0), ("llama3_8b_qo", 256, (100, 156), 0), ("llama3_8b_qo", 256, (1, 255), 1),
         ("llama3_8b_down", 96, (40, 56), 0), ("llama3_70b_qo", 64, (17, 30, 17), 0)]


@pytest.mark.parametrize("name,M,split,flags", CASES)
def test_sharded_passes_equal_one_call_and_oracle(rrs, name, M, split, flags):
    L = wl.LAYERS[name]
    X = wl.make_activations(L, M=M)
    perm = wl.random_perm(L.K, 6)
    Xd, pd = X.to(DEV), perm.to(DEV)
    qX1, s1, st1 = rrs.smooth_quant(Xd, pd, L.G, L.had_block, flags)
    shards = torch.split(Xd, list(split))
    s_parts = [rrs.group_max(x, pd, L.G, L.had_block, flags) for x in shards]
    s = s_parts[0].clone()
    for sp in s_parts[1:]:
        s = torch.maximum(s, sp)
    outs = [rrs.smooth_quant_scaled(x, pd, s, L.G, L.had_block, flags) for x in shards]
    torch.cuda.synchronize()
    qX = torch.cat([o[0] for o in outs])
    st = torch.cat([o[1] for o in outs])
    assert _same(s, s1), "s (MAX over shards) vs one call"
    assert _same(qX, qX1) and _same(st, st1), "codes/scales (sharded) vs one call"
    n_eff = 1 if flags & rrs.NO_ROTATE else L.had_block
    _, oqX, os_, ost = oracle.smooth_quant(X, L.G, n_eff, perm.numpy())
    assert _same(s, os_) and _same(qX, oqX) and _same(st, ost), "sharded path vs oracle"


def test_pass_a_under_unit_scales_writes_ones(rrs):
    L = wl.LAYERS["llama3_8b_kv"]
    X = wl.make_activations(L, M=8).to(DEV)
    s = rrs.group_max(X, wl.identity_perm(L.K).to(DEV), L.G, L.had_block, rrs.FORCE_UNIT_SCALES)
    torch.cuda.synchronize()
    assert torch.all(s == 1.0)


def _free_port() -> int:
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _rank_main(rank, world, port, path):
    import torch.distributed as dist
    import activation_smoothing_b200 as rrs_m
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = wl.LAYERS["llama3_8b_qo"]
        X = wl.make_activations(L, M=192)
        perm = wl.random_perm(L.K, 9)
        rows = np.array_split(np.arange(X.shape[0]), world)[rank]
        Xd = X[torch.from_numpy(rows)].contiguous().to(DEV)
        pd = perm.to(DEV)
        s = rrs_m.group_max(Xd, pd, L.G, L.had_block)
        sh = s.cpu()
        dist.all_reduce(sh, op=dist.ReduceOp.MAX)        # the one exchange of the sharded path
        qX, st = rrs_m.smooth_quant_scaled(Xd, pd, sh.to(DEV), L.G, L.had_block)
        torch.cuda.synchronize()
        np.savez(os.path.join(path, f"rank{rank}.npz"), s=sh.numpy(), qX=qX.cpu().numpy(), st=st.cpu().numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_processes_all_reduce_max_of_s(rrs, tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    parts = [np.load(os.path.join(tmp_path, f"rank{r}.npz")) for r in range(world)]
    L = wl.LAYERS["llama3_8b_qo"]
    X = wl.make_activations(L, M=192)
    perm = wl.random_perm(L.K, 9)
    _, oqX, os_, ost = oracle.smooth_quant(X, L.G, L.had_block, perm.numpy())
    for p in parts:
        assert np.array_equal(p["s"].view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(np.concatenate([p["qX"] for p in parts]), oqX)
    assert np.array_equal(np.concatenate([p["st"] for p in parts]).view(np.uint32), ost.view(np.uint32))
