"""Data-parallel host logic with two gloo ranks on CPU (no GPU needed)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from moe_inputs import small_config


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from mixture_experts_lora_b200 import dp
        cfg = small_config(T=16, m=32, n=16, E=4, k=2, r=8)
        inp = dp.rank_inputs(cfg, rank)
        grads = [torch.full((3, 4), float(rank + 1)), torch.arange(6, dtype=torch.float32) * (rank + 1)]
        dp.allreduce_adapter_grads(grads)
        q.put((rank, inp["W_gu"].float().sum().item(), inp["X"].float().sum().item(),
               grads[0].tolist(), grads[1].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_rank_shared_weights_own_tokens_and_grad_sum():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, wsum, xsum, g0, g1 = q.get(timeout=120)
        res[rank] = (wsum, xsum, g0, g1)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0]                 # same expert weights on every rank
    assert res[0][1] != res[1][1]                 # each rank its own tokens
    for r in range(world):
        assert res[r][2] == [[3.0] * 4] * 3       # 1 + 2
        assert res[r][3] == [3.0 * i for i in range(6)]


def test_single_rank_is_the_single_gpu_workload():
    from mixture_experts_lora_b200 import dp
    from moe_inputs import generate
    cfg = small_config(T=8, m=32, n=16, E=4, k=2, r=8)
    a, b = dp.rank_inputs(cfg, 0), generate(cfg, seed=0)
    assert all(torch.equal(a[k], b[k]) for k in a)
    dp.allreduce_adapter_grads([torch.ones(2)])    # no process group: a no-op
