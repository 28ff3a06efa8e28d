"""Data-parallel plumbing for the layer (one process per GPU).

Tokens are independent, so data parallelism shards the batch: every rank runs the
whole layer on its own tokens against the same expert weights and adapters, and
the only exchange is one sum of the adapter gradients dA_gu, dB_gu, dA_d, dB_d
across ranks (E * r * (2m + 3n) elements; 26 MB in bf16 for the Qwen3-30B-A3B
shape), done with torch.distributed (NCCL over NVLink on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from moe_inputs import LayerConfig, generate, generate_tokens

WEIGHT_SEED = 0
TOKEN_SEED_BASE = 1000


def rank_inputs(cfg: LayerConfig, rank: int, device="cpu") -> dict:
    """Inputs of one rank: the shared weights (seed 0) and, for rank > 0, its own
    tokens (logits, X, dY) from a rank-specific generator.  Rank 0 keeps the
    seed-0 tokens, so a one-rank run sees exactly the single-GPU workload."""
    inp = generate(cfg, seed=WEIGHT_SEED, device=str(device))
    if rank > 0:
        inp.update(generate_tokens(cfg, seed=TOKEN_SEED_BASE + rank, device=str(device)))
    return inp


def allreduce_adapter_grads(grads, group=None) -> None:
    """Sum the adapter gradients over the ranks of `group`, in place."""
    if not dist.is_available() or not dist.is_initialized():
        return
    if dist.get_world_size(group) == 1:
        return
    for g in grads:
        dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
