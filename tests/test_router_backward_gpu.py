"""Router backward through the C ABI against the fp64 oracle.

moe_router_backward gives dlogits [T, E]: the gradient into the router logits
through the softmax over the k picked logits (zero for experts not picked).
Checked three ways: against the oracle's own forward (end to end, bf16 tolerance),
against the oracle fed the GPU's expert outputs (the kernel's arithmetic alone,
fp32-accumulation tolerance), and at full size on sampled tokens.
"""
import numpy as np
import pytest
import torch

import mixture_experts_lora_b200 as ml
import oracle.moe_lora_oracle as O
from moe_inputs import CONFIGS, small_config

from gpu_common import TOL, ensure_built, inputs_on, oracle_full, rel_err, run_layer, to_np

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4   # fp32 accumulation of bf16 products over m, relative to the row scale


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _dlogits(inp, buf, cfg):
    dl = torch.full((cfg.T, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    ml.moe_router_backward(inp["dY"], buf.Y_sorted, buf.ids, buf.w, buf.pair_pos, cfg.E, dl)
    torch.cuda.synchronize()
    assert ml.moe_get_device_error() == ml.MOE_OK
    return dl


def _check_structure(dl, ids):
    dl = dl.cpu().numpy()
    mask = np.zeros_like(dl, dtype=bool)
    np.put_along_axis(mask, ids, True, axis=1)
    assert np.all(dl[~mask] == 0.0), "experts not picked get exactly zero"
    assert np.all(np.isfinite(dl)), "every entry written"
    scale = max(np.max(np.abs(dl)), 1e-30)
    assert np.max(np.abs(dl.sum(axis=1))) <= 1e-5 * scale   # softmax Jacobian rows sum to 0


@pytest.mark.parametrize("cfg", [CONFIGS["tiny"],
                                 small_config(T=70, m=64, n=32, E=8, k=8, r=8, alpha=8),
                                 small_config(T=33, m=144, n=80, E=5, k=3, r=16, alpha=16)],
                         ids=["tiny", "k_equals_E", "ragged"])
def test_router_backward_matches_oracle(cfg):
    inp, cpu = inputs_on(cfg)
    buf = run_layer(inp, cfg)
    dl = _dlogits(inp, buf, cfg)
    Y, aux, g = oracle_full(cpu, cfg)
    ref, _ = O.router_backward(cpu["dY"], aux["yp"], aux["ids"], aux["w"], aux["pair_pos"], cfg.E)
    assert rel_err(to_np(dl), ref) <= TOL
    # the kernel's arithmetic alone: the oracle fed the GPU's expert outputs and weights
    ref2, _ = O.router_backward(cpu["dY"], to_np(buf.Y_sorted), aux["ids"], to_np(buf.w),
                                aux["pair_pos"], cfg.E)
    assert rel_err(to_np(dl), ref2) <= TOL_F32
    _check_structure(dl, aux["ids"])


def test_router_backward_k32_synthetic():
    """k = 32 (the widest supported), m = 8 (one 16-byte piece), random expert outputs."""
    T, E, k, m = 45, 40, 32, 8
    g = torch.Generator().manual_seed(11)
    logits = torch.randn(T, E, generator=g)
    ids, w = O.route_topk(logits.numpy(), k)
    _, _, sp, pos = O.permute(ids, E)
    ys = torch.randn(T * k, m, generator=g).to(torch.bfloat16)
    dY = torch.randn(T, m, generator=g).to(torch.bfloat16)
    dl = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    ml.moe_router_backward(dY.cuda(), ys.cuda(), torch.from_numpy(ids.astype(np.int32)).cuda(),
                           torch.from_numpy(w.astype(np.float32)).cuda(),
                           torch.from_numpy(pos.astype(np.int32)).cuda(), E, dl)
    torch.cuda.synchronize()
    ref, _ = O.router_backward(dY, ys, ids, w.astype(np.float32).astype(np.float64), pos, E)
    assert rel_err(to_np(dl), ref) <= TOL_F32
    _check_structure(dl, ids)


def test_router_backward_full_size_sampled():
    cfg = CONFIGS["qwen3_30b_a3b"]
    inp, cpu = inputs_on(cfg)
    buf = run_layer(inp, cfg)
    dl = to_np(_dlogits(inp, buf, cfg))
    rng = np.random.default_rng(0)
    toks = rng.choice(cfg.T, size=64, replace=False)
    ids = buf.ids.cpu().numpy()[toks]
    w = to_np(buf.w)[toks]
    pos = buf.pair_pos.cpu().numpy().reshape(cfg.T, cfg.k)[toks]
    ys = to_np(buf.Y_sorted)
    dY = O.to64(cpu["dY"])[toks]
    dw = np.stack([np.sum(dY * ys[pos[:, j]], axis=1) for j in range(cfg.k)], axis=1)
    ref = np.zeros((len(toks), cfg.E))
    np.put_along_axis(ref, ids, w * (dw - np.sum(w * dw, axis=1, keepdims=True)), axis=1)
    assert rel_err(dl[toks], ref) <= TOL_F32
