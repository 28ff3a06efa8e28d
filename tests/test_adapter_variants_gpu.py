"""Adapter variants through the C ABI against the fp64 oracle.

- Separate gate and up adapters (rank r each), run as the fused rank-2r adapter
  A = [A_g | A_u], B = blockdiag(B_g, B_u) with the down adapter zero-padded, held by
  SplitGateUpAdapters; compared with the oracle's layer with separate adapters.
- rsLoRA: the scale alpha / sqrt(r) instead of alpha / r is the scale argument.
"""
import math

import numpy as np
import pytest
import torch

import mixture_experts_lora_b200 as ml
import oracle.moe_lora_oracle as O
from moe_inputs import LayerConfig, small_config

from gpu_common import TOL, check_full_parity, ensure_built, inputs_on, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


@pytest.mark.parametrize("cfg", [small_config(T=180, m=128, n=64, E=6, k=2, r=8, alpha=16),
                                 small_config(T=150, m=256, n=128, E=8, k=2, r=16, alpha=32)],
                         ids=["r8", "r16"])
def test_separate_gate_up_adapters(cfg):
    inp, cpu = inputs_on(cfg, seed=3)
    g = torch.Generator().manual_seed(9)
    E, m, n, r = cfg.E, cfg.m, cfg.n, cfg.r
    ad = ml.SplitGateUpAdapters(E, m, n, r)
    vals = {"A_g": torch.randn(E, m, r, generator=g) / math.sqrt(m),
            "A_u": torch.randn(E, m, r, generator=g) / math.sqrt(m),
            "B_g": torch.randn(E, r, n, generator=g) * 0.05,
            "B_u": torch.randn(E, r, n, generator=g) * 0.05,
            "A_d": cpu["A_d"].float(), "B_d": cpu["B_d"].float()}
    for name, v in vals.items():
        getattr(ad, name).copy_(v.to(torch.bfloat16))
    buf = ml.alloc_buffers(cfg.T, m, n, E, cfg.k, 2 * r, cfg.scale)
    ml.layer_step(ad.layer_inputs(inp), cfg.k, cfg.scale, buf)
    assert ml.moe_get_device_error() == ml.MOE_OK
    ref_inp = dict(cpu)
    for name in vals:
        ref_inp[name] = getattr(ad, name).cpu()
    Y, grads = O.layer_split_gate_up(ref_inp, cfg.k, cfg.scale)
    errs = {"Y": rel_err(to_np(buf.Y), Y), "dX": rel_err(to_np(buf.dX), grads["dX"])}
    for name, view in ad.grads(buf).items():
        errs[name] = rel_err(to_np(view), grads[name])
    assert max(errs.values()) <= TOL, errs
    # the down adapter's padding gets exactly zero gradient
    assert not torch.any(buf.dA_d[:, :, r:] != 0) and not torch.any(buf.dB_d[:, r:, :] != 0)


def test_rslora_scale():
    # rsLoRA scales by alpha / sqrt(r): r = 16, alpha = 16 gives c = 4, the same c as
    # the usual alpha / r with alpha = 64
    r, alpha = 16, 16
    c = alpha / math.sqrt(r)
    cfg = LayerConfig("rslora", T=200, m=128, n=96, E=8, k=2, r=r, alpha=c * r)
    assert cfg.scale == c
    inp, cpu = inputs_on(cfg, seed=6)
    buf = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r, c)
    ml.layer_step(inp, cfg.k, c, buf)
    assert ml.moe_get_device_error() == ml.MOE_OK
    check_full_parity(buf, cpu, cfg)
