"""Seeded synthetic inputs for the MoE expert-MLP + Split-LoRA layer.

This module is shared by the fp64 oracle tests, the CUDA parity tests and the
benchmark.  It only draws random numbers and rounds them to the storage
precision; it holds none of the layer's arithmetic.

Shapes follow the model families the pages benchmark (Qwen3-30B-A3B,
gpt-oss-20b, DeepSeek-V3 / GLM): the real checkpoints and datasets are not
used, only their layer shapes.

Recipe (one generator, fixed draw order, every tensor rounded once):
  logits  fp32 [T, E]     ~ N(0, 1)  (+ Zipf bias for the skewed workload)
  X       bf16 [T, m]     ~ N(0, 1)
  W_gu    bf16 [E, m, 2n] ~ N(0, std 0.02)   gate columns [0, n), up [n, 2n)
  W_d     bf16 [E, n, m]  ~ N(0, std 0.02)
  A_gu    bf16 [E, m, r]  ~ N(0, var 1/m)
  B_gu    bf16 [E, r, 2n] ~ N(0, std 0.02)
  A_d     bf16 [E, n, r]  ~ N(0, var 1/n)
  B_d     bf16 [E, r, m]  ~ N(0, std 0.02)
  dY      bf16 [T, m]     ~ N(0, 1)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int          # tokens
    m: int          # hidden size
    n: int          # expert intermediate size
    E: int          # experts
    k: int          # experts per token
    r: int          # LoRA rank
    alpha: float    # LoRA alpha; scale c = alpha / r
    zipf_s: float = 0.0      # > 0: add bias_scale * log(Zipf rank weight) to logits
    bias_scale: float = 0.0

    @property
    def scale(self) -> float:
        return self.alpha / self.r

    @property
    def P(self) -> int:
        return self.T * self.k

    def as_dict(self) -> dict:
        d = asdict(self)
        d["scale"] = self.scale
        return d


CONFIGS = {
    "tiny": LayerConfig("tiny", T=256, m=128, n=64, E=8, k=2, r=8, alpha=16),
    "qwen3_30b_a3b": LayerConfig("qwen3_30b_a3b", T=4096, m=2048, n=768, E=128, k=8, r=16, alpha=16),
    "gpt_oss_20b": LayerConfig("gpt_oss_20b", T=8192, m=2880, n=2880, E=32, k=4, r=16, alpha=32),
    "qwen3_skewed": LayerConfig("qwen3_skewed", T=16384, m=2048, n=768, E=128, k=8, r=16, alpha=16,
                                zipf_s=1.2, bias_scale=3.0),
    "deepseek_v3": LayerConfig("deepseek_v3", T=32768, m=7168, n=2048, E=256, k=8, r=32, alpha=32),
    # the DeepSeek-V3 expert geometry (m, n, about 1024 rows per expert) on 16 experts:
    # a tensor-bound case small enough for a full ncu capture (about 2.5 GB on the device)
    "deepseek_v3_e16": LayerConfig("deepseek_v3_e16", T=2048, m=7168, n=2048, E=16, k=8, r=32, alpha=32),
}

DRAW_ORDER = ("logits", "X", "W_gu", "W_d", "A_gu", "B_gu", "A_d", "B_d", "dY")


def zipf_logit_bias(E: int, s: float, bias_scale: float) -> torch.Tensor:
    """Per-expert logit bias bias_scale * log(w_e), w_e = (e+1)^-s / H_{E,s}."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    w = ranks.pow(-s)
    w = w / w.sum()
    return (bias_scale * torch.log(w)).to(torch.float32)


def _normal(gen, shape, std, device):
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32) * std


def generate(cfg: LayerConfig | str, seed: int = 0, device: str = "cpu",
             with_dy: bool = True) -> dict:
    """Draw every input of one layer step with a single seeded generator.

    Returns a dict of tensors on `device`: logits fp32, the rest bf16.
    """
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, m, n, E, r = cfg.T, cfg.m, cfg.n, cfg.E, cfg.r
    out = {}
    logits = _normal(gen, (T, E), 1.0, device)
    if cfg.zipf_s > 0:
        logits = logits + zipf_logit_bias(E, cfg.zipf_s, cfg.bias_scale).to(device)
    out["logits"] = logits.contiguous()
    out["X"] = _normal(gen, (T, m), 1.0, device).to(torch.bfloat16)
    out["W_gu"] = _normal(gen, (E, m, 2 * n), 0.02, device).to(torch.bfloat16)
    out["W_d"] = _normal(gen, (E, n, m), 0.02, device).to(torch.bfloat16)
    out["A_gu"] = _normal(gen, (E, m, r), 1.0 / math.sqrt(m), device).to(torch.bfloat16)
    out["B_gu"] = _normal(gen, (E, r, 2 * n), 0.02, device).to(torch.bfloat16)
    out["A_d"] = _normal(gen, (E, n, r), 1.0 / math.sqrt(n), device).to(torch.bfloat16)
    out["B_d"] = _normal(gen, (E, r, m), 0.02, device).to(torch.bfloat16)
    if with_dy:
        out["dY"] = _normal(gen, (T, m), 1.0, device).to(torch.bfloat16)
    return out


def small_config(T=64, m=64, n=32, E=4, k=2, r=8, alpha=16.0, name="custom") -> LayerConfig:
    """A free-form small configuration (oracle pins, edge cases)."""
    return LayerConfig(name, T=T, m=m, n=n, E=E, k=k, r=r, alpha=alpha)


def generate_tokens(cfg: LayerConfig | str, seed: int, device: str = "cpu") -> dict:
    """Per-token inputs only (logits, X, dY) from their own seeded generator, with
    the same distributions as generate(); used to give data-parallel ranks their
    own batch while the expert weights stay shared."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    logits = _normal(gen, (cfg.T, cfg.E), 1.0, device)
    if cfg.zipf_s > 0:
        logits = logits + zipf_logit_bias(cfg.E, cfg.zipf_s, cfg.bias_scale).to(device)
    return {"logits": logits.contiguous(),
            "X": _normal(gen, (cfg.T, cfg.m), 1.0, device).to(torch.bfloat16),
            "dY": _normal(gen, (cfg.T, cfg.m), 1.0, device).to(torch.bfloat16)}
