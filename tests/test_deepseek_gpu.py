"""Full-size sampled parity at the DeepSeek-V3/GLM-shaped layer: T=32768, m=7168, n=2048,
E=256, k=8, r=32, alpha=32 (P = 262144 pairs, 22.5 GB of expert weights drawn on the
device), through the C ABI in the launch configuration bench.py uses.

Routing and the permutation are checked in full (bit-exact).  The oracle evaluates Y
and dX rows of sampled tokens, and the adapter and expert-weight gradients of a
median expert.  It reads only the weights of the experts it touches, converted to
fp64 when asked for, so the 22.5 GB never sit in host memory.
"""
import numpy as np
import pytest
import torch

import mixture_experts_lora_b200 as ml
import oracle.moe_lora_oracle as O
from moe_inputs import CONFIGS, generate

from gpu_common import TOL, TOL_W, ensure_built, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


class _ExpertsOnDevice:
    """W[e] as an fp64 array, copied from the device tensor when indexed."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, e):
        return self.t[int(e)].to(torch.float64).cpu().numpy()


def test_deepseek_shape_sampled_parity():
    cfg = CONFIGS["deepseek_v3"]
    inp = generate(cfg, seed=0, device="cuda")
    T, m, n, E, k = cfg.T, cfg.m, cfg.n, cfg.E, cfg.k
    buf = ml.alloc_buffers(T, m, n, E, k, cfg.r, cfg.scale)
    dW_gu = torch.empty(E, m, 2 * n, dtype=torch.bfloat16, device="cuda")
    dW_d = torch.empty(E, n, m, dtype=torch.bfloat16, device="cuda")
    ml.layer_forward(inp, k, cfg.scale, buf)
    ml.layer_backward_full(inp, inp["dY"], k, cfg.scale, buf, dW_gu, dW_d)
    torch.cuda.synchronize()
    st = ml.moe_get_device_error()
    assert st == ml.MOE_OK, ml.status_string(st)

    # routing and permutation in full
    ids, w = O.route_topk(inp["logits"].cpu().numpy(), k)
    assert np.array_equal(buf.ids.cpu().numpy(), ids)
    assert rel_err(to_np(buf.w), w) <= TOL_W
    counts, offsets, sp, pos = O.permute(ids, E)
    assert np.array_equal(buf.counts.cpu().numpy(), counts)
    assert np.array_equal(buf.offsets.cpu().numpy(), offsets)
    assert np.array_equal(buf.sorted_pairs.cpu().numpy(), sp)
    assert np.array_equal(buf.pair_pos.cpu().numpy(), pos)

    W = {name: _ExpertsOnDevice(inp[name]) for name in ("W_gu", "W_d", "A_gu", "B_gu", "A_d", "B_d")}
    toks = [0, 12345, T - 1]
    Yo = np.stack([O.token_forward(inp, t, k, cfg.scale, W=W) for t in toks])
    dXo = np.stack([O.token_backward_dx(inp, t, k, cfg.scale, W=W) for t in toks])
    errs = {"Y": rel_err(to_np(buf.Y[toks]), Yo), "dX": rel_err(to_np(buf.dX[toks]), dXo)}

    e = int(np.argsort(counts, kind="stable")[E // 2])      # a median expert
    ref = O.expert_lora_grads(inp, e, k, cfg.scale, ids=ids, w=w, W=W)
    for name, got, r in zip(("dA_gu", "dB_gu", "dA_d", "dB_d"),
                            (buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d), ref):
        errs[f"{name}[{e}]"] = rel_err(to_np(got[e]), r)
    rg, rd = O.expert_weight_grads(inp, e, k, cfg.scale, ids=ids, w=w, W=W)
    errs[f"dW_gu[{e}]"] = rel_err(to_np(dW_gu[e]), rg)
    errs[f"dW_d[{e}]"] = rel_err(to_np(dW_d[e]), rd)
    bad = {key: v for key, v in errs.items() if not v <= TOL}
    assert not bad, f"DeepSeek-shape parity failures {bad} (all: {errs})"
    print("deepseek_v3", counts[e], errs)
