"""Full fine-tuning: expert-weight gradients through the C ABI against the fp64 oracle.

moe_grouped_gemm_full_bwd gives dW_gu[e] = X_e^T dGU_e [m, 2n] and dW_d[e] = H_e^T dy_e
[n, m], contractions over each expert's ragged row count, next to everything the
LoRA backward gives.  Checked element by element at small sizes (ragged segments;
widths that are and are not multiples of 64; experts with no rows, one row, and
segments on and off the 16- and 64-row steps), per expert against that expert's own
scale; the other outputs bit-identical to moe_grouped_gemm_lora_bwd; the adapter
gradients left untouched when not asked for; and, at full size, sampled experts.
"""
import numpy as np
import pytest
import torch

import mixture_experts_lora_b200 as ml
import oracle.moe_lora_oracle as O
from moe_inputs import CONFIGS, small_config

from gpu_common import (TOL, check_full_parity, ensure_built, inputs_on, oracle_full, rel_err,
                        to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def _full(inp, cfg, adapters=True, buf=None):
    T, m = inp["X"].shape
    n, E = cfg.n, cfg.E
    if buf is None:
        buf = ml.alloc_buffers(T, m, n, E, cfg.k, cfg.r, cfg.scale)
    nan = float("nan")
    dW_gu = torch.full((E, m, 2 * n), nan, dtype=torch.bfloat16, device="cuda")
    dW_d = torch.full((E, n, m), nan, dtype=torch.bfloat16, device="cuda")
    ml.layer_forward(inp, cfg.k, cfg.scale, buf)
    ml.layer_backward_full(inp, inp["dY"], cfg.k, cfg.scale, buf, dW_gu, dW_d, adapters=adapters)
    torch.cuda.synchronize()
    st = ml.moe_get_device_error()
    assert st == ml.MOE_OK, ml.status_string(st)
    return buf, dW_gu, dW_d


def _check_weight_grads(dW_gu, dW_d, ref_gu, ref_d, counts):
    g, d = to_np(dW_gu), to_np(dW_d)
    assert np.all(np.isfinite(g)) and np.all(np.isfinite(d)), "every entry written"
    errs = {"dW_gu": rel_err(g, ref_gu), "dW_d": rel_err(d, ref_d)}
    for e in range(len(counts)):
        if counts[e] == 0:
            assert not np.any(g[e]) and not np.any(d[e]), f"expert {e} has no rows"
        else:
            errs[f"dW_gu[{e}]"] = rel_err(g[e], ref_gu[e])
            errs[f"dW_d[{e}]"] = rel_err(d[e], ref_d[e])
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, f"weight-gradient parity failures {bad}"
    return errs


def _hot_empty(cpu):
    cpu["logits"][:, 2] += 25.0            # expert 2 takes every token (k = 2: plus one more)
    cpu["logits"][:, 6:] -= 25.0           # experts 6, 7: no rows ...
    cpu["logits"][5, 7] += 60.0            # ... except one row for expert 7


CASES = {
    "tiny": (CONFIGS["tiny"], None),
    "ragged_odd_widths": (small_config(T=33, m=144, n=80, E=5, k=3, r=16, alpha=16), None),
    "hot_and_empty": (small_config(T=200, m=128, n=64, E=8, k=2, r=8, alpha=16), _hot_empty),
    "one_expert_whole_steps": (small_config(T=192, m=64, n=32, E=1, k=1, r=8, alpha=8), None),
    "wide_rank32": (small_config(T=300, m=256, n=192, E=6, k=2, r=32, alpha=32), None),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_weight_grads_match_oracle(name):
    cfg, mutate = CASES[name]
    inp, cpu = inputs_on(cfg, seed=2)
    if mutate is not None:
        mutate(cpu)
        inp = {k: v.cuda().contiguous() for k, v in cpu.items()}
    buf, dW_gu, dW_d = _full(inp, cfg)
    Y, aux, g = oracle_full(cpu, cfg)
    ref_gu, ref_d = O.moe_weight_grads(cpu, aux, g, cpu["dY"], cfg.k)
    errs = _check_weight_grads(dW_gu, dW_d, ref_gu, ref_d, aux["counts"])
    check_full_parity(buf, cpu, cfg)     # routing, forward, dX and adapter gradients
    if name == "hot_and_empty":
        counts = aux["counts"]
        assert counts[6] == 0 and counts[7] == 1 and counts[2] == cfg.T
    print(name, {k: v for k, v in errs.items() if "[" not in k})


def test_other_outputs_match_lora_backward_bitwise():
    cfg = small_config(T=260, m=192, n=96, E=6, k=2, r=16, alpha=32)
    inp, _ = inputs_on(cfg, seed=4)
    a = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r, cfg.scale)
    ml.layer_step(inp, cfg.k, cfg.scale, a)
    torch.cuda.synchronize()
    snap = {k: getattr(a, k).clone() for k in ("dX", "dX_sorted", "dA_gu", "dB_gu", "dA_d", "dB_d")}
    b, _, _ = _full(inp, cfg)
    for k, v in snap.items():
        assert torch.equal(_bits(v), _bits(getattr(b, k))), k


def test_adapter_gradients_skipped_when_not_asked():
    cfg = small_config(T=150, m=128, n=64, E=4, k=2, r=8, alpha=16)
    inp, cpu = inputs_on(cfg, seed=5)
    # a layer without adapters: B = 0, so the rank-r terms add exact zeros
    for name in ("B_gu", "B_d"):
        cpu[name] = torch.zeros_like(cpu[name])
        inp[name] = torch.zeros_like(inp[name])
    buf = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r, cfg.scale)
    for t in (buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d):
        t.fill_(float("nan"))
    buf, dW_gu, dW_d = _full(inp, cfg, adapters=False, buf=buf)
    for t in (buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d):
        assert torch.all(torch.isnan(t)), "adapter gradients untouched"
    Y, aux, g = oracle_full(cpu, cfg)
    assert rel_err(to_np(buf.dX), g["dX"]) <= TOL
    ref_gu, ref_d = O.moe_weight_grads(cpu, aux, g, cpu["dY"], cfg.k)
    _check_weight_grads(dW_gu, dW_d, ref_gu, ref_d, aux["counts"])


def test_weight_grads_deterministic_bitwise():
    cfg = small_config(T=400, m=128, n=64, E=4, k=2, r=8, alpha=16)
    inp, _ = inputs_on(cfg, seed=8)
    _, a_gu, a_d = _full(inp, cfg)
    _, b_gu, b_d = _full(inp, cfg)
    assert torch.equal(_bits(a_gu), _bits(b_gu)) and torch.equal(_bits(a_d), _bits(b_d))


@pytest.mark.parametrize("name", ["qwen3_30b_a3b", "qwen3_skewed"])
def test_full_size_sampled_weight_grads(name):
    cfg = CONFIGS[name]
    inp, cpu = inputs_on(cfg)
    buf, dW_gu, dW_d = _full(inp, cfg)
    ids, w = O.route_topk(cpu["logits"].numpy(), cfg.k)
    assert np.array_equal(buf.ids.cpu().numpy(), ids)
    counts = np.bincount(ids.reshape(-1), minlength=cfg.E)
    order = np.argsort(counts, kind="stable")
    experts = [int(order[-1]), int(order[len(order) // 2])]
    if counts[order[0]] == 0:
        experts.append(int(order[0]))
    W = {k: O.to64(cpu[k]) for k in ("W_gu", "W_d", "A_gu", "B_gu", "A_d", "B_d")}
    errs = {}
    for e in experts:
        rg, rd = O.expert_weight_grads(cpu, e, cfg.k, cfg.scale, ids=ids, w=w, W=W)
        g, d = to_np(dW_gu[e]), to_np(dW_d[e])
        if counts[e] == 0:
            assert not np.any(g) and not np.any(d)
        else:
            errs[f"dW_gu[{e}]"] = rel_err(g, rg)
            errs[f"dW_d[{e}]"] = rel_err(d, rd)
    assert max(errs.values()) <= TOL, errs
    assert bool(torch.isfinite(dW_gu).all()) and bool(torch.isfinite(dW_d).all())
    print(name, errs)
