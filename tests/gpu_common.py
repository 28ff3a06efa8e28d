"""Shared helpers of the GPU parity tests: run the layer through the C ABI and
compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_lora_b200 as ml
import oracle.moe_lora_oracle as O
from moe_inputs import generate

TOL = 1e-2          # max|gpu - oracle| / max|oracle| for bf16 outputs (fp32 accumulation)
TOL_W = 1e-5        # routing weights, relative


def ensure_built():
    from mixture_experts_lora_b200 import build
    build.build(quiet=True)
    ml.lib()


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref)) / den)


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def inputs_on(cfg, device="cuda", seed=0, gen_device="cpu"):
    """Inputs drawn on `gen_device` and copied to `device` (identical bits)."""
    t = generate(cfg, seed=seed, device=gen_device)
    return {k: v.to(device).contiguous() for k, v in t.items()}, t


def run_layer(inp, cfg, buf=None):
    """Forward + backward of the whole layer through the ABI; returns the buffers."""
    if buf is None:
        T, m = inp["X"].shape
        buf = ml.alloc_buffers(T, m, cfg.n, cfg.E, cfg.k, cfg.r, cfg.scale)
    ml.layer_step(inp, cfg.k, cfg.scale, buf)
    torch.cuda.synchronize()
    st = ml.moe_get_device_error()
    assert st == ml.MOE_OK, ml.status_string(st)
    return buf


def oracle_full(cpu_inp, cfg):
    Y, aux = O.moe_forward(cpu_inp, cfg.k, cfg.scale)
    g = O.moe_backward(cpu_inp, aux, cpu_inp["dY"], cfg.k, cfg.scale)
    return Y, aux, g


def check_full_parity(buf, cpu_inp, cfg, tol=TOL):
    """Element-by-element comparison of every output and saved intermediate."""
    Y, aux, g = oracle_full(cpu_inp, cfg)
    ids = buf.ids.cpu().numpy()
    assert np.array_equal(ids, aux["ids"]), "expert ids"
    assert rel_err(to_np(buf.w), aux["w"]) <= TOL_W, "routing weights"
    assert np.array_equal(buf.counts.cpu().numpy(), aux["counts"]), "counts"
    assert np.array_equal(buf.offsets.cpu().numpy(), aux["offsets"]), "offsets"
    assert np.array_equal(buf.sorted_pairs.cpu().numpy(), aux["sorted_pairs"]), "sorted_pairs"
    assert np.array_equal(buf.pair_pos.cpu().numpy(), aux["pair_pos"]), "pair_pos"
    # the saved sorted input rows are X itself, gathered: bit-exact
    assert torch.equal(buf.save_Xs.cpu(), cpu_inp["X"][torch.from_numpy(aux["sorted_pairs"] // cfg.k)]), "save_Xs"
    errs = {
        "GU": rel_err(to_np(buf.save_GU), aux["gu"]),
        "H": rel_err(to_np(buf.save_H), aux["h"]),
        "XA": rel_err(to_np(buf.save_XA), aux["xa"]),
        "HA": rel_err(to_np(buf.save_HA), aux["ha"]),
        "Y_sorted": rel_err(to_np(buf.Y_sorted), aux["yp"]),
        "Y": rel_err(to_np(buf.Y), Y),
        "dX_sorted": rel_err(to_np(buf.dX_sorted), g["dxp"]),
        "dX": rel_err(to_np(buf.dX), g["dX"]),
        "dA_gu": rel_err(to_np(buf.dA_gu), g["dA_gu"]),
        "dB_gu": rel_err(to_np(buf.dB_gu), g["dB_gu"]),
        "dA_d": rel_err(to_np(buf.dA_d), g["dA_d"]),
        "dB_d": rel_err(to_np(buf.dB_d), g["dB_d"]),
    }
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"parity failures {bad} (all: {errs})"
    # experts with no rows get exactly zero adapter gradients
    for e in np.nonzero(aux["counts"] == 0)[0]:
        for t in (buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d):
            assert not torch.any(t[int(e)] != 0)
    return errs


def check_sampled_parity(buf, cpu_inp, cfg, n_tokens=24, n_experts=3, seed=0, tol=TOL):
    """Full-size check on sampled outputs the oracle computes one by one: routing
    and permutation in full (bit-exact), Y and dX rows of sampled tokens, and the
    adapter gradients of sampled experts (busiest, a median one, and an empty one
    if any)."""
    logits = cpu_inp["logits"].numpy()
    ids, w = O.route_topk(logits, cfg.k)
    gids = buf.ids.cpu().numpy()
    assert np.array_equal(gids, ids), "expert ids"
    assert rel_err(to_np(buf.w), w) <= TOL_W, "routing weights"
    counts, offsets, sp, pos = O.permute(ids, cfg.E)
    assert np.array_equal(buf.counts.cpu().numpy(), counts)
    assert np.array_equal(buf.offsets.cpu().numpy(), offsets)
    assert np.array_equal(buf.sorted_pairs.cpu().numpy(), sp)
    assert np.array_equal(buf.pair_pos.cpu().numpy(), pos)
    W = {k: O.to64(cpu_inp[k]) for k in ("W_gu", "W_d", "A_gu", "B_gu", "A_d", "B_d")}
    rng = np.random.default_rng(seed)
    T = logits.shape[0]
    toks = sorted(set([0, T - 1] + list(rng.choice(T, size=min(n_tokens, T), replace=False))))
    Yg = buf.Y[toks].to("cpu", torch.float64).numpy()
    dXg = buf.dX[toks].to("cpu", torch.float64).numpy()
    Yo = np.stack([O.token_forward(cpu_inp, t, cfg.k, cfg.scale, W=W) for t in toks])
    dXo = np.stack([O.token_backward_dx(cpu_inp, t, cfg.k, cfg.scale, W=W) for t in toks])
    errs = {"Y": rel_err(Yg, Yo), "dX": rel_err(dXg, dXo)}
    order = np.argsort(counts, kind="stable")
    experts = [int(order[-1]), int(order[len(order) // 2])]
    if counts[order[0]] == 0:
        experts.append(int(order[0]))
    experts += [int(e) for e in rng.choice(cfg.E, size=max(0, n_experts - len(experts)), replace=False)]
    for e in experts:
        ref = O.expert_lora_grads(cpu_inp, e, cfg.k, cfg.scale, ids=ids, w=w, W=W)
        got = [to_np(t[e]) for t in (buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d)]
        for name, a, b in zip(("dA_gu", "dB_gu", "dA_d", "dB_d"), got, ref):
            if counts[e] == 0:
                assert not np.any(a), (name, e)
            else:
                errs[f"{name}[{e}]"] = rel_err(a, b)
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"sampled parity failures {bad} (all: {errs})"
    return errs
