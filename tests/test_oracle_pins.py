"""Pins for the fp64 oracle: each checks it against something other than itself.

- Split-LoRA equals the materialised PEFT form X (W + c A B)   (associativity)
- B = 0 reduces exactly to the base MoE with no adapters
- k = E with equal logits is the plain average of all experts
- gradients match central finite differences and torch.autograd (fp64)
- full fine-tuning: the expert-weight gradients match finite differences and
  autograd, and chain to the adapter gradients through W' = W + c A B
- routing and permutation match brute force, ties included
- a single expert with k = 1 and no adapters is the textbook SwiGLU MLP
- the accounting helpers match the worked numbers the pages print
- planted mistakes in the oracle are caught by these pins
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.moe_lora_oracle as O
from moe_inputs import generate, small_config, CONFIGS
from mixture_experts_lora_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_numbers.json")


def _inp64(cfg, seed=0):
    """Inputs as fp64 numpy arrays (bf16-rounded values), logits fp32."""
    t = generate(cfg, seed=seed)
    out = {k: O.to64(v) for k, v in t.items()}
    out["logits"] = t["logits"].numpy().astype(np.float32)
    return out


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


CFG_S = small_config(T=48, m=64, n=32, E=6, k=2, r=8, alpha=16.0)   # c = 2


# ---------------------------------------------------------------- identities
def check_split_equals_merged(cfg=CFG_S):
    inp = _inp64(cfg)
    Y, _ = O.moe_forward(inp, cfg.k, cfg.scale)
    Ym = O.moe_forward_merged(inp, cfg.k, cfg.scale)
    return _rel(Y, Ym)


def test_split_equals_merged():
    assert check_split_equals_merged() < 1e-12


def test_b_zero_is_base_moe():
    inp = _inp64(CFG_S)
    inp["B_gu"] = np.zeros_like(inp["B_gu"])
    inp["B_d"] = np.zeros_like(inp["B_d"])
    Y, _ = O.moe_forward(inp, CFG_S.k, CFG_S.scale)
    Yb = O.moe_forward_base(inp, CFG_S.k)
    assert np.array_equal(Y, Yb)


def test_k_equals_E_equal_logits_is_average():
    cfg = small_config(T=16, m=32, n=16, E=4, k=4, r=4, alpha=8.0)
    inp = _inp64(cfg)
    inp["logits"] = np.zeros_like(inp["logits"])
    Y, aux = O.moe_forward(inp, cfg.k, cfg.scale)
    assert np.allclose(aux["w"], 1.0 / cfg.E, rtol=0, atol=1e-15)
    ref = np.zeros_like(Y)
    for e in range(cfg.E):
        f = O.expert_forward(inp["X"], inp["W_gu"][e], inp["A_gu"][e], inp["B_gu"][e],
                             inp["W_d"][e], inp["A_d"][e], inp["B_d"][e], cfg.scale)
        ref += f["y"]
    ref /= cfg.E
    assert _rel(Y, ref) < 1e-13


def test_single_expert_is_textbook_swiglu():
    cfg = small_config(T=20, m=32, n=24, E=1, k=1, r=4, alpha=4.0)
    inp = _inp64(cfg)
    Y = O.moe_forward_base(inp, 1)
    x = torch.from_numpy(inp["X"])
    Wg = torch.from_numpy(inp["W_gu"][0][:, :cfg.n])
    Wu = torch.from_numpy(inp["W_gu"][0][:, cfg.n:])
    Wd = torch.from_numpy(inp["W_d"][0])
    ref = (torch.nn.functional.silu(x @ Wg) * (x @ Wu)) @ Wd
    assert _rel(Y, ref.numpy()) < 1e-13


# ---------------------------------------------------------------- gradients
def _loss(inp, dY, cfg):
    Y, _ = O.moe_forward(inp, cfg.k, cfg.scale, keep=False)
    return float(np.sum(dY * Y))


def check_fd(cfg=None, n_coords=64, seed=1):
    """Max relative error of the analytic gradient against central differences."""
    cfg = cfg or small_config(T=24, m=32, n=16, E=4, k=2, r=4, alpha=8.0)
    inp = _inp64(cfg)
    dY = inp["dY"]
    Y, aux = O.moe_forward(inp, cfg.k, cfg.scale)
    g = O.moe_backward(inp, aux, dY, cfg.k, cfg.scale)
    grads = {"X": g["dX"], "A_gu": g["dA_gu"], "B_gu": g["dB_gu"], "A_d": g["dA_d"], "B_d": g["dB_d"]}
    rng = np.random.default_rng(seed)
    h = 1e-6
    worst = 0.0
    for name, G in grads.items():
        base = inp[name]
        flat_idx = rng.choice(base.size, size=min(n_coords, base.size), replace=False)
        scale = max(np.max(np.abs(G)), 1e-12)
        for fi in flat_idx:
            idx = np.unravel_index(fi, base.shape)
            orig = base[idx]
            base[idx] = orig + h
            lp = _loss(inp, dY, cfg)
            base[idx] = orig - h
            lm = _loss(inp, dY, cfg)
            base[idx] = orig
            fd = (lp - lm) / (2 * h)
            worst = max(worst, abs(fd - G[idx]) / scale)
    return worst


def test_gradients_match_finite_differences():
    assert check_fd() < 1e-6


def test_gradients_match_torch_autograd():
    cfg = small_config(T=12, m=16, n=8, E=3, k=2, r=4, alpha=8.0)
    inp = _inp64(cfg)
    Y, aux = O.moe_forward(inp, cfg.k, cfg.scale)
    g = O.moe_backward(inp, aux, inp["dY"], cfg.k, cfg.scale)

    dW_gu, dW_d = O.moe_weight_grads(inp, aux, g, inp["dY"], cfg.k)
    g["dW_gu"], g["dW_d"] = dW_gu, dW_d
    T = {k: torch.tensor(v, dtype=torch.float64,
                         requires_grad=k in ("X", "A_gu", "B_gu", "A_d", "B_d", "W_gu", "W_d"))
         for k, v in inp.items() if k != "logits"}
    # routing written differently from the oracle: softmax over all experts, then
    # torch.topk, then renormalise (no ties at these random logits)
    probs = torch.softmax(torch.tensor(inp["logits"], dtype=torch.float64), dim=-1)
    pv, pi = torch.topk(probs, cfg.k, dim=-1)
    pv = pv / pv.sum(-1, keepdim=True)
    c = cfg.scale
    n = cfg.n
    rows = []
    for t in range(cfg.T):
        y = torch.zeros(cfg.m, dtype=torch.float64)
        for j in range(cfg.k):
            e = int(pi[t, j])
            Wgu = T["W_gu"][e] + c * T["A_gu"][e] @ T["B_gu"][e]    # merged on purpose
            Wd = T["W_d"][e] + c * T["A_d"][e] @ T["B_d"][e]
            gu = T["X"][t] @ Wgu
            y = y + pv[t, j] * ((torch.nn.functional.silu(gu[:n]) * gu[n:]) @ Wd)
        rows.append(y)
    Yt = torch.stack(rows)
    assert _rel(Y, Yt.detach().numpy()) < 1e-12
    (Yt * T["dY"]).sum().backward()
    for name, key in (("X", "dX"), ("A_gu", "dA_gu"), ("B_gu", "dB_gu"), ("A_d", "dA_d"), ("B_d", "dB_d"),
                      ("W_gu", "dW_gu"), ("W_d", "dW_d")):
        assert _rel(g[key], T[name].grad.numpy()) < 1e-11, name


# ---------------------------------------------------------------- routing / permute
def _route_bruteforce(logits, k):
    T, E = logits.shape
    ids = np.zeros((T, k), np.int64)
    w = np.zeros((T, k))
    for t in range(T):
        taken = set()
        vals = []
        for _ in range(k):
            best = None
            for e in range(E):
                if e in taken:
                    continue
                if best is None or float(logits[t, e]) > float(logits[t, best]):
                    best = e          # strict '>' keeps the lower index on ties
            taken.add(best)
            vals.append(float(logits[t, best]))
        ids[t] = sorted(taken, key=lambda e: (-float(logits[t, e]), e))
        z = [math.exp(v - max(vals)) for v in vals]
        w[t] = [zi / sum(z) for zi in z]
    return ids, w


def check_route(seed=3):
    rng = np.random.default_rng(seed)
    # coarse values force many ties
    logits = (np.round(rng.normal(size=(40, 9)) * 2) / 2).astype(np.float32)
    ids, w = O.route_topk(logits, 3)
    bids, bw = _route_bruteforce(logits, 3)
    return np.array_equal(ids, bids) and np.allclose(w, bw, rtol=1e-14, atol=0)


def test_route_matches_bruteforce_with_ties():
    assert check_route()


def test_permute_matches_bruteforce():
    rng = np.random.default_rng(4)
    E, T, k = 7, 50, 3
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    ids[:, 0] = 2                       # one hot expert
    counts, offsets, sp, pos = O.permute(ids, E)
    flat = ids.reshape(-1)
    want = [p for e in range(E) for p in range(flat.size) if flat[p] == e]
    assert list(sp) == want
    assert list(counts) == [int(np.sum(flat == e)) for e in range(E)]
    assert offsets[0] == 0 and offsets[-1] == flat.size
    assert all(pos[sp[q]] == q for q in range(flat.size))
    assert counts[5] >= 0 and offsets[E] == T * k


def test_unpermute_combine_matches_per_token_bruteforce():
    # Y[t] is token t's routing-weighted sum of its k expert outputs, wherever the
    # permutation put those rows; the plain form sums them with weight 1
    rng = np.random.default_rng(11)
    T, k, m = 9, 3, 5
    yp = rng.standard_normal((T * k, m))
    w = rng.random((T, k))
    pos = rng.permutation(T * k)
    for weights in (w, None):
        Y = O.unpermute_combine(yp, weights, pos, k)
        for t in range(T):
            want = np.zeros(m)
            for j in range(k):
                want = want + (1.0 if weights is None else w[t, j]) * yp[pos[t * k + j]]
            assert np.allclose(Y[t], want, rtol=1e-15, atol=1e-15)
    # the identity permutation with one-hot weights picks a single row
    one = np.zeros((T, k))
    one[:, 1] = 1.0
    assert np.array_equal(O.unpermute_combine(yp, one, np.arange(T * k), k), yp[1::k])


def test_permute_rejects_bad_ids():
    with pytest.raises(ValueError):
        O.permute(np.array([[0, 9]]), 4)


def test_empty_experts_have_zero_grads():
    cfg = small_config(T=16, m=32, n=16, E=6, k=1, r=4, alpha=4.0)
    inp = _inp64(cfg)
    inp["logits"][:, :] = -5.0
    inp["logits"][:, 1] = 5.0           # every token picks expert 1
    Y, aux = O.moe_forward(inp, cfg.k, cfg.scale)
    g = O.moe_backward(inp, aux, inp["dY"], cfg.k, cfg.scale)
    g["dW_gu"], g["dW_d"] = O.moe_weight_grads(inp, aux, g, inp["dY"], cfg.k)
    assert aux["counts"][1] == cfg.T
    for e in (0, 2, 3, 4, 5):
        for key in ("dA_gu", "dB_gu", "dA_d", "dB_d", "dW_gu", "dW_d"):
            assert not np.any(g[key][e])
    assert np.any(g["dW_gu"][1]) and np.any(g["dW_d"][1])


def test_sampled_helpers_agree_with_full_layer():
    inp = _inp64(CFG_S)
    Y, aux = O.moe_forward(inp, CFG_S.k, CFG_S.scale)
    g = O.moe_backward(inp, aux, inp["dY"], CFG_S.k, CFG_S.scale)
    for t in (0, 7, CFG_S.T - 1):
        assert _rel(O.token_forward(inp, t, CFG_S.k, CFG_S.scale), Y[t]) < 1e-13
        assert _rel(O.token_backward_dx(inp, t, CFG_S.k, CFG_S.scale), g["dX"][t]) < 1e-13
    dW_gu, dW_d = O.moe_weight_grads(inp, aux, g, inp["dY"], CFG_S.k)
    for e in (0, 3):
        gs = O.expert_lora_grads(inp, e, CFG_S.k, CFG_S.scale)
        for got, key in zip(gs, ("dA_gu", "dB_gu", "dA_d", "dB_d")):
            assert _rel(got, g[key][e]) < 1e-13
        wg, wd = O.expert_weight_grads(inp, e, CFG_S.k, CFG_S.scale)
        assert _rel(wg, dW_gu[e]) < 1e-13 and _rel(wd, dW_d[e]) < 1e-13


# ---------------------------------------------------------------- worked numbers
def test_accounting_matches_pages_worked_numbers():
    with open(GOLDEN) as f:
        entries = json.load(f)["entries"]
    for ent in entries:
        fn = getattr(acc, ent["quantity"])
        got = fn(**ent["args"])
        if "value" in ent:
            assert got == ent["value"], ent
        elif "approx" in ent:
            assert abs(got - ent["approx"]) <= ent["rel_tol"] * ent["approx"], (ent, got)
        else:
            assert abs(got - ent["value_by_formula"]) <= ent["rel_tol"] * ent["value_by_formula"], (ent, got)
            # the page's own rounded figure does not follow from its formula
            assert abs(got - ent["printed"]) > 0.2 * ent["printed"]


def test_flop_formula_matches_qwen_figure():
    c = CONFIGS["qwen3_30b_a3b"]
    total = acc.flops_step(c.T, c.m, c.n, c.k, c.r)
    assert abs(total - 6.386e11) / 6.386e11 < 1e-3
    parts = (acc.flops_gemm_gate_up_fwd, acc.flops_gemm_down_fwd, acc.flops_gemm_down_bwd,
             acc.flops_gemm_gate_up_bwd, acc.flops_lora_wgrad)
    assert sum(f(c.T, c.m, c.n, c.k, c.r) for f in parts) == total


# ---------------------------------------------------------------- full fine-tuning
CFG_W = small_config(T=24, m=32, n=16, E=4, k=2, r=4, alpha=8.0)


def _weight_case(cfg=CFG_W):
    inp = _inp64(cfg)
    Y, aux = O.moe_forward(inp, cfg.k, cfg.scale)
    g = O.moe_backward(inp, aux, inp["dY"], cfg.k, cfg.scale)
    dW_gu, dW_d = O.moe_weight_grads(inp, aux, g, inp["dY"], cfg.k)
    return inp, g, dW_gu, dW_d


def check_weight_fd(n_coords=40, seed=4, h=1e-6):
    """Max relative error of dW_gu, dW_d against central differences of <dY, Y>."""
    cfg = CFG_W
    inp, _, dW_gu, dW_d = _weight_case(cfg)
    rng = np.random.default_rng(seed)
    worst = 0.0
    for name, G in (("W_gu", dW_gu), ("W_d", dW_d)):
        base = inp[name]
        scale = max(np.max(np.abs(G)), 1e-12)
        for fi in rng.choice(base.size, size=n_coords, replace=False):
            idx = np.unravel_index(fi, base.shape)
            orig = base[idx]
            base[idx] = orig + h
            lp = _loss(inp, inp["dY"], cfg)
            base[idx] = orig - h
            lm = _loss(inp, inp["dY"], cfg)
            base[idx] = orig
            worst = max(worst, abs((lp - lm) / (2 * h) - G[idx]) / scale)
    return worst


def test_weight_grads_match_finite_differences():
    assert check_weight_fd() < 1e-6


def test_weight_grads_chain_to_adapter_grads():
    # the layer sees W and the adapters only through W' = W + c A B, so
    # dL/dA = c dL/dW' B^T and dL/dB = c A^T dL/dW' (the adapter gradients are
    # pinned on their own by finite differences and autograd)
    cfg = CFG_S
    inp, g, dW_gu, dW_d = _weight_case(cfg)
    c = cfg.scale
    for e in range(cfg.E):
        assert _rel(c * dW_gu[e] @ inp["B_gu"][e].T, g["dA_gu"][e]) < 1e-12
        assert _rel(c * inp["A_gu"][e].T @ dW_gu[e], g["dB_gu"][e]) < 1e-12
        assert _rel(c * dW_d[e] @ inp["B_d"][e].T, g["dA_d"][e]) < 1e-12
        assert _rel(c * inp["A_d"][e].T @ dW_d[e], g["dB_d"][e]) < 1e-12


def test_weight_pin_catches_planted_mistakes(monkeypatch):
    good = O.moe_weight_grads

    def unweighted(inp, aux, bwd, dY, k):       # dW_d from dY without the routing weight
        a = dict(aux)
        a["w"] = np.ones_like(aux["w"])
        return good(inp, a, bwd, dY, k)
    monkeypatch.setattr(O, "moe_weight_grads", unweighted)
    assert check_weight_fd(n_coords=8) > 1e-3

    def scaled(inp, aux, bwd, dY, k):           # the LoRA scale applied to dW_gu
        gu, d = good(inp, aux, bwd, dY, k)
        return CFG_W.scale * gu, d
    monkeypatch.setattr(O, "moe_weight_grads", scaled)
    assert check_weight_fd(n_coords=8) > 1e-3
    monkeypatch.setattr(O, "moe_weight_grads", good)


# ---------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    good_fwd, good_bwd, good_route = O.expert_forward, O.expert_backward, O.route_topk

    # 1. LoRA scale applied twice on the down projection (forward)
    def bad_fwd(x, W_gu, A_gu, B_gu, W_d, A_d, B_d, c):
        f = good_fwd(x, W_gu, A_gu, B_gu, W_d, A_d, B_d, c)
        f["y"] = f["y"] + (c * c - c) * (f["ha"] @ B_d)
        return f
    monkeypatch.setattr(O, "expert_forward", bad_fwd)
    assert check_split_equals_merged() > 1e-6
    monkeypatch.setattr(O, "expert_forward", good_fwd)

    # 2. dA_gu without its scale c
    def bad_bwd_scale(*a):
        b = good_bwd(*a)
        b["dA_gu"] = b["dA_gu"] / a[-1]
        return b
    monkeypatch.setattr(O, "expert_backward", bad_bwd_scale)
    assert check_fd(n_coords=8) > 1e-3
    monkeypatch.setattr(O, "expert_backward", good_bwd)

    # 3. SwiGLU derivative missing the g(1-s) term: perturbs dX
    def bad_bwd_swiglu(x, fwd, dy, W_gu, A_gu, B_gu, W_d, A_d, B_d, c):
        b = good_bwd(x, fwd, dy, W_gu, A_gu, B_gu, W_d, A_d, B_d, c)
        n = W_gu.shape[1] // 2
        g, u = fwd["gu"][:, :n], fwd["gu"][:, n:]
        s = O.sigmoid(g)
        dg = b["dh"] * u * s
        dgu = np.concatenate([dg, b["dgu"][:, n:]], axis=1)
        b["dx"] = dgu @ W_gu.T + c * ((dgu @ B_gu.T) @ A_gu.T)
        return b
    monkeypatch.setattr(O, "expert_backward", bad_bwd_swiglu)
    assert check_fd(n_coords=8) > 1e-3
    monkeypatch.setattr(O, "expert_backward", good_bwd)

    # 4. ties broken toward the higher expert index
    def bad_route(logits, k):
        lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
        order = np.argsort(-lg[:, ::-1], axis=1, kind="stable")
        ids = (lg.shape[1] - 1 - order[:, :k]).astype(np.int64)
        sel = np.take_along_axis(lg, ids, axis=1)
        z = np.exp(sel - sel[:, :1])
        return ids, z / z.sum(1, keepdims=True)
    monkeypatch.setattr(O, "route_topk", bad_route)
    assert not check_route()
    monkeypatch.setattr(O, "route_topk", good_route)


# ---------------------------------------------------------------- router backward
def _router_loss(logits64, ids, yp, pos, dY):
    """L = sum_t <dY[t], sum_j w[t,j] y_(t,j)> with w = softmax over the fixed picks."""
    T, k = ids.shape
    sel = np.take_along_axis(logits64, ids, axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    w = z / z.sum(axis=1, keepdims=True)
    Y = np.zeros_like(dY)
    for j in range(k):
        Y += w[:, j:j + 1] * yp[pos.reshape(T, k)[:, j]]
    return float(np.sum(Y * dY))


def _router_case(seed=3):
    cfg = small_config(T=40, m=32, n=16, E=7, k=3, r=8, alpha=16.0)
    inp = _inp64(cfg, seed=seed)
    Y, aux = O.moe_forward(inp, cfg.k, cfg.scale)
    return cfg, inp, Y, aux


def check_router_fd(h=1e-6):
    cfg, inp, Y, aux = _router_case()
    dl, _ = O.router_backward(inp["dY"], aux["yp"], aux["ids"], aux["w"], aux["pair_pos"], cfg.E)
    lg = inp["logits"].astype(np.float64)
    worst, scale = 0.0, max(np.max(np.abs(dl)), 1e-12)
    for t in range(0, cfg.T, 3):
        for e in range(cfg.E):            # picked and unpicked logits alike
            lp, lm = lg.copy(), lg.copy()
            lp[t, e] += h
            lm[t, e] -= h
            fd = (_router_loss(lp, aux["ids"], aux["yp"], aux["pair_pos"], inp["dY"]) -
                  _router_loss(lm, aux["ids"], aux["yp"], aux["pair_pos"], inp["dY"])) / (2 * h)
            worst = max(worst, abs(fd - dl[t, e]) / scale)
    return worst


def test_router_backward_matches_finite_differences():
    assert check_router_fd() < 1e-6


def test_router_backward_matches_autograd_and_sums_to_zero():
    cfg, inp, Y, aux = _router_case(seed=5)
    dl, dw = O.router_backward(inp["dY"], aux["yp"], aux["ids"], aux["w"], aux["pair_pos"], cfg.E)
    # autograd through a differently written renormalisation: full softmax over E,
    # pick, divide by the picked sum (equal to a softmax over the picked logits)
    lt = torch.tensor(inp["logits"].astype(np.float64), requires_grad=True)
    probs = torch.softmax(lt, dim=-1)
    ids = torch.tensor(aux["ids"])
    pv = torch.gather(probs, 1, ids)
    pv = pv / pv.sum(-1, keepdim=True)
    yp = torch.tensor(aux["yp"])
    pos = torch.tensor(aux["pair_pos"]).reshape(cfg.T, cfg.k)
    Yt = sum(pv[:, j:j + 1] * yp[pos[:, j]] for j in range(cfg.k))
    assert _rel(Y, Yt.detach().numpy()) < 1e-12
    (Yt * torch.tensor(inp["dY"])).sum().backward()
    assert _rel(dl, lt.grad.numpy()) < 1e-11
    # the softmax Jacobian annihilates constants: every row sums to zero
    assert np.max(np.abs(dl.sum(axis=1))) < 1e-12 * max(1.0, np.max(np.abs(dl)))


def test_router_pin_catches_planted_mistake(monkeypatch):
    good = O.router_backward

    def bad(dY, yp, ids, w, pair_pos, E):       # forgets the - sum_i w_i dw_i term
        dl, dw = good(dY, yp, ids, w, pair_pos, E)
        out = np.zeros_like(dl)
        np.put_along_axis(out, np.asarray(ids), np.asarray(w) * dw, axis=1)
        return out, dw
    monkeypatch.setattr(O, "router_backward", bad)
    assert check_router_fd() > 1e-3


# ---------------------------------------------------------------- separate gate/up adapters
def _split_inputs(cfg, seed=7, b_std=0.5):
    inp = _inp64(cfg, seed=seed)
    rng = np.random.default_rng(seed)
    E, m, n, r = cfg.E, cfg.m, cfg.n, cfg.r
    inp["A_g"] = rng.normal(0, 1 / math.sqrt(m), (E, m, r))
    inp["A_u"] = rng.normal(0, 1 / math.sqrt(m), (E, m, r))
    inp["B_g"] = rng.normal(0, b_std, (E, r, n))
    inp["B_u"] = rng.normal(0, b_std, (E, r, n))
    return inp


def _packed(inp):
    """Rank-2r fused adapter A = [A_g | A_u], B = [[B_g, 0], [0, B_u]]; the down
    adapter is padded to rank 2r with zeros (one rank for both projections)."""
    E, r, n = inp["B_g"].shape
    A = np.concatenate([inp["A_g"], inp["A_u"]], axis=2)
    B = np.zeros((E, 2 * r, 2 * n))
    B[:, :r, :n] = inp["B_g"]
    B[:, r:, n:] = inp["B_u"]
    Ad = np.concatenate([inp["A_d"], np.zeros_like(inp["A_d"])], axis=2)
    Bd = np.concatenate([inp["B_d"], np.zeros_like(inp["B_d"])], axis=1)
    return A, B, Ad, Bd


CFG_SPLIT = small_config(T=40, m=32, n=16, E=5, k=2, r=4, alpha=8.0)


def test_split_gate_up_equals_block_packed_fused_adapter():
    cfg = CFG_SPLIT
    inp = _split_inputs(cfg)
    Y, g = O.layer_split_gate_up(inp, cfg.k, cfg.scale)
    packed = dict(inp)
    packed["A_gu"], packed["B_gu"], packed["A_d"], packed["B_d"] = _packed(inp)
    Yp, aux = O.moe_forward(packed, cfg.k, cfg.scale)
    gp = O.moe_backward(packed, aux, packed["dY"], cfg.k, cfg.scale)
    r, n = cfg.r, cfg.n
    assert _rel(Y, Yp) < 1e-12
    assert _rel(g["dX"], gp["dX"]) < 1e-12
    assert _rel(g["dA_g"], gp["dA_gu"][:, :, :r]) < 1e-12
    assert _rel(g["dA_u"], gp["dA_gu"][:, :, r:]) < 1e-12
    assert _rel(g["dB_g"], gp["dB_gu"][:, :r, :n]) < 1e-12
    assert _rel(g["dB_u"], gp["dB_gu"][:, r:, n:]) < 1e-12
    assert _rel(g["dA_d"], gp["dA_d"][:, :, :r]) < 1e-12 and _rel(g["dB_d"], gp["dB_d"][:, :r]) < 1e-12
    assert np.all(gp["dA_d"][:, :, r:] == 0) and np.all(gp["dB_d"][:, r:] == 0)   # padding stays zero


def test_split_gate_up_zero_b_is_base_moe():
    cfg = CFG_SPLIT
    inp = _split_inputs(cfg)
    inp["B_g"][:] = 0.0
    inp["B_u"][:] = 0.0
    inp["B_d"][:] = 0.0
    Y, _ = O.layer_split_gate_up(inp, cfg.k, cfg.scale)
    assert _rel(Y, O.moe_forward_base(inp, cfg.k)) < 1e-13


def check_split_fd(h=1e-6, n_coords=24, seed=2):
    cfg = CFG_SPLIT
    inp = _split_inputs(cfg)
    _, g = O.layer_split_gate_up(inp, cfg.k, cfg.scale)
    dY = inp["dY"]
    rng = np.random.default_rng(seed)
    worst = 0.0
    for name, key in (("X", "dX"), ("A_g", "dA_g"), ("B_g", "dB_g"), ("A_u", "dA_u"), ("B_u", "dB_u")):
        base = inp[name]
        G = g[key]
        scale = max(np.max(np.abs(G)), 1e-12)
        for fi in rng.choice(base.size, size=n_coords, replace=False):
            idx = np.unravel_index(fi, base.shape)
            orig = base[idx]
            base[idx] = orig + h
            lp = float(np.sum(O.layer_split_gate_up(inp, cfg.k, cfg.scale)[0] * dY))
            base[idx] = orig - h
            lm = float(np.sum(O.layer_split_gate_up(inp, cfg.k, cfg.scale)[0] * dY))
            base[idx] = orig
            worst = max(worst, abs((lp - lm) / (2 * h) - G[idx]) / scale)
    return worst


def test_split_gate_up_gradients_match_finite_differences():
    assert check_split_fd() < 1e-6


def test_split_pin_catches_planted_mistake(monkeypatch):
    good = O.layer_split_gate_up

    def bad(inp, k, c):                     # gate adapter gradient scaled twice
        Y, g = good(inp, k, c)
        g["dA_g"] = g["dA_g"] * c
        return Y, g
    monkeypatch.setattr(O, "layer_split_gate_up", bad)
    assert check_split_fd(n_coords=6) > 1e-3
