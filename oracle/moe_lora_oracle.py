"""fp64 CPU oracle for the MoE expert-MLP layer with Split-LoRA (forward and backward).

TEST INFRASTRUCTURE.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
calls it, it never calls the CUDA library, and the two share no code: the only
thing both sides consume is the seeded input generator (`moe_inputs`).

Every function is plain NumPy float64 on bf16-rounded inputs, one expert
group at a time, with a library matmul as its only primitive.  No blocking,
fusion or reordering beyond what the definitions below state.

Sources (web pages on the method):
  [MoE12x]   Unsloth docs, "Fine-tune MoE models 12x faster with Unsloth"
             (unsloth.ai/docs, faster-moe; same text in its Japanese, German
             and French editions).
  [Cookbook] "Accelerating Mixture-of-Experts Fine-Tuning: Unsloth Faster MoE,
             Split LoRA, and Grouped GEMM" (ailinkdeeptech.com cookbook).
  [Terra]    "GPT-5.6-Terraに触れてみたよ" (bluecore.net blog post on Unsloth's
             training modes).

Readings taken where the pages are silent or inconsistent (each is listed in
the design notes): adapters A:[K,r], B:[r,N] with delta W = A B and scale
c = alpha/r; expert weights stored [E, K, N]; SwiGLU activation h = silu(g)*u
with gate = first n columns; renormalised top-k softmax with ties broken
toward the lower expert index; stable (ascending pair index) order inside an
expert segment; the router is frozen and its logits are an input.

Beyond the path, router_backward gives the gradient into the router logits
(for when the logits come from x W_r inside a model), layer_split_gate_up
the layer with separate gate and up adapters, and moe_weight_grads the
gradients of the expert weights themselves (full fine-tuning).

Pins (tests/test_oracle_pins.py): Split-LoRA equals the materialised
X(W + c A B); B = 0 gives the base MoE exactly; k = E with equal logits gives
the plain average of all experts; gradients match central finite differences
and an independent torch.autograd evaluation; routing and permutation match
brute force; the accounting helpers match the worked numbers the pages print.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "to64", "route_topk", "permute", "silu", "sigmoid",
    "expert_forward", "expert_forward_merged", "expert_backward",
    "unpermute_combine", "moe_forward", "moe_backward", "moe_forward_merged", "moe_forward_base",
    "token_forward", "token_backward_dx", "expert_lora_grads", "router_backward",
    "layer_split_gate_up", "moe_weight_grads", "expert_weight_grads",
]


def to64(x) -> np.ndarray:
    """Exact float64 copy of a torch tensor (bf16 / fp32) or array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Routing.  [Cookbook] "The Dynamic Dispatch Bottleneck in Mixture-of-Experts
# Architectures": y_t = sum over i in Top-k(Softmax(x_t W_r)) of s_{t,i} Expert_i(x_t).
# Reading: logits are given (frozen router); selection is by logit value,
# ties go to the lower expert index; the k selected probabilities are
# renormalised to sum to one (equivalently, a softmax over the selected logits).
# --------------------------------------------------------------------------
def route_topk(logits, k: int):
    """Return (ids int64 [T,k] in descending-logit order, weights fp64 [T,k])."""
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    # stable sort of -logit keeps equal logits in ascending index order
    order = np.argsort(-lg, axis=1, kind="stable")
    ids = order[:, :k].astype(np.int64)
    sel = np.take_along_axis(lg, ids, axis=1)
    z = np.exp(sel - sel[:, :1])          # sel[:, 0] is the row maximum
    w = z / z.sum(axis=1, keepdims=True)
    return ids, w


# --------------------------------------------------------------------------
# Permute into contiguous per-expert segments.  [MoE12x] "What is
# torch._grouped_mm?": the per-expert loop with a mask lookup per expert is
# replaced by one grouped launch over rows already grouped by expert.
# Reading: pair p = t*k + j; segment of expert e is [offsets[e], offsets[e+1]);
# inside a segment pairs keep ascending p.
# --------------------------------------------------------------------------
def permute(ids, E: int):
    """Return (counts [E], offsets [E+1], sorted_pairs [P], pair_pos [P]) as int64."""
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_pairs = np.argsort(flat, kind="stable").astype(np.int64)
    pair_pos = np.empty_like(sorted_pairs)
    pair_pos[sorted_pairs] = np.arange(flat.size, dtype=np.int64)
    return counts, offsets, sorted_pairs, pair_pos


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    return z * sigmoid(z)


# --------------------------------------------------------------------------
# One expert on a block of rows.  [Cookbook] "Mathematical Formulation", §2
# (Split LoRA Associative Transformation): Y = X W + (alpha/r) (X A) B, with the
# low-rank intermediate X A of shape [s, r]; [MoE12x] "MoE LoRA changes things":
# LoRA on gate/up (fused as gate_up_proj) and on down_proj.
# --------------------------------------------------------------------------
def expert_forward(x, W_gu, A_gu, B_gu, W_d, A_d, B_d, c: float):
    """Split-LoRA SwiGLU expert on rows x [R, m] (all fp64 arrays)."""
    n = W_gu.shape[1] // 2
    xa = x @ A_gu                                   # [R, r]
    gu = x @ W_gu + c * (xa @ B_gu)                 # [R, 2n]
    g, u = gu[:, :n], gu[:, n:]
    h = silu(g) * u                                 # [R, n]
    ha = h @ A_d                                    # [R, r]
    y = h @ W_d + c * (ha @ B_d)                    # [R, m]
    return {"xa": xa, "gu": gu, "h": h, "ha": ha, "y": y}


def expert_forward_merged(x, W_gu, A_gu, B_gu, W_d, A_d, B_d, c: float):
    """The PEFT route: materialise W' = W + c A B, then one product.

    [Cookbook] §1 (Standard PEFT Materialization Overhead) and [MoE12x]
    "Faster LoRA MoE training": merging forms the full per-expert delta.
    Used only to pin the Split-LoRA form (same result up to rounding order).
    """
    n = W_gu.shape[1] // 2
    Wgu_m = W_gu + c * (A_gu @ B_gu)
    Wd_m = W_d + c * (A_d @ B_d)
    gu = x @ Wgu_m
    h = silu(gu[:, :n]) * gu[:, n:]
    return h @ Wd_m


def expert_backward(x, fwd, dy, W_gu, A_gu, B_gu, W_d, A_d, B_d, c: float):
    """Chain rule through one expert with W frozen, for rows x [R, m].

    dy [R, m] is the routing-weighted upstream gradient w * dY[t] of each row.
    Returns the input gradient rows and this expert's adapter gradients.
    [MoE12x] "Implementation details": only the m*r + r*n adapter parameters
    train; [MoE12x] "Faster LoRA MoE training": gradients are unchanged by the
    reordering, so they follow from the plain chain rule below.
    """
    n = W_gu.shape[1] // 2
    g, u = fwd["gu"][:, :n], fwd["gu"][:, n:]
    h, ha, xa = fwd["h"], fwd["ha"], fwd["xa"]
    # down projection: y = h W_d + c (h A_d) B_d
    t1 = dy @ B_d.T                                  # [R, r]
    dh = dy @ W_d.T + c * (t1 @ A_d.T)               # [R, n]
    dA_d = c * (h.T @ t1)                            # [n, r]
    dB_d = c * (ha.T @ dy)                           # [r, m]
    # SwiGLU: h = g sigmoid(g) u
    s = sigmoid(g)
    dg = dh * u * s * (1.0 + g * (1.0 - s))
    du = dh * g * s
    dgu = np.concatenate([dg, du], axis=1)           # [R, 2n]
    # gate_up projection: gu = x W_gu + c (x A_gu) B_gu
    t2 = dgu @ B_gu.T                                # [R, r]
    dx = dgu @ W_gu.T + c * (t2 @ A_gu.T)            # [R, m]
    dA_gu = c * (x.T @ t2)                           # [m, r]
    dB_gu = c * (xa.T @ dgu)                         # [r, 2n]
    return {"dx": dx, "dgu": dgu, "t1": t1, "t2": t2, "dh": dh,
            "dA_gu": dA_gu, "dB_gu": dB_gu, "dA_d": dA_d, "dB_d": dB_d}


def _weights64(inp):
    return {k: to64(inp[k]) for k in ("W_gu", "W_d", "A_gu", "B_gu", "A_d", "B_d")}


def _route_and_permute(inp, k):
    E = inp["W_gu"].shape[0]
    ids, w = route_topk(to64(inp["logits"]).astype(np.float32), k)
    counts, offsets, sorted_pairs, pair_pos = permute(ids, E)
    return ids, w, counts, offsets, sorted_pairs, pair_pos


def unpermute_combine(yp, w, pair_pos, k: int):
    """Un-permute: Y[t] = sum_j w[t,j] * yp[pair_pos[t*k + j]], j ascending; w None
    means every weight is 1 (the sum of dX over a token's pairs in the backward).
    The output of a token is its experts' outputs mixed by the routing weights
    ([Cookbook] "The Dynamic Dispatch Bottleneck in Mixture-of-Experts
    Architectures"; [MoE12x] "What is torch._grouped_mm?").
    """
    yp = np.asarray(yp, dtype=np.float64)
    T = pair_pos.shape[0] // k
    Y = np.zeros((T, yp.shape[1]))
    for j in range(k):
        rows = yp[pair_pos[np.arange(T) * k + j]]
        Y += rows if w is None else np.asarray(w, dtype=np.float64)[:, j:j + 1] * rows
    return Y


def moe_forward(inp, k: int, c: float, keep=True):
    """Whole layer forward: route, permute, experts, weighted combine.

    Y[t] = sum_j w[t,j] * y_(t,j), summed over j ascending.
    Returns (Y [T, m] fp64, aux dict with routing and sorted-order intermediates).
    """
    X = to64(inp["X"])
    T, m = X.shape
    W = _weights64(inp)
    E = W["W_gu"].shape[0]
    n = W["W_gu"].shape[2] // 2
    r = W["A_gu"].shape[2]
    ids, w, counts, offsets, sorted_pairs, pair_pos = _route_and_permute(inp, k)
    P = T * k
    Yp = np.zeros((P, m))
    aux = {"ids": ids, "w": w, "counts": counts, "offsets": offsets,
           "sorted_pairs": sorted_pairs, "pair_pos": pair_pos}
    if keep:
        for name, width in (("gu", 2 * n), ("h", n), ("xa", r), ("ha", r)):
            aux[name] = np.zeros((P, width))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        tok = sorted_pairs[lo:hi] // k
        f = expert_forward(X[tok], W["W_gu"][e], W["A_gu"][e], W["B_gu"][e],
                           W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
        Yp[lo:hi] = f["y"]
        if keep:
            for name in ("gu", "h", "xa", "ha"):
                aux[name][lo:hi] = f[name]
    aux["yp"] = Yp
    return unpermute_combine(Yp, w, pair_pos, k), aux


def moe_backward(inp, aux, dY, k: int, c: float):
    """Whole layer backward with W and the router frozen.

    Returns dX [T, m], dA_gu [E,m,r], dB_gu [E,r,2n], dA_d [E,n,r], dB_d [E,r,m]
    and sorted-order intermediates (dgu, t1, t2, dxp).
    """
    X = to64(inp["X"])
    dY = to64(dY)
    T, m = X.shape
    W = _weights64(inp)
    E, _, n2 = W["W_gu"].shape
    n = n2 // 2
    r = W["A_gu"].shape[2]
    w, offsets = aux["w"], aux["offsets"]
    sorted_pairs, pair_pos = aux["sorted_pairs"], aux["pair_pos"]
    P = T * k
    out = {"dA_gu": np.zeros((E, m, r)), "dB_gu": np.zeros((E, r, 2 * n)),
           "dA_d": np.zeros((E, n, r)), "dB_d": np.zeros((E, r, m)),
           "dgu": np.zeros((P, 2 * n)), "t1": np.zeros((P, r)),
           "t2": np.zeros((P, r)), "dxp": np.zeros((P, m))}
    wflat = w.reshape(-1)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        pairs = sorted_pairs[lo:hi]
        tok = pairs // k
        x = X[tok]
        if "gu" in aux:
            fwd = {name: aux[name][lo:hi] for name in ("gu", "h", "xa", "ha")}
        else:
            fwd = expert_forward(x, W["W_gu"][e], W["A_gu"][e], W["B_gu"][e],
                                 W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
        dy = wflat[pairs][:, None] * dY[tok]
        b = expert_backward(x, fwd, dy, W["W_gu"][e], W["A_gu"][e], W["B_gu"][e],
                            W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
        for name in ("dA_gu", "dB_gu", "dA_d", "dB_d"):
            out[name][e] = b[name]
        out["dgu"][lo:hi] = b["dgu"]
        out["t1"][lo:hi] = b["t1"]
        out["t2"][lo:hi] = b["t2"]
        out["dxp"][lo:hi] = b["dx"]
    out["dX"] = unpermute_combine(out["dxp"], None, pair_pos, k)
    return out


def moe_forward_merged(inp, k: int, c: float):
    """Layer forward with materialised adapters (PEFT route); for the pins."""
    X = to64(inp["X"])
    T, m = X.shape
    W = _weights64(inp)
    E = W["W_gu"].shape[0]
    ids, w, counts, offsets, sorted_pairs, pair_pos = _route_and_permute(inp, k)
    Yp = np.zeros((T * k, m))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        tok = sorted_pairs[lo:hi] // k
        Yp[lo:hi] = expert_forward_merged(X[tok], W["W_gu"][e], W["A_gu"][e], W["B_gu"][e],
                                          W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
    Y = np.zeros((T, m))
    for j in range(k):
        Y += w[:, j:j + 1] * Yp[pair_pos[np.arange(T) * k + j]]
    return Y


def moe_forward_base(inp, k: int):
    """Layer forward with no adapters at all: the base MoE the pages start from."""
    X = to64(inp["X"])
    T, m = X.shape
    W_gu, W_d = to64(inp["W_gu"]), to64(inp["W_d"])
    E, _, n2 = W_gu.shape
    n = n2 // 2
    ids, w, counts, offsets, sorted_pairs, pair_pos = _route_and_permute(inp, k)
    Yp = np.zeros((T * k, m))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        x = X[sorted_pairs[lo:hi] // k]
        gu = x @ W_gu[e]
        Yp[lo:hi] = (silu(gu[:, :n]) * gu[:, n:]) @ W_d[e]
    Y = np.zeros((T, m))
    for j in range(k):
        Y += w[:, j:j + 1] * Yp[pair_pos[np.arange(T) * k + j]]
    return Y


# --------------------------------------------------------------------------
# Per-token and per-expert evaluations, for sampled parity at sizes where the
# whole-layer oracle is too slow.  Y and dX rows depend only on their own
# token; adapter gradients depend only on their own expert's rows.
# --------------------------------------------------------------------------
def token_forward(inp, t: int, k: int, c: float, W=None):
    """Y[t] alone (fp64 [m]) from the token's own routing."""
    W = W if W is not None else _weights64(inp)
    x = to64(inp["X"][t:t + 1])
    ids, w = route_topk(to64(inp["logits"][t:t + 1]).astype(np.float32), k)
    y = np.zeros(x.shape[1])
    for j in range(k):
        e = int(ids[0, j])
        f = expert_forward(x, W["W_gu"][e], W["A_gu"][e], W["B_gu"][e],
                           W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
        y += w[0, j] * f["y"][0]
    return y


def token_backward_dx(inp, t: int, k: int, c: float, W=None):
    """dX[t] alone (fp64 [m])."""
    W = W if W is not None else _weights64(inp)
    x = to64(inp["X"][t:t + 1])
    dyt = to64(inp["dY"][t:t + 1])
    ids, w = route_topk(to64(inp["logits"][t:t + 1]).astype(np.float32), k)
    dx = np.zeros(x.shape[1])
    for j in range(k):
        e = int(ids[0, j])
        args = (W["W_gu"][e], W["A_gu"][e], W["B_gu"][e], W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
        f = expert_forward(x, *args)
        b = expert_backward(x, f, w[0, j] * dyt, *args)
        dx += b["dx"][0]
    return dx


def expert_lora_grads(inp, e: int, k: int, c: float, ids=None, w=None, W=None):
    """Adapter gradients of expert e alone: (dA_gu, dB_gu, dA_d, dB_d)."""
    W = W if W is not None else _weights64(inp)
    if ids is None:
        ids, w = route_topk(to64(inp["logits"]).astype(np.float32), k)
    flat = ids.reshape(-1)
    pairs = np.nonzero(flat == e)[0]            # ascending pair index
    m = W["W_gu"].shape[1]
    n = W["W_gu"].shape[2] // 2
    r = W["A_gu"].shape[2]
    if pairs.size == 0:
        return (np.zeros((m, r)), np.zeros((r, 2 * n)), np.zeros((n, r)), np.zeros((r, m)))
    tok = pairs // k
    x = to64(inp["X"][tok])
    dy = w.reshape(-1)[pairs][:, None] * to64(inp["dY"][tok])
    args = (W["W_gu"][e], W["A_gu"][e], W["B_gu"][e], W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
    f = expert_forward(x, *args)
    b = expert_backward(x, f, dy, *args)
    return b["dA_gu"], b["dB_gu"], b["dA_d"], b["dB_d"]


# --------------------------------------------------------------------------
# Router backward: the step before the path once the logits come from x W_r
# inside a model ([Cookbook] "The Dynamic Dispatch Bottleneck in
# Mixture-of-Experts Architectures", router equation; [MoE12x] "Implementation
# details": the router weights stay frozen, a gradient still flows into x).
# Y[t] = sum_j w[t,j] y_(t,j), so dL/dw[t,j] = <dY[t], y_(t,j)>.  The weights are
# a softmax over the k picked logits, so
#     dL/dl[t, ids[t,j]] = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i]),
# and logits that were not picked get zero (the selection is piecewise constant).
# --------------------------------------------------------------------------
def router_backward(dY, yp, ids, w, pair_pos, E: int):
    """Return (dlogits fp64 [T, E], dw fp64 [T, k]); yp = expert outputs in sorted order."""
    dY = to64(dY)
    yp = to64(yp)
    ids = np.asarray(ids, dtype=np.int64)
    w = np.asarray(w, dtype=np.float64)
    T, k = ids.shape
    pos = np.asarray(pair_pos, dtype=np.int64).reshape(T, k)
    dw = np.zeros((T, k))
    for j in range(k):
        dw[:, j] = np.sum(dY * yp[pos[:, j]], axis=1)
    s = np.sum(w * dw, axis=1, keepdims=True)
    dlogits = np.zeros((T, E))
    np.put_along_axis(dlogits, ids, w * (dw - s), axis=1)
    return dlogits, dw


# --------------------------------------------------------------------------
# Adapter variant: separate gate and up adapters ([MoE12x] "MoE LoRA changes
# things": LoRA targets gate, up and down projections; the fused gate_up weight
# then carries two adapters).  Per expert
#     g = x W_g + c (x A_g) B_g,   u = x W_u + c (x A_u) B_u,   W_gu = [W_g | W_u],
# the SwiGLU and the down projection as above.  Written out on its own (not via
# the fused adapter) so that it pins the rank-2r block packing the library uses.
# --------------------------------------------------------------------------
def layer_split_gate_up(inp, k: int, c: float):
    """Forward and backward of the layer with separate gate/up adapters.

    inp holds X, logits, dY, W_gu, W_d, A_d, B_d and A_g, B_g, A_u, B_u
    ([E, m, r], [E, r, n] each).  Returns (Y [T, m], grads: dX, dA_g, dB_g, dA_u,
    dB_u, dA_d, dB_d).
    """
    X = to64(inp["X"])
    dY = to64(inp["dY"])
    T, m = X.shape
    Wgu, Wd = to64(inp["W_gu"]), to64(inp["W_d"])
    Ag, Bg, Au, Bu = (to64(inp[name]) for name in ("A_g", "B_g", "A_u", "B_u"))
    Ad, Bd = to64(inp["A_d"]), to64(inp["B_d"])
    E = Wgu.shape[0]
    n = Wgu.shape[2] // 2
    r = Ag.shape[2]
    ids, w, counts, offsets, sorted_pairs, pair_pos = _route_and_permute(inp, k)
    P = T * k
    yp = np.zeros((P, m))
    dxp = np.zeros((P, m))
    gr = {"dA_g": np.zeros((E, m, r)), "dB_g": np.zeros((E, r, n)),
          "dA_u": np.zeros((E, m, r)), "dB_u": np.zeros((E, r, n)),
          "dA_d": np.zeros((E, n, r)), "dB_d": np.zeros((E, r, m))}
    wflat = w.reshape(-1)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        pairs = sorted_pairs[lo:hi]
        x = X[pairs // k]
        xg, xu = x @ Ag[e], x @ Au[e]
        g = x @ Wgu[e][:, :n] + c * (xg @ Bg[e])
        u = x @ Wgu[e][:, n:] + c * (xu @ Bu[e])
        h = silu(g) * u
        ha = h @ Ad[e]
        yp[lo:hi] = h @ Wd[e] + c * (ha @ Bd[e])
        dy = wflat[pairs][:, None] * dY[pairs // k]
        t1 = dy @ Bd[e].T
        dh = dy @ Wd[e].T + c * (t1 @ Ad[e].T)
        gr["dA_d"][e] = c * (h.T @ t1)
        gr["dB_d"][e] = c * (ha.T @ dy)
        s = sigmoid(g)
        dg = dh * u * s * (1.0 + g * (1.0 - s))
        du = dh * g * s
        tg, tu = dg @ Bg[e].T, du @ Bu[e].T
        dxp[lo:hi] = dg @ Wgu[e][:, :n].T + du @ Wgu[e][:, n:].T + c * (tg @ Ag[e].T + tu @ Au[e].T)
        gr["dA_g"][e] = c * (x.T @ tg)
        gr["dB_g"][e] = c * (xg.T @ dg)
        gr["dA_u"][e] = c * (x.T @ tu)
        gr["dB_u"][e] = c * (xu.T @ du)
    Y = np.zeros((T, m))
    dX = np.zeros((T, m))
    for j in range(k):
        sel = pair_pos[np.arange(T) * k + j]
        Y += w[:, j:j + 1] * yp[sel]
        dX += dxp[sel]
    gr["dX"] = dX
    return Y, gr


# --------------------------------------------------------------------------
# Full fine-tuning: gradients of the expert weights themselves.  [Terra],
# section "フルファインチューニングもできるが、別物として考える" (full fine-tuning
# is possible but a different thing): it trains the base weights W0 instead of
# freezing them as LoRA does; [MoE12x] opening list: the kernels serve full
# fine-tuning as well as LoRA.  The loss sees W_gu only through x W_gu and W_d
# only through h W_d, so for expert e over its rows (any number, zero included)
#     dW_gu[e] = X_e^T dGU_e        [m, 2n]
#     dW_d[e]  = H_e^T dy_e         [n, m],   dy = w * dY[t]
# with dGU the SwiGLU-backward rows of moe_backward and H the forward's.
def moe_weight_grads(inp, aux, bwd, dY, k: int):
    """(dW_gu [E, m, 2n], dW_d [E, n, m]) from the forward's aux (keep=True) and
    moe_backward's output; experts with no rows get zeros."""
    X = to64(inp["X"])
    dY = to64(dY)
    E, m, n2 = inp["W_gu"].shape
    n = n2 // 2
    offsets, sorted_pairs = aux["offsets"], aux["sorted_pairs"]
    wflat = aux["w"].reshape(-1)
    dW_gu = np.zeros((E, m, n2))
    dW_d = np.zeros((E, n, m))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        pairs = sorted_pairs[lo:hi]
        tok = pairs // k
        dW_gu[e] = X[tok].T @ bwd["dgu"][lo:hi]
        dW_d[e] = aux["h"][lo:hi].T @ (wflat[pairs][:, None] * dY[tok])
    return dW_gu, dW_d


def expert_weight_grads(inp, e: int, k: int, c: float, ids=None, w=None, W=None):
    """(dW_gu[e], dW_d[e]) of expert e alone, from its rows' forward and backward."""
    W = W if W is not None else _weights64(inp)
    if ids is None:
        ids, w = route_topk(to64(inp["logits"]).astype(np.float32), k)
    pairs = np.nonzero(ids.reshape(-1) == e)[0]            # ascending pair index
    m = W["W_gu"].shape[1]
    n = W["W_gu"].shape[2] // 2
    if pairs.size == 0:
        return np.zeros((m, 2 * n)), np.zeros((n, m))
    tok = pairs // k
    x = to64(inp["X"][tok])
    dy = w.reshape(-1)[pairs][:, None] * to64(inp["dY"][tok])
    args = (W["W_gu"][e], W["A_gu"][e], W["B_gu"][e], W["W_d"][e], W["A_d"][e], W["B_d"][e], c)
    f = expert_forward(x, *args)
    b = expert_backward(x, f, dy, *args)
    return x.T @ b["dgu"], f["h"].T @ dy
