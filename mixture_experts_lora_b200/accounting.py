"""FLOP, byte and parameter accounting for the MoE + Split-LoRA layer.

Pure arithmetic on shapes (no tensors).  The benchmark uses these figures as
the algorithmic work of a step; the tests pin them to the worked numbers the
pages print (tests/golden/worked_numbers.json).

Notation: T tokens, hidden m, expert intermediate n, E experts, top-k, rank r,
P = T*k routed (token, expert) pairs.  bf16 = 2 bytes.
"""
from __future__ import annotations


def pairs(T: int, k: int) -> int:
    return T * k


# ---- FLOPs -----------------------------------------------------------------
def flops_forward(T, m, n, k, r) -> int:
    """Base SwiGLU expert GEMMs 2P*m*2n + 2P*n*m, plus Split-LoRA x@A, (xA)@B on
    gate_up (2P*r*(m+2n)) and down (2P*r*(n+m)).  Elementwise work not counted."""
    P = pairs(T, k)
    return 6 * P * m * n + 2 * P * r * (2 * m + 3 * n)


def flops_backward(T, m, n, k, r) -> int:
    """dX path (2P*m*n + 4P*m*n) plus the LoRA input-gradient and adapter-gradient
    products; W is frozen so no dW."""
    P = pairs(T, k)
    return 6 * P * m * n + 4 * P * r * (2 * m + 3 * n)


def flops_step(T, m, n, k, r) -> int:
    return flops_forward(T, m, n, k, r) + flops_backward(T, m, n, k, r)


def flops_gemm_gate_up_fwd(T, m, n, k, r) -> int:
    P = pairs(T, k)
    return 2 * P * m * 2 * n + 2 * P * r * (m + 2 * n)


def flops_gemm_down_fwd(T, m, n, k, r) -> int:
    P = pairs(T, k)
    return 2 * P * n * m + 2 * P * r * (n + m)


def flops_gemm_down_bwd(T, m, n, k, r) -> int:
    """dH = dy W_d^T + c (dy B_d^T) A_d^T."""
    P = pairs(T, k)
    return 2 * P * m * n + 2 * P * r * (m + n)


def flops_gemm_gate_up_bwd(T, m, n, k, r) -> int:
    """dXp = dGU W_gu^T + c (dGU B_gu^T) A_gu^T."""
    P = pairs(T, k)
    return 2 * P * 2 * n * m + 2 * P * r * (2 * n + m)


def flops_lora_wgrad(T, m, n, k, r) -> int:
    """dA_d, dB_d, dA_gu, dB_gu: 2P*r*(n + m + m + 2n)."""
    P = pairs(T, k)
    return 2 * P * r * (2 * m + 3 * n)


# ---- bytes (algorithmic: each operand once) ---------------------------------
def bytes_route(T, E, k) -> int:
    return T * E * 4 + T * k * 8


def bytes_permute(T, E, k) -> int:
    P = pairs(T, k)
    return P * 4 + (2 * E + 1) * 4 + 2 * P * 4


def bytes_combine(T, m, k) -> int:
    P = pairs(T, k)
    return P * m * 2 + T * k * 8 + T * m * 2


def bytes_gather(T, m, k) -> int:
    P = pairs(T, k)
    return T * m * 2 + P * 4 + P * m * 2


def bytes_expert_weights(E, m, n) -> int:
    """W_gu + W_d, bf16."""
    return E * (m * 2 * n + n * m) * 2


# ---- parameter and memory counts the pages work through ---------------------
def lora_params_per_projection(m, n, r) -> int:
    """Adapter parameters of one (m, n) projection: m*r + r*n."""
    return r * (m + n)


def lora_fraction_of_projection(m, n, r) -> float:
    return lora_params_per_projection(m, n, r) / (m * n)


def peft_delta_elements(E, m, n) -> int:
    """Elements of the materialised per-expert delta across all experts: E*m*n."""
    return E * m * n


def memory_crossover_tokens_split_vs_merge(E, m, n, k) -> float:
    """Split LoRA holds k*s*n activation elements versus E*m*n for the merged
    delta, so it is smaller while s < E*m*n / (k*n) = E*m/k."""
    return E * m * n / (k * n)


def memory_crossover_tokens_lowrank(E, m, n, k, r) -> float:
    """Same comparison counting only the rank-r intermediate k*s*r: s < E*m*n/(k*r)."""
    return E * m * n / (k * r)


def compute_crossover_tokens(E, m, n, k, r=None) -> float:
    """Token count where the merged route's one-off cost E*(2mnr + mn) equals the
    Split route's extra 2k*s*r*(m+n): s = E*m*n/(k*(m+n)) * (1 + 1/(2r))."""
    base = E * m * n / (k * (m + n))
    return base if r is None else base * (1.0 + 1.0 / (2 * r))


def bandwidth_speedup_estimate(E, m, n, k, s) -> float:
    """Rough traffic ratio E*m*n / (k*s*(m+n))."""
    return E * m * n / (k * s * (m + n))
