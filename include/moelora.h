/*
 * moelora.h - C ABI of the MoE expert-MLP + Split-LoRA layer for NVIDIA B200 (sm_100a).
 *
 * The layer (forward and backward, expert weights W frozen):
 *   route   : per token t, pick the k largest of E router logits (ties go to the
 *             lower expert index) and weight them by a softmax over the k picked
 *             logits.  Source: "Accelerating Mixture-of-Experts Fine-Tuning"
 *             (ailinkdeeptech cookbook), section "The Dynamic Dispatch Bottleneck
 *             in Mixture-of-Experts Architectures", router equation.
 *   permute : group the P = T*k (token, slot) pairs into one contiguous segment
 *             per expert so every expert is one block of rows of a single grouped
 *             GEMM.  Source: Unsloth docs "Fine-tune MoE models 12x faster with
 *             Unsloth", section "What is torch._grouped_mm?".
 *   experts : SwiGLU expert with Split-LoRA on gate_up and down:
 *               GU = X W_gu + c (X A_gu) B_gu,  H = silu(GU[:, :n]) * GU[:, n:],
 *               Y  = H W_d  + c (H A_d)  B_d,   c = alpha / r,
 *             so no E x K x N adapter delta is ever formed.  Source: cookbook
 *             "Mathematical Formulation" section 2 (Split LoRA Associative
 *             Transformation); Unsloth docs sections "Faster LoRA MoE training"
 *             and "MoE LoRA changes things".
 *   combine : Y[t] = sum_j w[t,j] * Yp[pair (t,j)]  (router equation above).
 *   backward: dX and the adapter gradients dA_gu, dB_gu, dA_d, dB_d by the chain
 *             rule; W and the router are frozen (Unsloth docs, "Implementation
 *             details": only the m*r + r*n adapter parameters train, and the
 *             router is not fine-tuned).
 *
 * Conventions shared by every call
 *   - All tensors are dense, row-major, contiguous, in device memory unless a
 *     call says otherwise, with 16-byte aligned base pointers.
 *   - bf16 tensors are passed as moe_bf16_t (raw IEEE bfloat16 bits).
 *   - Index conventions: pair p = t*k + j; sorted position q in [0, P); the
 *     segment of expert e is rows [offsets[e], offsets[e+1]) of every "sorted"
 *     tensor, in ascending p inside the segment.
 *   - Expert weights are stored [E, K, N]: W_gu [E, m, 2n] (gate = columns
 *     [0, n), up = columns [n, 2n)), W_d [E, n, m]; adapters A [E, K, r] and
 *     B [E, r, N]: A_gu [E, m, r], B_gu [E, r, 2n], A_d [E, n, r], B_d [E, r, m].
 *   - The caller owns all memory; the library never allocates or frees device
 *     memory.  Scratch memory is the caller's workspace `ws` of `ws_bytes`
 *     (at least moe_workspace_bytes(), 256-byte aligned); calls that share one
 *     workspace must be ordered on one stream.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronises, except moe_get_device_error().
 *   - Arguments are checked on the host before any launch; a failed check
 *     launches nothing and returns the status.  Problems only the device can see
 *     (an expert id outside [0, E), a bounded wait that expired) set a device
 *     error word instead of trapping; read it with moe_get_device_error().
 *   - Supported shapes: 1 <= k <= 32, k <= E <= 1024; m and n multiples of 16,
 *     at least 16; r a multiple of 8 with 8 <= r <= 128; P = T*k < 2^31.
 *     T = 0 is valid and produces empty outputs (adapter gradients are zero).
 *     Other shapes return MOE_ERR_UNSUPPORTED.
 *   - Results are deterministic: no floating-point atomics; repeated calls with
 *     the same inputs give the same bits.
 */
#ifndef MOELORA_H_
#define MOELORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* NULL pointer, negative size, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,   /* shape outside the supported set above */
  MOE_ERR_WORKSPACE = 3,     /* ws_bytes smaller than moe_workspace_bytes() */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_INDEX = 5,  /* device-detected: expert id outside [0, E) */
  MOE_ERR_TIMEOUT = 6,       /* device-detected: a bounded wait expired */
  MOE_ERR_DEVICE_CHECK = 7   /* device-detected: moe_check_permutation() found a broken invariant */
} moe_status_t;

/* Layer shape.  scale is the LoRA scale c = alpha / r (the caller chooses it). */
typedef struct {
  int64_t T;   /* tokens */
  int32_t m;   /* hidden size */
  int32_t n;   /* expert intermediate size */
  int32_t E;   /* experts */
  int32_t k;   /* experts per token */
  int32_t r;   /* LoRA rank */
  float scale; /* c = alpha / r */
} moe_dims_t;

/* Bytes of workspace every call below needs for these dims (the maximum over
 * calls; one buffer of this size serves them all).  Returns 0 for dims that
 * are not supported. */
size_t moe_workspace_bytes(const moe_dims_t* dims);

/* Top-k routing.
 * logits   fp32 [T, E]  (device, read)
 * topk_ids int32 [T, k] (device, written): expert ids in descending logit order,
 *          equal logits ordered by ascending expert id.
 * topk_w   fp32 [T, k]  (device, written): exp(l_j - l_max) / sum over the k
 *          picked logits (the softmax over E restricted to the picked experts and
 *          renormalised to sum to one).
 * Errors: INVALID_ARG (NULL, T < 0), UNSUPPORTED (k, E out of range), CUDA. */
moe_status_t moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k,
                            int32_t* topk_ids, float* topk_w, void* stream);

/* Counting-sort permutation into per-expert segments (stable by pair index).
 * topk_ids     int32 [T, k] (device, read)
 * counts       int32 [E]    (written) pairs routed to each expert
 * offsets      int32 [E+1]  (written) exclusive prefix sum of counts, offsets[E] = P
 * sorted_pairs int32 [P]    (written) pair index p at sorted position q
 * pair_pos     int32 [P]    (written) sorted position of pair p (inverse of sorted_pairs)
 * ws, ws_bytes              scratch: (ceil(T*k / 512) * E + 32 * E + 1) int32
 *                           (per-chunk histograms, expert totals 128 bytes apart, one
 *                           counter); contents on entry do not matter
 * An id outside [0, E) sets MOE_ERR_DEVICE_INDEX in the device error word; that
 * pair is left out and the outputs are then incomplete.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
moe_status_t moe_permute(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                         int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                         int32_t* pair_pos, void* ws, size_t ws_bytes, void* stream);

/* moe_route_topk() and moe_permute() in one call, for the common case where the
 * permutation follows the routing directly: one cooperative kernel routes the tokens,
 * counts their pairs per expert, and after a grid barrier (its wait bounded) scans the
 * counts and scatters the pairs; a memset of the scratch comes first.  Same definitions
 * and outputs as the two calls (stable order,
 * ties to the lower expert index).
 * ws, ws_bytes: scratch of at least (ceil(T / floor(512 / k)) * E + 32 * E + 1) int32
 * (per-chunk histograms of whole-token chunks, expert totals, one counter);
 * moe_workspace_bytes() for any dims with this T, E, k is enough.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
moe_status_t moe_route_permute(const float* logits, int64_t T, int32_t E, int32_t k,
                               int32_t* topk_ids, float* topk_w, int32_t* counts,
                               int32_t* offsets, int32_t* sorted_pairs, int32_t* pair_pos,
                               void* ws, size_t ws_bytes, void* stream);

/* Debug check of a permutation, on the device (the stand-in for a sanitizer run, which
 * this library's test machines do not offer): every invariant moe_permute() promises.
 *   offsets[0] = 0, offsets[E] = P, offsets non-decreasing, counts[e] = offsets[e+1] -
 *   offsets[e]; for every sorted position q: p = sorted_pairs[q] is in [0, P),
 *   pair_pos[p] = q, q lies in the segment of expert topk_ids[p], and p is larger than
 *   the pair before it in the same segment (stable order).
 * Arguments as moe_permute() (all read).  A violation sets MOE_ERR_DEVICE_CHECK in the
 * device error word (read it with moe_get_device_error()); nothing is written otherwise.
 * The Python binding runs it after every permutation when the environment variable
 * MOE_CHECK is set.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
moe_status_t moe_check_permutation(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                                   const int32_t* counts, const int32_t* offsets,
                                   const int32_t* sorted_pairs, const int32_t* pair_pos,
                                   void* stream);

/* Forward of all experts over their segments (grouped GEMMs, one launch each):
 *   Y_sorted[q] = H[q] W_d[e] + c (H[q] A_d[e]) B_d[e],
 *   H[q]        = silu(GU[q, :n]) * GU[q, n:],
 *   GU[q]       = X[t] W_gu[e] + c (X[t] A_gu[e]) B_gu[e],   t = sorted_pairs[q] / k,
 * for every q in the segment of expert e.
 * Inputs (device, read): X bf16 [T, m]; sorted_pairs [P]; offsets [E+1]; the six
 *   weight tensors in the layouts above.
 * Outputs (device, written, bf16, sorted order):
 *   Y_sorted [P, m]; save_Xs [P, m] = X[sorted_pairs / k] (the expert-sorted input
 *   rows, the grouped GEMM's operand, kept for the backward as an autograd
 *   implementation keeps the permuted input); save_GU [P, 2n]; save_H [P, n];
 *   save_XA [P, r] = X A_gu (unscaled); save_HA [P, r] = H A_d (unscaled).  The
 *   save_* tensors are what moe_grouped_gemm_lora_bwd() needs.
 * Accumulation is fp32; every stored value is rounded once to bf16 (H from the
 * bf16-rounded GU).  The LoRA term multiplies bf16(c * X A) by B.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
moe_status_t moe_grouped_gemm_lora_fwd(
    const moe_dims_t* dims, const moe_bf16_t* X, const int32_t* sorted_pairs,
    const int32_t* offsets, const moe_bf16_t* W_gu, const moe_bf16_t* W_d,
    const moe_bf16_t* A_gu, const moe_bf16_t* B_gu, const moe_bf16_t* A_d,
    const moe_bf16_t* B_d, moe_bf16_t* Y_sorted, moe_bf16_t* save_Xs, moe_bf16_t* save_GU,
    moe_bf16_t* save_H, moe_bf16_t* save_XA, moe_bf16_t* save_HA, void* ws,
    size_t ws_bytes, void* stream);

/* Backward of all experts (W frozen) for upstream gradient dY:
 *   dy_q     = w[p] dY[t]                          (p = sorted_pairs[q], t = p / k)
 *   T1       = dy B_d^T,  dH = dy W_d^T + c T1 A_d^T
 *   dGU      = [dH * u * s * (1 + g (1 - s)),  dH * g * s],  s = sigmoid(g), [g|u] = GU
 *   T2       = dGU B_gu^T, dX_sorted = dGU W_gu^T + c T2 A_gu^T
 *   dA_d[e]  = c H_e^T T1_e,   dB_d[e]  = c HA_e^T dy_e
 *   dA_gu[e] = c X_e^T T2_e,   dB_gu[e] = c XA_e^T dGU_e
 * Inputs (device, read): dY bf16 [T, m]; topk_w fp32 [T, k]; sorted_pairs;
 *   offsets; the six weights; save_Xs, save_GU, save_H, save_XA, save_HA from the
 *   forward.
 * Outputs (device, written, bf16): dX_sorted [P, m] (sorted order; reduce with
 *   moe_unpermute_combine(topk_w = NULL)); dA_gu [E, m, r]; dB_gu [E, r, 2n];
 *   dA_d [E, n, r]; dB_d [E, r, m].  Experts with no rows get zero gradients.
 * Adapter gradients are reduced over rows in a fixed order (deterministic).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
moe_status_t moe_grouped_gemm_lora_bwd(
    const moe_dims_t* dims, const moe_bf16_t* dY, const float* topk_w,
    const int32_t* sorted_pairs, const int32_t* offsets,
    const moe_bf16_t* W_gu, const moe_bf16_t* W_d, const moe_bf16_t* A_gu,
    const moe_bf16_t* B_gu, const moe_bf16_t* A_d, const moe_bf16_t* B_d,
    const moe_bf16_t* save_Xs, const moe_bf16_t* save_GU, const moe_bf16_t* save_H,
    const moe_bf16_t* save_XA, const moe_bf16_t* save_HA, moe_bf16_t* dX_sorted,
    moe_bf16_t* dA_gu, moe_bf16_t* dB_gu, moe_bf16_t* dA_d, moe_bf16_t* dB_d, void* ws,
    size_t ws_bytes, void* stream);

/* Backward for full fine-tuning: everything moe_grouped_gemm_lora_bwd() computes,
 * plus the gradients of the expert weights themselves ("GPT-5.6-Terraに触れてみたよ",
 * section on full fine-tuning: the base weights W0 are trained instead of frozen;
 * "Fine-tune MoE models 12x faster with Unsloth", opening list: the kernels serve
 * full fine-tuning as well as LoRA):
 *   dW_gu[e] = X_e^T dGU_e     bf16 [E, m, 2n]
 *   dW_d[e]  = H_e^T dy_e      bf16 [E, n, m]
 * summed in fp32 over the rows of expert e (a contraction of P_e rows, P_e >= 0;
 * experts with no rows get zeros), rounded once.  dW_gu and dW_d are required.
 * dA_gu, dB_gu, dA_d, dB_d: all four given (computed as in the LoRA backward) or
 * all four NULL (adapter gradients skipped; pass B_gu = B_d = 0 for a layer
 * without adapters, whose rank-r terms then add exact zeros).  Other arguments,
 * outputs and errors as moe_grouped_gemm_lora_bwd(); each weight-gradient tile
 * sums its rows in one fixed order (deterministic). */
moe_status_t moe_grouped_gemm_full_bwd(
    const moe_dims_t* dims, const moe_bf16_t* dY, const float* topk_w,
    const int32_t* sorted_pairs, const int32_t* offsets,
    const moe_bf16_t* W_gu, const moe_bf16_t* W_d, const moe_bf16_t* A_gu,
    const moe_bf16_t* B_gu, const moe_bf16_t* A_d, const moe_bf16_t* B_d,
    const moe_bf16_t* save_Xs, const moe_bf16_t* save_GU, const moe_bf16_t* save_H,
    const moe_bf16_t* save_XA, const moe_bf16_t* save_HA, moe_bf16_t* dX_sorted,
    moe_bf16_t* dW_gu, moe_bf16_t* dW_d, moe_bf16_t* dA_gu, moe_bf16_t* dB_gu,
    moe_bf16_t* dA_d, moe_bf16_t* dB_d, void* ws, size_t ws_bytes, void* stream);

/* The same permutation as moe_permute(), for callers that cannot allocate device
 * memory: plug-ins hosted inside another framework that owns all device memory
 * and hands them no allocator, or code that must run with a fixed device-memory
 * footprint decided before it starts.  It takes no workspace; its scratch (the
 * per-chunk histograms) is a 2 MiB array built into the library (with 128 KiB more
 * for the expert totals and one counter), which every GPU that loads the library
 * holds until the process exits.  There is no
 * counterpart on the pages: this is an interface convenience.
 * Limit: ceil(T*k / 512) * E <= 524288 (e.g. T*k <= 2^21 pairs at E = 128);
 * larger problems return MOE_ERR_WORKSPACE before any launch.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture.  The address is kept per device and CUDA context, so a call
 * after a device reset (a new context) looks it up again; the array's contents do
 * not survive the reset.  All calls share the one array: calls that overlap on the
 * GPU (different streams, no ordering between them) race and must be avoided.
 * Arguments, outputs and errors otherwise as moe_permute(). */
moe_status_t moe_permute_noalloc(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                                 int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                                 int32_t* pair_pos, void* stream);

/* Weighted un-permute: Y[t] = sum_{j=0..k-1} w[t,j] * Y_sorted[pair_pos[t*k+j]],
 * summed in fp32 over ascending j and rounded once to bf16.  With topk_w = NULL
 * every weight is 1 (the dX reduction of the backward).
 * Inputs (device, read): Y_sorted bf16 [P, m]; topk_w fp32 [T, k] or NULL;
 *   pair_pos int32 [P].  Output (device, written): Y bf16 [T, m].
 * Errors: INVALID_ARG, UNSUPPORTED (m % 8), CUDA. */
moe_status_t moe_unpermute_combine(const moe_bf16_t* Y_sorted, const float* topk_w,
                                   const int32_t* pair_pos, int64_t T, int32_t k,
                                   int32_t m, moe_bf16_t* Y, void* stream);

/* Router backward, the step before the path once the logits come from x W_r
 * inside a model ("Accelerating Mixture-of-Experts Fine-Tuning", section "The
 * Dynamic Dispatch Bottleneck in Mixture-of-Experts Architectures": router
 * equation; Unsloth faster-moe docs, "Implementation details": the router stays
 * frozen but a gradient still flows into its input).  With Y[t] = sum_j
 * w[t,j] y_(t,j) and w the softmax over the k picked logits:
 *   dw[t,j]                = <dY[t], Y_sorted[pair_pos[t*k + j]]>   (fp32)
 *   dlogits[t, ids[t,j]]   = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i])
 *   dlogits[t, e]          = 0 for every expert e not picked for token t.
 * Inputs (device, read): dY bf16 [T, m]; Y_sorted bf16 [P, m] (the expert outputs
 *   of moe_grouped_gemm_lora_fwd); topk_ids int32 [T, k]; topk_w fp32 [T, k];
 *   pair_pos int32 [P].  Output (device, written): dlogits fp32 [T, E], every entry.
 * Supported: 1 <= k <= 32, k <= E <= 1024, m % 8 == 0; dY and Y_sorted 16-byte
 * aligned.  Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
moe_status_t moe_router_backward(const moe_bf16_t* dY, const moe_bf16_t* Y_sorted,
                                 const int32_t* topk_ids, const float* topk_w,
                                 const int32_t* pair_pos, int64_t T, int32_t k, int32_t E,
                                 int32_t m, float* dlogits, void* stream);

/* Self-test of the failure path (no counterpart on the pages: a check of this
 * library's own error handling).  Every wait of every kernel here is bounded: it
 * gives up after a wall-clock limit, sets MOE_ERR_TIMEOUT in the device error word
 * and lets its kernel return, so a lost arrival cannot hang the GPU.  This call
 * launches one single-thread kernel that makes that same bounded wait on a barrier
 * nothing arrives at, with the limit `limit_ns` (1 us to 1 s), and then writes
 * *done = 1 (device int32) as it returns (2 if the wait had not expired).  After it,
 * moe_get_device_error() returns MOE_ERR_TIMEOUT and the GPU stays usable.
 * Errors: INVALID_ARG (limit out of range, done NULL), CUDA. */
moe_status_t moe_selftest_bounded_wait(uint64_t limit_ns, int32_t* done, void* stream);

/* Synchronises `stream`, returns the device error word of the current device
 * (MOE_OK if no kernel reported a problem) and clears it. */
moe_status_t moe_get_device_error(void* stream);

/* Static description of a status code. */
const char* moe_status_string(moe_status_t status);

/* Kernel timing, a tracing aid (no counterpart on the pages).  While enabled,
 * every kernel the library launches is bracketed by two CUDA events recorded
 * on its stream (a few hundred nanoseconds of device time each); events come
 * from a host-side pool, no device memory is allocated.  Off by default.
 * Launches made while the stream is captured into a CUDA graph get event-record
 * nodes instead; moe_profile_read then reports the times of the graph's most
 * recent launch, so read after launching it (each capture holds its own events). */
void moe_profile_enable(int on);

/* Restricts the tracing to the kernel kinds named in `kinds`, a comma-separated
 * list of the names moe_profile_read reports (e.g. "gemm_gateup_fwd,lora_wgrad");
 * NULL or "" selects every kind (the default).  Returns the number of kinds
 * selected, or -1 (selection unchanged) if a name is unknown.  Tracing one kernel
 * kind keeps the event overhead out of the rest of a timed step. */
int moe_profile_select(const char* kinds);

/* Waits for the recorded events and reports, per kernel kind that ran since
 * the last read, its name (NUL-terminated, at most name_len bytes, row w of
 * `names`), its launch count and its summed device time in milliseconds.
 * Returns the number of kinds written (at most max_kinds) and clears the
 * records.  Any output pointer may be NULL. */
int moe_profile_read(int max_kinds, char* names, int name_len, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* MOELORA_H_ */
