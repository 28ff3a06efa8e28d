// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moelora.h"

namespace moe {

struct TileInfo;
struct TableBuild;

// Launch with programmatic stream serialization (the kernel calls pdl_begin() before
// touching global memory; see common.cuh), plus an optional cluster size.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- kernel timing (profile.cu): while enabled, each launch is bracketed by
// CUDA events on its stream and attributed to one of these kinds.
enum KernelKind : int {
  K_ROUTE = 0, K_PERM_HIST, K_PERM_SCATTER,
  K_GEMM_GATEUP_FWD, K_GEMM_DOWN_FWD, K_GEMM_DOWN_BWD, K_GEMM_GATEUP_BWD, K_WGRAD,
  K_COMBINE, K_MEMSET, K_RANK_XA, K_RANK_HA, K_RANK_T1, K_RANK_T2,
  K_ROUTER_BWD, K_GEMM_DW_GU, K_GEMM_DW_D, K_NUM_KINDS
};
extern const char* const kKernelNames[K_NUM_KINDS];
bool prof_enabled();
bool prof_traced(int kind);   // enabled and the kind is selected
void* prof_begin(int kind, cudaStream_t s);   // returns a record token (or nullptr)
void prof_end(void* token, cudaStream_t s);

struct ProfScope {
  void* tok;
  cudaStream_t s;
  ProfScope(int kind, cudaStream_t st) : tok(prof_traced(kind) ? prof_begin(kind, st) : nullptr), s(st) {}
  ~ProfScope() { if (tok) prof_end(tok, s); }
};

// Device address of the status word of the current device (api.cu), or nullptr.
int* moe_status_word();
// The current CUDA context (a CUcontext), or nullptr: caches of device addresses key
// on it, so that a device reset or a new primary context looks them up again.
void* current_context();

// ---- SIMT kernels (simt_kernels.cu)
cudaError_t launch_route_topk(const float* logits, int64_t T, int E, int k, int32_t* ids,
                              float* w, int* err, cudaStream_t s);
// Counting-sort scratch: per-chunk histograms [n_chunks][E], expert totals (one per
// kTotStride ints) and an arrival counter (the last block of the histogram launch is the one that scans).
constexpr int kPermuteChunk = 512;
constexpr int kTotStride = 32;            // ints between two experts' totals (128 bytes)
inline size_t permute_scratch_ints(int64_t n_chunks, int E) {
  return (size_t)n_chunks * E + (size_t)E * kTotStride + 1;
}
// One block per chunk of kPermuteChunk pairs; scratch holds
// permute_scratch_ints(ceil(P / kPermuteChunk), E) ints (the call zeroes what it needs).
cudaError_t launch_permute(const int32_t* ids, int64_t P, int E, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_pairs, int32_t* pair_pos,
                           int32_t* scratch, int* err, cudaStream_t s);
// Routing and the counting sort in one cooperative launch (after a memset of the
// scratch): chunks of route_tokens_per_chunk(k) tokens (their k pairs each); scratch
// holds permute_scratch_ints(ceil(T / route_tokens_per_chunk(k)), E) ints.
int route_tokens_per_chunk(int k);
cudaError_t launch_route_permute(const float* logits, int64_t T, int E, int k, int32_t* ids,
                                 float* w, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                                 int32_t* pair_pos, int32_t* scratch, cudaStream_t s);
// dlogits [T, E] fp32 = router backward (see simt_kernels.cu); m % 8 == 0
cudaError_t launch_router_backward(const uint16_t* dY, const uint16_t* ys, const int32_t* ids,
                                   const float* w, const int32_t* pos, int64_t T, int k, int E,
                                   int m, float* dlogits, cudaStream_t s);
// Debug check of moe_permute()'s invariants; sets MOE_ERR_DEVICE_CHECK on a violation.
cudaError_t launch_check_permutation(const int32_t* ids, int64_t P, int E, const int32_t* counts,
                                     const int32_t* offsets, const int32_t* sorted_pairs,
                                     const int32_t* pair_pos, int* err, cudaStream_t s);
cudaError_t launch_combine(const uint16_t* ysorted, const float* w, const int32_t* pair_pos,
                           int64_t T, int k, int m, uint16_t* y, cudaStream_t s);
cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t s);

// ---- tcgen05 GEMMs (gemm_*.cu), rank-r products (rank_launch.cu), adapter and
// expert-weight gradients (wgrad_launch.cu)
struct LayerPtrs {
  const uint16_t* W_gu;   // [E, m, 2n]
  const uint16_t* W_d;    // [E, n, m]
  const uint16_t* A_gu;   // [E, m, r]
  const uint16_t* B_gu;   // [E, r, 2n]
  const uint16_t* A_d;    // [E, n, r]
  const uint16_t* B_d;    // [E, r, m]
};

struct GemmShape {
  int64_t P;
  int m, n, E, r, rp;         // rp: r rounded up to 16, 32, 64 or 128
  float scale;
  int max_row_tiles;          // 128-row tiles (rank-r kernels)
  const TileInfo* tiles;
  const int* n_row_tiles;
  int max_gchunks;            // token chunks of at most 256 rows (grouped GEMMs)
  const TileInfo* gchunks;
  const int* n_gchunks;
  int* err;
  int num_sms;
};

// Grouped GEMMs (features on M, expert tokens on N, CTA pairs), sorted token order.
// GU, H = SwiGLU(Xs W_gu + XAc B_gu)   (XAc = bf16(c Xs A_gu))
cudaError_t launch_gemm_gateup_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* Xs,
                                   const uint16_t* XAc, uint16_t* GU, uint16_t* H, cudaStream_t s);
// Yp = H W_d + HAc B_d
cudaError_t launch_gemm_down_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* H,
                                 const uint16_t* HAc, uint16_t* Yp, cudaStream_t s);
// dH = dy W_d^T + T1c A_d^T
cudaError_t launch_gemm_down_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dys,
                                 const uint16_t* T1c, uint16_t* dH, cudaStream_t s);
// dXp = dGU W_gu^T + T2c A_gu^T
cudaError_t launch_gemm_gateup_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dGU,
                                   const uint16_t* T2c, uint16_t* dXp, cudaStream_t s);

// Rank-r products LR = Rows L[e] (rank_r.cuh); every variant writes out_save [P, ld_save]
// (first r_save columns, unscaled) and out_c = bf16(scale LR) [P, rp].
// Gathered rows s_q src[sorted_pairs[q] / k] of K columns (s_q = w[pair] if w is
// given), written to rows_out [P, K]; L [E, K, r] (l_mn) or [E, r, K].
cudaError_t launch_rank_gathered(int kind, const GemmShape& g, const uint16_t* src, int K,
                                 const int32_t* sorted_pairs, int k, const float* w,
                                 uint16_t* rows_out, const uint16_t* L, bool l_mn,
                                 uint16_t* out_save, int ld_save, int r_save, uint16_t* out_c,
                                 const TableBuild* tb, cudaStream_t s);
// Sorted rows [P, K].
cudaError_t launch_rank_sorted(int kind, const GemmShape& g, const uint16_t* rows, int K,
                               const uint16_t* L, bool l_mn, uint16_t* out_save, int ld_save,
                               int r_save, uint16_t* out_c, cudaStream_t s);
// The SwiGLU backward dGU [P, 2n] of dH [P, n] and GU [P, 2n], written out, with
// T2 = dGU B_gu^T.
cudaError_t launch_rank_dswiglu(const GemmShape& g, const uint16_t* dH, const uint16_t* GU,
                                const uint16_t* B_gu, uint16_t* dGU, uint16_t* out_save,
                                int ld_save, int r_save, uint16_t* out_c, cudaStream_t s);

// One adapter-gradient problem G_e = Big_e^T Small_e (see lora_wgrad.cuh):
// out = scale * G per expert, out [E, D, r] or (transpose) [E, r, D].
struct WgradJob {
  const uint16_t* big;   // [P, D] sorted rows
  int D;
  const uint16_t* small; // [P, ld_small]
  int ld_small;
  bool transpose;
  uint16_t* out;
  float* partial;        // [max_chunks, D, rp] fp32 partials of multi-chunk experts
  int* counters;         // [E, ceil(D / 256)], zero before the launch
};
// One launch for one or two problems.
cudaError_t launch_lora_wgrad(const GemmShape& g, const WgradJob* jobs, int n_jobs,
                              const TileInfo* chunks, const int* n_chunks, int max_chunks,
                              const int32_t* chunk_start, cudaStream_t s);

// Expert-weight gradients (expert_dw.cuh): out[e] = Lm_e^T Rm_e over the rows of expert
// e (offsets), Lm [P, Mdim], Rm [P, Ndim] sorted rows, out [E, Mdim, Ndim] bf16.
cudaError_t launch_expert_dw(int kind, const GemmShape& g, const int32_t* offsets, const uint16_t* Lm,
                             int Mdim, const uint16_t* Rm, int Ndim, uint16_t* out, cudaStream_t s);

}  // namespace moe
