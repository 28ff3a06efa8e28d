// Host launchers for the tcgen05 grouped GEMMs and the adapter-gradient kernel:
// TMA tensor-map encoding, per-GEMM operand wiring and launch geometry.
#include <cudaTypedefs.h>

#include <mutex>

#include "grouped_gemm.cuh"
#include "internal.h"
#include "lora_wgrad.cuh"
#include "lowrank.cuh"

namespace moe {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

CUtensorMapSwizzle swz_for_bytes(int inner_bytes) {
  switch (inner_bytes) {
    case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
    case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
    default: return CU_TENSOR_MAP_SWIZZLE_128B;
  }
}

// bf16 tensor of `rank` dims (dims[0] innermost, contiguous), box `box`.
bool encode(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
            const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base),
                  reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes),
                  reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [rows, cols] row-major, box [box_rows, box_cols]
bool encode2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t str[1] = {cols * 2};
  const uint32_t box[2] = {box_cols, box_rows};
  return encode(m, base, 2, dims, str, box, swz_for_bytes((int)box_cols * 2));
}

// [E, rows, cols] row-major, box [1, box_rows, box_cols]
bool encode3d(CUtensorMap* m, const void* base, uint64_t E, uint64_t rows, uint64_t cols,
              uint32_t box_rows, uint32_t box_cols) {
  const uint64_t dims[3] = {cols, rows, E};
  const uint64_t str[2] = {cols * 2, rows * cols * 2};
  const uint32_t box[3] = {box_cols, box_rows, 1};
  return encode(m, base, 3, dims, str, box, swz_for_bytes((int)box_cols * 2));
}

template <class Kern>
cudaError_t ensure_smem(Kern kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <class C>
cudaError_t launch_gemm(int kind, const GemmShape& g, const CUtensorMap& tw, const CUtensorMap& ta,
                        const CUtensorMap& tlw, const CUtensorMap& tlr, const GemmParams& p,
                        cudaStream_t s) {
  auto kern = moe_gemm_kernel<C>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  const int64_t tiles = (int64_t)g.max_gchunks * p.n_ftiles;
  const int grid = (int)(tiles < g.num_sms ? (tiles > 0 ? tiles : 1) : g.num_sms);
  ProfScope ps(kind, s);
  kern<<<grid, 192, C::SMEM_BYTES, s>>>(tw, ta, tlw, tlr, p);
  return cudaGetLastError();
}

GemmParams base_params(const GemmShape& g, int F, int K, int feat_per_tile) {
  GemmParams p{};
  p.chunks = g.gchunks;
  p.n_chunks = g.n_gchunks;
  p.F = F;
  p.K = K;
  p.n_ftiles = (F + feat_per_tile - 1) / feat_per_tile;
  p.nk = (K + 63) / 64;
  p.err = g.err;
  return p;
}

}  // namespace

// Token-row operand boxes: 32 rows x 64 K (activations) or 32 rows x rp (LoRA operand).
constexpr uint32_t kTokBox = 32;

cudaError_t launch_gemm_gateup_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* Xs,
                                   const uint16_t* XAc, uint16_t* GU, uint16_t* H, cudaStream_t s) {
  CUtensorMap tw, ta, tlw, tlr;
  const uint64_t P = g.P, m = g.m, n = g.n, E = g.E, rp = g.rp;
  if (!encode3d(&tw, w.W_gu, E, m, 2 * n, 64, 64) || !encode2d(&ta, Xs, P, m, kTokBox, 64) ||
      !encode3d(&tlw, w.B_gu, E, rp, 2 * n, (uint32_t)rp, 64) ||
      !encode2d(&tlr, XAc, P, rp, kTokBox, (uint32_t)rp))
    return cudaErrorInvalidValue;
  GemmParams p = base_params(g, g.n, g.m, 64);
  p.n_half = g.n;
  p.out0 = reinterpret_cast<__nv_bfloat16*>(GU);
  p.ld0 = 2 * g.n;
  p.out1 = reinterpret_cast<__nv_bfloat16*>(H);
  p.ld1 = g.n;
  if (g.rp == 16) return launch_gemm<GemmCfg<EPI_GATEUP_FWD, true, 16>>(K_GEMM_GATEUP_FWD, g, tw, ta, tlw, tlr, p, s);
  return launch_gemm<GemmCfg<EPI_GATEUP_FWD, true, 32>>(K_GEMM_GATEUP_FWD, g, tw, ta, tlw, tlr, p, s);
}

cudaError_t launch_gemm_down_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* H,
                                 const uint16_t* HAc, uint16_t* Yp, cudaStream_t s) {
  CUtensorMap tw, ta, tlw, tlr;
  const uint64_t P = g.P, m = g.m, n = g.n, E = g.E, rp = g.rp;
  if (!encode3d(&tw, w.W_d, E, n, m, 64, 64) || !encode2d(&ta, H, P, n, kTokBox, 64) ||
      !encode3d(&tlw, w.B_d, E, rp, m, (uint32_t)rp, 64) ||
      !encode2d(&tlr, HAc, P, rp, kTokBox, (uint32_t)rp))
    return cudaErrorInvalidValue;
  GemmParams p = base_params(g, g.m, g.n, 128);
  p.out0 = reinterpret_cast<__nv_bfloat16*>(Yp);
  p.ld0 = g.m;
  if (g.rp == 16) return launch_gemm<GemmCfg<EPI_STORE, true, 16>>(K_GEMM_DOWN_FWD, g, tw, ta, tlw, tlr, p, s);
  return launch_gemm<GemmCfg<EPI_STORE, true, 32>>(K_GEMM_DOWN_FWD, g, tw, ta, tlw, tlr, p, s);
}

cudaError_t launch_gemm_down_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dys,
                                 const uint16_t* T1c, const uint16_t* GU, uint16_t* dGU,
                                 cudaStream_t s) {
  CUtensorMap tw, ta, tlw, tlr;
  const uint64_t P = g.P, m = g.m, n = g.n, E = g.E, rp = g.rp;
  if (!encode3d(&tw, w.W_d, E, n, m, 128, 64) || !encode2d(&ta, dys, P, m, kTokBox, 64) ||
      !encode3d(&tlw, w.A_d, E, n, rp, 128, (uint32_t)rp) ||
      !encode2d(&tlr, T1c, P, rp, kTokBox, (uint32_t)rp))
    return cudaErrorInvalidValue;
  GemmParams p = base_params(g, g.n, g.m, 128);
  p.n_half = g.n;
  p.out0 = reinterpret_cast<__nv_bfloat16*>(dGU);
  p.ld0 = 2 * g.n;
  p.in0 = reinterpret_cast<const __nv_bfloat16*>(GU);
  p.ldi0 = 2 * g.n;
  if (g.rp == 16) return launch_gemm<GemmCfg<EPI_SWIGLU_BWD, false, 16>>(K_GEMM_DOWN_BWD, g, tw, ta, tlw, tlr, p, s);
  return launch_gemm<GemmCfg<EPI_SWIGLU_BWD, false, 32>>(K_GEMM_DOWN_BWD, g, tw, ta, tlw, tlr, p, s);
}

cudaError_t launch_gemm_gateup_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dGU,
                                   const uint16_t* T2c, uint16_t* dXp, cudaStream_t s) {
  CUtensorMap tw, ta, tlw, tlr;
  const uint64_t P = g.P, m = g.m, n = g.n, E = g.E, rp = g.rp;
  if (!encode3d(&tw, w.W_gu, E, m, 2 * n, 128, 64) || !encode2d(&ta, dGU, P, 2 * n, kTokBox, 64) ||
      !encode3d(&tlw, w.A_gu, E, m, rp, 128, (uint32_t)rp) ||
      !encode2d(&tlr, T2c, P, rp, kTokBox, (uint32_t)rp))
    return cudaErrorInvalidValue;
  GemmParams p = base_params(g, g.m, 2 * g.n, 128);
  p.out0 = reinterpret_cast<__nv_bfloat16*>(dXp);
  p.ld0 = g.m;
  if (g.rp == 16) return launch_gemm<GemmCfg<EPI_STORE, false, 16>>(K_GEMM_GATEUP_BWD, g, tw, ta, tlw, tlr, p, s);
  return launch_gemm<GemmCfg<EPI_STORE, false, 32>>(K_GEMM_GATEUP_BWD, g, tw, ta, tlw, tlr, p, s);
}

template <int RP, bool L_MN>
static cudaError_t lowrank_rp(const GemmShape& g, const CUtensorMap& ta, const CUtensorMap& tl,
                              const LowrankParams& lp, cudaStream_t s) {
  using C = LowrankCfg<RP, L_MN>;
  auto kern = lowrank_kernel<RP, L_MN>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  ProfScope ps(K_LOWRANK, s);
  kern<<<g.max_row_tiles, 128, C::SMEM_BYTES, s>>>(ta, tl, lp);
  return cudaGetLastError();
}

cudaError_t launch_lowrank(const GemmShape& g, const uint16_t* act, int K, const uint16_t* L,
                           bool L_mn, uint16_t* save, int ld_save, int r_save, uint16_t* outc,
                           cudaStream_t s) {
  CUtensorMap ta, tl;
  const uint64_t E = g.E, rp = g.rp;
  bool ok = encode2d(&ta, act, (uint64_t)g.P, (uint64_t)K, 128, 64);
  ok = ok && (L_mn ? encode3d(&tl, L, E, (uint64_t)K, rp, 64, (uint32_t)rp)
                   : encode3d(&tl, L, E, rp, (uint64_t)K, (uint32_t)rp, 64));
  if (!ok) return cudaErrorInvalidValue;
  LowrankParams lp{};
  lp.tiles = g.tiles;
  lp.n_tiles = g.n_row_tiles;
  lp.nk = (K + 63) / 64;
  lp.scale = g.scale;
  lp.save = reinterpret_cast<__nv_bfloat16*>(save);
  lp.ld_save = ld_save;
  lp.r_save = r_save;
  lp.outc = reinterpret_cast<__nv_bfloat16*>(outc);
  lp.err = g.err;
  if (g.rp == 16) return L_mn ? lowrank_rp<16, true>(g, ta, tl, lp, s) : lowrank_rp<16, false>(g, ta, tl, lp, s);
  return L_mn ? lowrank_rp<32, true>(g, ta, tl, lp, s) : lowrank_rp<32, false>(g, ta, tl, lp, s);
}

template <int RP>
static cudaError_t wgrad_rp(const GemmShape& g, const CUtensorMap& tm, const WgradParams& wp, int D,
                            int max_chunks, const int32_t* chunk_start, bool transpose,
                            uint16_t* out, cudaStream_t s) {
  using C = WgradCfg<RP>;
  auto kern = lora_wgrad_kernel<RP>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  if (max_chunks > 0) {
    dim3 grid((D + 127) / 128, max_chunks);
    ProfScope ps(K_WGRAD, s);
    kern<<<grid, 128, C::SMEM_BYTES, s>>>(tm, wp);
    st = cudaGetLastError();
    if (st != cudaSuccess) return st;
  }
  const int64_t total = (int64_t)g.E * D;
  ProfScope ps(K_WGRAD_REDUCE, s);
  lora_wgrad_reduce_kernel<RP><<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
      wp.partial, chunk_start, g.E, D, g.r, g.scale, transpose,
      reinterpret_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

cudaError_t launch_lora_wgrad(const GemmShape& g, const uint16_t* big, int D, const uint16_t* small,
                              int ld_small, const TileInfo* chunks, const int* n_chunks,
                              int max_chunks, const int32_t* chunk_start, float* partial,
                              bool transpose, uint16_t* out, cudaStream_t s) {
  CUtensorMap tm;
  if (!encode2d(&tm, big, (uint64_t)(g.P > 0 ? g.P : 1), (uint64_t)D, 64, 64))
    return cudaErrorInvalidValue;
  WgradParams wp{};
  wp.small = reinterpret_cast<const __nv_bfloat16*>(small);
  wp.ld_small = ld_small;
  wp.r_small = ld_small;  // the caller's buffer has exactly ld_small columns
  wp.chunks = chunks;
  wp.n_chunks = n_chunks;
  wp.D = D;
  wp.partial = partial;
  wp.err = g.err;
  if (g.rp == 16) return wgrad_rp<16>(g, tm, wp, D, max_chunks, chunk_start, transpose, out, s);
  return wgrad_rp<32>(g, tm, wp, D, max_chunks, chunk_start, transpose, out, s);
}

}  // namespace moe
