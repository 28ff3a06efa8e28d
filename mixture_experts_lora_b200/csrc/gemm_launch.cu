// Host launchers for the tcgen05 grouped GEMMs and the adapter-gradient kernel:
// TMA tensor-map encoding, per-GEMM operand wiring and launch geometry.
#include <cudaTypedefs.h>

#include <mutex>

#include "expert_dw.cuh"
#include "grouped_gemm.cuh"
#include "internal.h"
#include "lora_wgrad.cuh"
#include "rows_gather.cuh"
#include "rows_swiglu.cuh"
#include "rows_common.cuh"

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
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
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

// [E, R, C] row-major (C % 64 == 0) seen as [E][C/64 atoms][R][64]: a box of
// `box_atoms` 64-wide atoms of `box_r` rows lands as atom-major 128-byte-swizzled
// tiles, so one copy fills a whole operand tile.  per_expert = false: a 2-D tensor
// [R, C] (3-D view, E ignored); true: always the 4-D view, even for E = 1, since the
// kernels address it with four coordinates.
bool encode_atoms(CUtensorMap* m, const void* base, bool per_expert, uint64_t E, uint64_t R,
                  uint64_t C, uint32_t box_r, uint32_t box_atoms) {
  const uint64_t dims[4] = {64, R, C / 64, E};
  const uint64_t str[3] = {C * 2, 128, R * C * 2};
  const uint32_t box[4] = {64, box_r, box_atoms, 1};
  return encode(m, base, per_expert ? 4 : 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <class Kern>
cudaError_t ensure_smem(Kern kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <class C>
cudaError_t launch_gemm(int kind, const GemmShape& g, const CUtensorMap* maps, const GemmParams& p,
                        cudaStream_t s) {
  auto kern = moe_gemm_kernel<C>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  const int64_t tiles = (int64_t)g.max_gchunks * p.n_ftiles;
  const int pairs_max = g.num_sms / 2 > 0 ? g.num_sms / 2 : 1;
  const int pairs = (int)(tiles < pairs_max ? (tiles > 0 ? tiles : 1) : pairs_max);
  ProfScope ps(kind, s);
  st = launch_pdl(kern, dim3(2 * pairs), dim3(320), C::SMEM_BYTES, s, 2, maps[0], maps[1], maps[2],
                  maps[3], maps[4], p);
  if (st != cudaSuccess) return st;
  return cudaGetLastError();
}

// One grouped GEMM: out [P, F] = act [P, K] x W[e] (+ LoRA block), features on M.
// w_fk: W stored [E, F, K] (K-major A) instead of [E, K, F] (MN-major A);
// lw: L_B^T stored [E, rp, F] (forward) or [E, F, rp] (backward).
cudaError_t gemm_any(int kind, const GemmShape& g, const uint16_t* W, bool w_fk, int F, int K,
                     const uint16_t* act, const uint16_t* lw, const uint16_t* lrc, uint16_t* out,
                     cudaStream_t s) {
  CUtensorMap mp[5];
  const uint64_t P = g.P, E = g.E, rp = g.rp;
  using C0 = GemmCfg<true, 16>;
  {
    // out [P, F]: 32-token x 32-feature blocks stored from the epilogue's staging
    const uint64_t dims[2] = {(uint64_t)F, P};
    const uint64_t str[1] = {(uint64_t)F * 2};
    const uint32_t box[2] = {32, 32};
    if (!encode(&mp[4], out, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorInvalidValue;
  }
  // atom views (one copy per operand and stage) when the K (and MN-major F) extents
  // are whole 64-wide atoms
  const bool v = K % 64 == 0 && (w_fk || F % 64 == 0);
  bool ok = (v ? encode_atoms(&mp[1], act, false, 1, P, (uint64_t)K, C0::NHALF, C0::BK / 64)
               : encode2d(&mp[1], act, P, (uint64_t)K, C0::NHALF, C0::KA)) &&
            encode2d(&mp[3], lrc, P, rp, C0::BOXR, (uint32_t)rp);
  if (w_fk) {
    ok = ok && (v ? encode_atoms(&mp[0], W, true, E, (uint64_t)F, (uint64_t)K, C0::BM, C0::BK / 64)
                  : encode3d(&mp[0], W, E, (uint64_t)F, (uint64_t)K, 128, 64)) &&
         encode3d(&mp[2], lw, E, (uint64_t)F, rp, 128, (uint32_t)rp);
  } else {
    ok = ok && (v ? encode_atoms(&mp[0], W, true, E, (uint64_t)K, (uint64_t)F, C0::BK, 2)
                  : encode3d(&mp[0], W, E, (uint64_t)K, (uint64_t)F, C0::BK, 64)) &&
         encode3d(&mp[2], lw, E, rp, (uint64_t)F, (uint32_t)rp, 64);
  }
  if (!ok) return cudaErrorInvalidValue;
  GemmParams p{};
  p.chunks = g.gchunks;
  p.n_chunks = g.n_gchunks;
  p.F = F;
  p.n_ftiles = (F + 255) / 256;
  p.nk = (K + C0::BK - 1) / C0::BK;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.err = g.err;
  if (w_fk) {
    if (v) {
      if (g.rp == 16) return launch_gemm<GemmCfg<false, 16, true>>(kind, g, mp, p, s);
      return launch_gemm<GemmCfg<false, 32, true>>(kind, g, mp, p, s);
    }
    if (g.rp == 16) return launch_gemm<GemmCfg<false, 16>>(kind, g, mp, p, s);
    return launch_gemm<GemmCfg<false, 32>>(kind, g, mp, p, s);
  }
  if (v) {
    if (g.rp == 16) return launch_gemm<GemmCfg<true, 16, true>>(kind, g, mp, p, s);
    return launch_gemm<GemmCfg<true, 32, true>>(kind, g, mp, p, s);
  }
  if (g.rp == 16) return launch_gemm<GemmCfg<true, 16>>(kind, g, mp, p, s);
  return launch_gemm<GemmCfg<true, 32>>(kind, g, mp, p, s);
}

}  // namespace

cudaError_t launch_gemm_gateup_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* Xs,
                                   const uint16_t* XAc, uint16_t* GU, cudaStream_t s) {
  return gemm_any(K_GEMM_GATEUP_FWD, g, w.W_gu, false, 2 * g.n, g.m, Xs, w.B_gu, XAc, GU, s);
}

cudaError_t launch_gemm_down_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* H,
                                 const uint16_t* HAc, uint16_t* Yp, cudaStream_t s) {
  return gemm_any(K_GEMM_DOWN_FWD, g, w.W_d, false, g.m, g.n, H, w.B_d, HAc, Yp, s);
}

cudaError_t launch_gemm_down_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dys,
                                 const uint16_t* T1c, uint16_t* dH, cudaStream_t s) {
  return gemm_any(K_GEMM_DOWN_BWD, g, w.W_d, true, g.n, g.m, dys, w.A_d, T1c, dH, s);
}

cudaError_t launch_gemm_gateup_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dGU,
                                   const uint16_t* T2c, uint16_t* dXp, cudaStream_t s) {
  return gemm_any(K_GEMM_GATEUP_BWD, g, w.W_gu, true, g.m, 2 * g.n, dGU, w.A_gu, T2c, dXp, s);
}

template <int RP, bool L_MN>
static cudaError_t rows_gather_rp(const GemmShape& g, const CUtensorMap* tl, const RowsParams& rp_,
                                  cudaStream_t s) {
  using C = RowsGatherCfg<RP>;
  auto kern = rows_gather_kernel<RP, L_MN>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  ProfScope ps(K_ROWS_GATHER, s);
  if (cudaError_t le_ = launch_pdl(kern, dim3(g.max_row_tiles), dim3(RG_THREADS), C::SMEM_BYTES, s, 1, tl[0], rp_); le_ != cudaSuccess) return le_;
  return cudaGetLastError();
}

template <int MODE, int RP>
static cudaError_t rows_swiglu_rp(const GemmShape& g, const CUtensorMap* tl, const RowsParams& rp_,
                                  cudaStream_t s) {
  using C = RowsSwigluCfg<MODE, RP>;
  auto kern = rows_swiglu_kernel<MODE, RP>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  // persistent: C::CTAS_PER_SM per SM (the kernel uses at most one CTA per unit)
  int grid = g.num_sms * C::CTAS_PER_SM;
  if (grid > kRowsMaxCtas) grid = kRowsMaxCtas;
  ProfScope ps(MODE == ROWS_SWIGLU ? K_ROWS_SWIGLU : K_ROWS_SWIGLU_BWD, s);
  if (cudaError_t le_ = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, 1, tl[0], tl[1], tl[2], rp_); le_ != cudaSuccess) return le_;
  return cudaGetLastError();
}

cudaError_t launch_rows_lowrank(const GemmShape& g, int mode, int K, const uint16_t* src,
                                const int32_t* sorted_pairs, const float* w, int k,
                                const uint16_t* gu, const uint16_t* dh, const uint16_t* L,
                                bool L_mn, uint16_t* rows_out, uint16_t* save, int ld_save,
                                int r_save, uint16_t* outc, float* partial, int* counters,
                                cudaStream_t s) {
  CUtensorMap tl[3];
  const uint64_t E = g.E, rp = g.rp, P = g.P, n = g.n;
  bool ok = L_mn ? encode3d(&tl[0], L, E, (uint64_t)K, rp, 64, (uint32_t)rp)
                 : encode3d(&tl[0], L, E, rp, (uint64_t)K, (uint32_t)rp, 64);
  // input tiles of 128 rows x 64 columns, no swizzle (the threads read them back)
  auto plain = [&](CUtensorMap* m, const void* base, uint64_t cols) {
    const uint64_t dims[2] = {cols, P};
    const uint64_t str[1] = {cols * 2};
    const uint32_t box[2] = {64, 128};
    return encode(m, base, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
  };
  ok = ok && plain(&tl[1], gu != nullptr ? gu : L, gu != nullptr ? 2 * n : 64);
  ok = ok && plain(&tl[2], dh != nullptr ? dh : L, dh != nullptr ? n : 64);
  if (!ok) return cudaErrorInvalidValue;
  RowsParams p{};
  p.tiles = g.tiles;
  p.n_tiles = g.n_row_tiles;
  p.K = K;
  p.nk = (K + 63) / 64;
  p.src = reinterpret_cast<const __nv_bfloat16*>(src);
  p.sorted_pairs = sorted_pairs;
  p.w = w;
  p.k = k;
  p.gu = reinterpret_cast<const __nv_bfloat16*>(gu);
  p.dh = reinterpret_cast<const __nv_bfloat16*>(dh);
  p.n = g.n;
  p.rows_out = reinterpret_cast<__nv_bfloat16*>(rows_out);
  p.scale = g.scale;
  p.save = reinterpret_cast<__nv_bfloat16*>(save);
  p.ld_save = ld_save;
  p.r_save = r_save;
  p.outc = reinterpret_cast<__nv_bfloat16*>(outc);
  p.partial = partial;
  p.counters = counters;
  p.err = g.err;
  if (mode == ROWS_GATHER) {
    if (g.rp == 16)
      return L_mn ? rows_gather_rp<16, true>(g, tl, p, s) : rows_gather_rp<16, false>(g, tl, p, s);
    return L_mn ? rows_gather_rp<32, true>(g, tl, p, s) : rows_gather_rp<32, false>(g, tl, p, s);
  }
  // SwiGLU modes: 128-row x 64-column input tiles, 128-byte swizzled (they become
  // the MMA operand in place)
  ok = encode2d(&tl[1], gu, P, 2 * n, 128, 64) &&
       encode2d(&tl[2], dh != nullptr ? dh : gu, P, dh != nullptr ? n : 2 * n, 128, 64);
  if (!ok) return cudaErrorInvalidValue;
  if (mode == ROWS_SWIGLU)
    return g.rp == 16 ? rows_swiglu_rp<ROWS_SWIGLU, 16>(g, tl, p, s) : rows_swiglu_rp<ROWS_SWIGLU, 32>(g, tl, p, s);
  return g.rp == 16 ? rows_swiglu_rp<ROWS_SWIGLU_BWD, 16>(g, tl, p, s)
                    : rows_swiglu_rp<ROWS_SWIGLU_BWD, 32>(g, tl, p, s);
}


template <int RP, bool V>
static cudaError_t wgrad_rp(const GemmShape& g, const CUtensorMap* tm, const WgradParams& wp,
                            int max_chunks, cudaStream_t s) {
  using C = WgradCfg<RP, V>;
  auto kern = lora_wgrad_kernel<RP, V>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  int dtiles = wp.pr[0].n_dtiles + (wp.n_problems > 1 ? wp.pr[1].n_dtiles : 0);
  const int64_t units = (int64_t)max_chunks * dtiles;
  // at least one CTA per SM: the zero fill of experts without rows runs in every CTA
  const int grid = (int)(units > 0 && units < g.num_sms ? units : g.num_sms);
  ProfScope ps(K_WGRAD, s);
  if (cudaError_t le_ = launch_pdl(kern, dim3(grid), dim3(192), C::SMEM_BYTES, s, 1, tm[0], tm[1], tm[2], tm[3], wp); le_ != cudaSuccess) return le_;
  return cudaGetLastError();
}

cudaError_t launch_lora_wgrad(const GemmShape& g, const WgradJob* jobs, int n_jobs,
                              const TileInfo* chunks, const int* n_chunks, int max_chunks,
                              const int32_t* chunk_start, cudaStream_t s) {
  if (n_jobs < 1 || n_jobs > 2) return cudaErrorInvalidValue;
  using C0 = WgradCfg<16>;
  CUtensorMap tm[4];      // Big of each problem, then Small of each problem
  WgradParams wp{};
  const uint64_t P = (uint64_t)(g.P > 0 ? g.P : 1);
  bool v = true;
  for (int j = 0; j < n_jobs; ++j) v = v && jobs[j].D % 64 == 0;
  for (int j = 0; j < n_jobs; ++j) {
    const WgradJob& jb = jobs[j];
    // Big [P, D]: BK rows x 256 columns per stage (four 64-column atoms)
    const bool okb = v ? encode_atoms(&tm[j], jb.big, false, 1, P, (uint64_t)jb.D, C0::BK, C0::BN / 64)
                       : encode2d(&tm[j], jb.big, P, (uint64_t)jb.D, C0::BK, 64);
    // Small [P, ld_small] seen as [ld_small / 8 groups][P rows][8 columns]: a box of
    // BK rows x rp / 8 groups lands group-major, groups past ld_small reading as zero
    const uint64_t sd[3] = {8, P, (uint64_t)jb.ld_small / 8};
    const uint64_t ss[2] = {(uint64_t)jb.ld_small * 2, 16};
    const uint32_t sb[3] = {8, (uint32_t)C0::BK, (uint32_t)g.rp / 8};
    if (!okb || !encode(&tm[2 + j], jb.small, 3, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    WgradProblem& q = wp.pr[j];
    q.small = reinterpret_cast<const __nv_bfloat16*>(jb.small);
    q.ld_small = jb.ld_small;
    q.r_small = jb.ld_small;  // the caller's buffer has exactly ld_small columns
    q.D = jb.D;
    q.n_dtiles = (jb.D + C0::BN - 1) / C0::BN;
    q.transpose = jb.transpose;
    q.out = reinterpret_cast<__nv_bfloat16*>(jb.out);
    q.partial = jb.partial;
    q.counters = jb.counters;
  }
  if (n_jobs == 1) {
    tm[1] = tm[0];
    tm[3] = tm[2];
  }
  wp.n_problems = n_jobs;
  wp.chunks = chunks;
  wp.n_chunks = n_chunks;
  wp.chunk_start = chunk_start;
  wp.E = g.E;
  wp.r = g.r;
  wp.scale = g.scale;
  wp.err = g.err;
  if (g.rp == 16) return v ? wgrad_rp<16, true>(g, tm, wp, max_chunks, s) : wgrad_rp<16, false>(g, tm, wp, max_chunks, s);
  return v ? wgrad_rp<32, true>(g, tm, wp, max_chunks, s) : wgrad_rp<32, false>(g, tm, wp, max_chunks, s);
}

template <class C>
static cudaError_t expert_dw_launch(int kind, const CUtensorMap* tm, const DwParams& p, int num_sms,
                                    cudaStream_t s) {
  auto kern = moe_dw_kernel<C>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  const int64_t total = (int64_t)p.E * p.n_mt * p.n_nt;
  const int grid = (int)(total < num_sms ? total : num_sms);
  ProfScope ps(kind, s);
  if (cudaError_t le_ = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, 1, tm[0], tm[1], tm[2], p); le_ != cudaSuccess) return le_;
  return cudaGetLastError();
}

cudaError_t launch_expert_dw(int kind, const GemmShape& g, const int32_t* offsets, const uint16_t* Lm,
                             int Mdim, const uint16_t* Rm, int Ndim, uint16_t* out, cudaStream_t s) {
  using C = DwCfg<true>;
  CUtensorMap tm[3];
  const uint64_t P = (uint64_t)g.P;
  const bool v = Mdim % 64 == 0 && Ndim % 64 == 0;
  const bool ok = v ? encode_atoms(&tm[0], Lm, false, 1, P, (uint64_t)Mdim, C::BK, 2) &&
                          encode_atoms(&tm[1], Rm, false, 1, P, (uint64_t)Ndim, C::BK, 4)
                    : encode2d(&tm[0], Lm, P, (uint64_t)Mdim, C::BK, 64) &&
                          encode2d(&tm[1], Rm, P, (uint64_t)Ndim, C::BK, 64);
  // output [E, Mdim, Ndim] in 32 x 32 blocks, 64-byte swizzle (the staging layout)
  const uint64_t odims[3] = {(uint64_t)Ndim, (uint64_t)Mdim, (uint64_t)g.E};
  const uint64_t ostr[2] = {(uint64_t)Ndim * 2, (uint64_t)Mdim * Ndim * 2};
  const uint32_t obox[3] = {32, 32, 1};
  if (!ok || !encode(&tm[2], out, 3, odims, ostr, obox, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  DwParams p{};
  p.offsets = offsets;
  p.E = g.E;
  p.Mdim = Mdim;
  p.Ndim = Ndim;
  p.n_mt = (Mdim + C::BM - 1) / C::BM;
  p.n_nt = (Ndim + C::BN - 1) / C::BN;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.err = g.err;
  return v ? expert_dw_launch<DwCfg<true>>(kind, tm, p, g.num_sms, s)
           : expert_dw_launch<DwCfg<false>>(kind, tm, p, g.num_sms, s);
}

}  // namespace moe
