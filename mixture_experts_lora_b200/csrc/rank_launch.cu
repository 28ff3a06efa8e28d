// Host launchers of the rank-r products (rank_r.cuh): XA and T1 on gathered rows
// (written out as the expert-ordered operands), HA on the sorted rows of H, and the
// SwiGLU backward with T2.
#include "rank_r.cuh"
#include "tmap.cuh"

namespace moe {

namespace {

template <class C>
cudaError_t launch_rank_cfg(int kind, const GemmShape& g, const CUtensorMap* tm, const RankParams& p,
                            cudaStream_t s) {
  auto kern = rank_r_kernel<C>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  ProfScope ps(kind, s);
  st = launch_pdl(kern, dim3(g.max_row_tiles), dim3(C::THREADS), C::SMEM_BYTES, s, 1, tm[0], tm[1],
                  tm[2], tm[3], tm[4], p);
  if (st != cudaSuccess) return st;
  return cudaGetLastError();
}

template <int MODE, bool L_MN>
cudaError_t dispatch_rank(int kind, const GemmShape& g, const CUtensorMap* tm, const RankParams& p,
                          cudaStream_t s) {
  switch (g.rp) {
    case 16: return launch_rank_cfg<RankCfg<16, MODE, L_MN>>(kind, g, tm, p, s);
    case 32: return launch_rank_cfg<RankCfg<32, MODE, L_MN>>(kind, g, tm, p, s);
    case 64: return launch_rank_cfg<RankCfg<64, MODE, L_MN>>(kind, g, tm, p, s);
    case 128: return launch_rank_cfg<RankCfg<128, MODE, L_MN>>(kind, g, tm, p, s);
  }
  return cudaErrorInvalidValue;
}

// L as the MMA's B operand: [E, K, r] (l_mn, rank innermost) in boxes of 64 K rows x
// min(rp, 64) ranks, or [E, r, Kl] in boxes of rp ranks x 64 K; ranks past r read zero.
bool encode_l(CUtensorMap* m, const GemmShape& g, const uint16_t* L, int K, bool l_mn) {
  const uint64_t E = g.E, r = g.r;
  if (l_mn) return encode3d(m, L, E, (uint64_t)K, r, 64, g.rp < 64 ? (uint32_t)g.rp : 64u);
  return encode3d(m, L, E, r, (uint64_t)K, (uint32_t)g.rp, 64);
}

RankParams base_params(const GemmShape& g, int K, uint16_t* out_save, int ld_save, int r_save,
                       uint16_t* out_c) {
  RankParams p{};
  p.tiles = g.tiles;
  p.n_tiles = g.n_row_tiles;
  p.K = K;
  p.n_it = (K + 63) / 64;
  p.scale = g.scale;
  p.out_save = reinterpret_cast<__nv_bfloat16*>(out_save);
  p.ld_save = ld_save;
  p.r_save = r_save;
  p.out_c = reinterpret_cast<__nv_bfloat16*>(out_c);
  p.err = g.err;
  return p;
}

}  // namespace

cudaError_t launch_rank_gathered(int kind, const GemmShape& g, const uint16_t* src, int K,
                                 const int32_t* sorted_pairs, int k, const float* w,
                                 uint16_t* rows_out, const uint16_t* L, bool l_mn,
                                 uint16_t* out_save, int ld_save, int r_save, uint16_t* out_c,
                                 const TableBuild* tb, cudaStream_t s) {
  CUtensorMap tm[5];
  // tm[1]: the sorted rows written out, [P, K] in 128-row x 64-column swizzled boxes
  if (!encode_l(&tm[0], g, L, K, l_mn) ||
      !encode2d(&tm[1], rows_out, (uint64_t)g.P, (uint64_t)K, (uint64_t)K, 128, 64))
    return cudaErrorInvalidValue;
  tm[2] = tm[3] = tm[4] = tm[0];
  RankParams p = base_params(g, K, out_save, ld_save, r_save, out_c);
  p.src = reinterpret_cast<const __nv_bfloat16*>(src);
  p.sorted_pairs = sorted_pairs;
  p.k = k;
  p.w = w;
  p.rows_out = reinterpret_cast<__nv_bfloat16*>(rows_out);
  if (tb != nullptr) p.tb = *tb;
  return l_mn ? dispatch_rank<RK_GATHER, true>(kind, g, tm, p, s)
              : dispatch_rank<RK_GATHER, false>(kind, g, tm, p, s);
}

cudaError_t launch_rank_sorted(int kind, const GemmShape& g, const uint16_t* rows, int K,
                               const uint16_t* L, bool l_mn, uint16_t* out_save, int ld_save,
                               int r_save, uint16_t* out_c, cudaStream_t s) {
  CUtensorMap tm[5];
  if (!encode_l(&tm[0], g, L, K, l_mn) ||
      !encode2d(&tm[1], rows, (uint64_t)g.P, (uint64_t)K, (uint64_t)K, 128, 64))
    return cudaErrorInvalidValue;
  tm[2] = tm[3] = tm[4] = tm[1];
  RankParams p = base_params(g, K, out_save, ld_save, r_save, out_c);
  return l_mn ? dispatch_rank<RK_SORTED, true>(kind, g, tm, p, s)
              : dispatch_rank<RK_SORTED, false>(kind, g, tm, p, s);
}

cudaError_t launch_rank_dswiglu(const GemmShape& g, const uint16_t* dH, const uint16_t* GU,
                                const uint16_t* B_gu, uint16_t* dGU, uint16_t* out_save,
                                int ld_save, int r_save, uint16_t* out_c, cudaStream_t s) {
  CUtensorMap tm[5];
  const uint64_t P = (uint64_t)g.P, n = (uint64_t)g.n;
  // tm[3], tm[4]: the dg and du halves of dGU [P, 2n] (each n wide, so a box past n is
  // clipped at the half's end)
  if (!encode_l(&tm[0], g, B_gu, 2 * g.n, false) || !encode2d(&tm[1], dH, P, n, n, 128, 64) ||
      !encode2d(&tm[2], GU, P, 2 * n, 2 * n, 128, 64) ||
      !encode2d(&tm[3], dGU, P, n, 2 * n, 128, 64) || !encode2d(&tm[4], dGU + n, P, n, 2 * n, 128, 64))
    return cudaErrorInvalidValue;
  RankParams p = base_params(g, g.n, out_save, ld_save, r_save, out_c);
  p.rows_out = reinterpret_cast<__nv_bfloat16*>(dGU);
  return dispatch_rank<RK_DSWIGLU, false>(K_RANK_T2, g, tm, p, s);
}

}  // namespace moe
