// Host launchers of the rank-r products (rank_r.cuh): XA and T1' from rows gathered
// out of X and dY, HA and T2 from the sorted rows of H and dGU.
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
  st = launch_pdl(kern, dim3(g.max_row_tiles), dim3(C::THREADS), C::SMEM_BYTES, s, 1, tm[0], tm[1], p);
  if (st != cudaSuccess) return st;
  return cudaGetLastError();
}

template <bool GATHER, bool L_MN>
cudaError_t dispatch_rank(int kind, const GemmShape& g, const CUtensorMap* tm, const RankParams& p,
                          cudaStream_t s) {
  switch (g.rp) {
    case 16: return launch_rank_cfg<RankCfg<16, GATHER, L_MN>>(kind, g, tm, p, s);
    case 32: return launch_rank_cfg<RankCfg<32, GATHER, L_MN>>(kind, g, tm, p, s);
    case 64: return launch_rank_cfg<RankCfg<64, GATHER, L_MN>>(kind, g, tm, p, s);
    case 128: return launch_rank_cfg<RankCfg<128, GATHER, L_MN>>(kind, g, tm, p, s);
  }
  return cudaErrorInvalidValue;
}

// L as the MMA's B operand: [E, K, r] (l_mn, rank innermost) in boxes of 64 K rows x
// min(rp, 64) ranks, or [E, r, K] in boxes of rp ranks x 64 K; ranks past r read zero.
bool encode_l(CUtensorMap* m, const GemmShape& g, const uint16_t* L, int K, bool l_mn) {
  const uint64_t E = g.E, r = g.r;
  if (l_mn) return encode3d(m, L, E, (uint64_t)K, r, 64, g.rp < 64 ? (uint32_t)g.rp : 64u);
  return encode3d(m, L, E, r, (uint64_t)K, (uint32_t)g.rp, 64);
}

RankParams base_params(const GemmShape& g, int K) {
  RankParams p{};
  p.tiles = g.tiles;
  p.n_tiles = g.n_row_tiles;
  p.K = K;
  p.n_it = (K + 63) / 64;
  p.scale = g.scale;
  p.err = g.err;
  return p;
}

}  // namespace

cudaError_t launch_rank_gathered(int kind, const GemmShape& g, const uint16_t* src, int K,
                                 const int32_t* sorted_pairs, int k, const float* w,
                                 const uint16_t* L, bool l_mn, uint16_t* out_save, int ld_save,
                                 int r_save, bool save_w, uint16_t* out_c, const uint16_t* wsrc,
                                 int r_wsrc, uint16_t* out_w, cudaStream_t s) {
  CUtensorMap tm[2];
  if (!encode_l(&tm[0], g, L, K, l_mn)) return cudaErrorInvalidValue;
  tm[1] = tm[0];   // rows gathered, no map
  RankParams p = base_params(g, K);
  p.src = reinterpret_cast<const __nv_bfloat16*>(src);
  p.sorted_pairs = sorted_pairs;
  p.k = k;
  p.w = w;
  p.out_save = reinterpret_cast<__nv_bfloat16*>(out_save);
  p.ld_save = ld_save;
  p.r_save = r_save;
  p.save_w = save_w;
  p.out_c = reinterpret_cast<__nv_bfloat16*>(out_c);
  p.wsrc = reinterpret_cast<const __nv_bfloat16*>(wsrc);
  p.r_wsrc = r_wsrc;
  p.out_w = reinterpret_cast<__nv_bfloat16*>(out_w);
  return l_mn ? dispatch_rank<true, true>(kind, g, tm, p, s) : dispatch_rank<true, false>(kind, g, tm, p, s);
}

cudaError_t launch_rank_sorted(int kind, const GemmShape& g, const uint16_t* rows, int K,
                               const uint16_t* L, bool l_mn, uint16_t* out_save, int ld_save,
                               int r_save, uint16_t* out_c, cudaStream_t s) {
  CUtensorMap tm[2];
  if (!encode_l(&tm[0], g, L, K, l_mn) ||
      !encode2d(&tm[1], rows, (uint64_t)g.P, (uint64_t)K, (uint64_t)K, 128, 64))
    return cudaErrorInvalidValue;
  RankParams p = base_params(g, K);
  p.out_save = reinterpret_cast<__nv_bfloat16*>(out_save);
  p.ld_save = ld_save;
  p.r_save = r_save;
  p.out_c = reinterpret_cast<__nv_bfloat16*>(out_c);
  return l_mn ? dispatch_rank<false, true>(kind, g, tm, p, s) : dispatch_rank<false, false>(kind, g, tm, p, s);
}

}  // namespace moe
