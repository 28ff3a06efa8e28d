// Host side of the grouped GEMMs: launch geometry and the dispatch over the rank
// width and the atom-view choice.  Each GEMM of the layer has its own translation
// unit (gemm_*.cu) that builds its tensor maps and parameters.
#pragma once

#include "grouped_gemm.cuh"
#include "tmap.cuh"

namespace moe {

// Tensor maps of one GEMM launch: weights, token operand (boxes of 128 rows), the
// LoRA block's two operands, up to three output maps (unused ones repeat a valid
// map), and the token operand in boxes of 32, 64 and 96 rows.
struct GemmMaps {
  CUtensorMap m[10];
};

// The token operand's narrower boxes (atom views only; otherwise copies of the
// 128-row map, which the kernel then does not use).
inline bool encode_act_boxes(GemmMaps& mp, const uint16_t* act, uint64_t P, uint64_t K, bool v) {
  for (int i = 0; i < 3; ++i) {
    if (!v) {
      mp.m[7 + i] = mp.m[1];
    } else if (!encode_atoms(&mp.m[7 + i], act, false, 1, P, K, 32u * (i + 1), 2)) {
      return false;
    }
  }
  return true;
}

template <class C>
cudaError_t launch_gemm_cfg(int kind, const GemmShape& g, const GemmMaps& mp, const GemmParams& p,
                            cudaStream_t s) {
  auto kern = moe_gemm_kernel<C>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  const int64_t tiles = (int64_t)g.max_gchunks * p.n_ftiles;
  const int pairs_max = g.num_sms / 2 > 0 ? g.num_sms / 2 : 1;
  const int pairs = (int)(tiles < pairs_max ? (tiles > 0 ? tiles : 1) : pairs_max);
  ProfScope ps(kind, s);
  st = launch_pdl(kern, dim3(2 * pairs), dim3(C::THREADS), C::SMEM_BYTES, s, 2, mp.m[0], mp.m[1],
                  mp.m[2], mp.m[3], mp.m[4], mp.m[5], mp.m[6], mp.m[7], mp.m[8], mp.m[9], p);
  if (st != cudaSuccess) return st;
  return cudaGetLastError();
}

template <bool A_MN, int EPI>
cudaError_t dispatch_gemm(int kind, const GemmShape& g, bool v, const GemmMaps& mp,
                          const GemmParams& p, cudaStream_t s) {
#define MOE_GEMM_RP(RPV)                                                                 \
  case RPV:                                                                              \
    return v ? launch_gemm_cfg<GemmCfg<A_MN, RPV, true, EPI>>(kind, g, mp, p, s)         \
             : launch_gemm_cfg<GemmCfg<A_MN, RPV, false, EPI>>(kind, g, mp, p, s);
  switch (g.rp) {
    MOE_GEMM_RP(16)
    MOE_GEMM_RP(32)
    MOE_GEMM_RP(64)
    MOE_GEMM_RP(128)
  }
#undef MOE_GEMM_RP
  return cudaErrorInvalidValue;
}

// The LoRA block's maps: L_B^T of the weights' orientation and the rank-r rows LRc
// [P, rp] in boxes of 64 rows x min(rp, 64) ranks.  a_mn: L stored [E, r, F] (the
// forward's B), boxes of rp rows x 64 features; else [E, F, r] (the backward's A),
// boxes of 128 features x min(rp, 64) ranks.  Ranks r .. rp - 1 read as zero.
inline bool encode_lora(GemmMaps& mp, const GemmShape& g, bool a_mn, const uint16_t* L, int F,
                        const uint16_t* lrc) {
  const uint32_t lk = g.rp < 64 ? (uint32_t)g.rp : 64u;
  const uint64_t E = g.E, r = g.r, P = g.P;
  const bool ok = a_mn ? encode3d(&mp.m[2], L, E, r, (uint64_t)F, (uint32_t)g.rp, 64)
                       : encode3d(&mp.m[2], L, E, (uint64_t)F, r, 128, lk);
  return ok && encode2d(&mp.m[3], lrc, P, (uint64_t)g.rp, (uint64_t)g.rp, 64, lk);
}

// An output map [P, cols] with row stride ld, written in 32 x 32 blocks.
inline bool encode_out(CUtensorMap* m, const uint16_t* base, const GemmShape& g, uint64_t cols,
                       uint64_t ld) {
  return encode2d(m, base, (uint64_t)g.P, cols, ld, 32, 32, /*plain=*/true);
}

}  // namespace moe
