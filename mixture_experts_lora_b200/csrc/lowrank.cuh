// Rank-r products of the Split-LoRA reordering on tcgen05:
//     LR[q, :] = Act[q, :] L[e]        (q in the segment of expert e, L[e] is [K, r])
// i.e. X A_gu, H A_d, dy B_d^T and dGU B_gu^T ("Accelerating Mixture-of-Experts
// Fine-Tuning", Mathematical Formulation section 2, step 1: the compact [s, r]
// intermediate).  One CTA per 128-row tile of one expert (row tiles never
// straddle experts): M = 128 rows, N = RP (r padded to 16 or 32), K streamed in
// 64-wide stages.  The epilogue writes LR unscaled (for the adapter gradients)
// and bf16(c * LR) (the LoRA operand of the grouped GEMMs).  HBM-bound: it reads
// the activation rows once.
#pragma once

#include "common.cuh"

namespace moe {

struct LowrankParams {
  const TileInfo* tiles;   // 128-row tiles {e, row0, row_end}
  const int* n_tiles;
  int nk;                  // K steps of 64
  float scale;
  __nv_bfloat16* save;     // [P, ld_save]: first r_save columns of LR (unscaled)
  int ld_save;
  int r_save;
  __nv_bfloat16* outc;     // [P, RP]: bf16(scale * LR)
  int* err;
};

template <int RP, bool L_MN>
struct LowrankCfg {
  static constexpr int BM = 128, BK = 64, STAGES = 4;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int L_BYTES = RP * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + L_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 1024;
  static constexpr int TMEM_COLS = 32;
};

// L_MN: L stored [E, K, RP] (rank contiguous, MN-major B operand);
// otherwise L stored [E, RP, K] (K contiguous, K-major B operand).
template <int RP, bool L_MN>
__global__ void __launch_bounds__(128)
    lowrank_kernel(const __grid_constant__ CUtensorMap tmAct, const __grid_constant__ CUtensorMap tmL,
                   const LowrankParams p) {
  using C = LowrankCfg<RP, L_MN>;
  const int tile = blockIdx.x;
  if (tile >= *p.n_tiles) return;
  const TileInfo ti = p.tiles[tile];

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* done = bars + 2 * C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * C::STAGES + 2);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmL);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int ks = 0; ks < p.nk; ++ks) {
        if (*abort_flag) { ok = false; break; }
        if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err)) { ok = false; break; }
        const uint32_t fb = smem_u32(&full[stage]);
        const uint32_t sa = s_base + stage * C::STAGE_BYTES;
        mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
        tma_load_2d(&tmAct, fb, sa, ks * C::BK, ti.row0);
        if constexpr (L_MN) tma_load_3d(&tmL, fb, sa + C::A_BYTES, 0, ks * C::BK, ti.e);
        else tma_load_3d(&tmL, fb, sa + C::A_BYTES, ks * C::BK, 0, ti.e);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) {
        *abort_flag = 1;
        for (int s = 0; s < C::STAGES; ++s)
          mbar_wait(smem_u32(&full[s]), phase ^ (s < stage ? 0u : 1u), nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, RP, 0, L_MN ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int ks = 0; ks < p.nk; ++ks) {
        if (*abort_flag) { ok = false; break; }
        if (!mbar_wait(smem_u32(&full[stage]), phase, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = s_base + stage * C::STAGE_BYTES;
        const uint32_t sl = sa + C::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk) {
          const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024, kSw128);
          uint64_t bd;
          if constexpr (L_MN) {
            bd = (RP == 16) ? smem_desc(sl + kk * 16 * 32, C::L_BYTES, 256, kSw32)
                            : smem_desc(sl + kk * 16 * 64, C::L_BYTES, 512, kSw64);
          } else {
            bd = smem_desc(sl + kk * 32, 16, 1024, kSw128);
          }
          umma_bf16(tmem, ad, bd, idesc, (ks | kk) ? 1u : 0u);
        }
        umma_commit(smem_u32(&empty[stage]));
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) *abort_flag = 1;
      umma_commit(smem_u32(done));
    }
    __syncwarp();
  }

  __syncthreads();
  {
    bool ok = mbar_wait(smem_u32(done), 0, p.err);
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    tc_fence_after();
    float v[RP];
    if constexpr (RP == 16) {
      uint32_t r[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
    } else {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    }
    const int row = ti.row0 + warp * 32 + lane;
    if (ok && row < ti.row_end) {
      __nv_bfloat16* sv = p.save + (size_t)row * p.ld_save;
      uint4* oc = reinterpret_cast<uint4*>(p.outc + (size_t)row * RP);
#pragma unroll
      for (int g = 0; g < RP / 8; ++g) {
        if (g * 8 < p.r_save) {
          uint4 w;
          w.x = pack_bf16x2(v[8 * g + 0], v[8 * g + 1]);
          w.y = pack_bf16x2(v[8 * g + 2], v[8 * g + 3]);
          w.z = pack_bf16x2(v[8 * g + 4], v[8 * g + 5]);
          w.w = pack_bf16x2(v[8 * g + 6], v[8 * g + 7]);
          *reinterpret_cast<uint4*>(sv + 8 * g) = w;
        }
        uint4 c;
        c.x = pack_bf16x2(p.scale * v[8 * g + 0], p.scale * v[8 * g + 1]);
        c.y = pack_bf16x2(p.scale * v[8 * g + 2], p.scale * v[8 * g + 3]);
        c.z = pack_bf16x2(p.scale * v[8 * g + 4], p.scale * v[8 * g + 5]);
        c.w = pack_bf16x2(p.scale * v[8 * g + 6], p.scale * v[8 * g + 7]);
        oc[g] = c;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace moe
