// SwiGLU row kernels of the layer fused with the rank-r products of the Split-LoRA
// reordering ("Accelerating Mixture-of-Experts Fine-Tuning", Mathematical
// Formulation section 2; gate = first n columns of GU, h = silu(g) * u):
//   ROWS_SWIGLU      H = silu(g) u                                   -> H,   HA = H A_d
//   ROWS_SWIGLU_BWD  dGU = [dH u s (1 + g (1 - s)), dH g s], s = sigmoid(g)
//                                                                    -> dGU, T2 = dGU B_gu^T
// One CTA owns a 128-row tile of one expert's sorted rows and walks the n columns
// in 64-column stages through a ring of shared-memory stages:
//   * a control thread loads each stage's input tiles (g, u and for the backward
//     dH) with TMA in the 128-byte-swizzled K-major layout, together with the
//     stage's adapter chunk, and issues the rank-r MMAs once the workers are done;
//   * 256 worker threads compute the activation (or its derivative) in place in
//     the swizzled tiles, which thereby become the MMA operand, and write the rows
//     to HBM.
// The epilogue writes LR unscaled (kept for the adapter gradients) and
// bf16(c * LR) (the LoRA operand of the next grouped GEMM).
#pragma once

#include "common.cuh"
#include "rows_common.cuh"

namespace moe {

template <int MODE, int RP>
struct RowsSwigluCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int NT = MODE == ROWS_SWIGLU ? 2 : 3;        // input tiles per stage
  static constexpr int HALVES = MODE == ROWS_SWIGLU ? 1 : 2;    // MMA operand tiles per stage
  static constexpr int TILE_BYTES = BM * BK * 2;                // 16 KB
  static constexpr int L_BYTES = HALVES * RP * BK * 2;
  static constexpr int STAGE_BYTES = NT * TILE_BYTES + L_BYTES;
  static constexpr int STAGES = MODE == ROWS_SWIGLU ? 3 : 4;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
  static constexpr int TMEM_COLS = 32;
  static constexpr int WORKERS = 256;
  static constexpr int THREADS = WORKERS + 32;
};

// Stage layout: [tile g][tile u][tile dH (backward)][L chunk(s)]
template <int MODE, int RP>
__global__ void __launch_bounds__(RowsSwigluCfg<MODE, RP>::THREADS)
    rows_swiglu_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmGU,
                       const __grid_constant__ CUtensorMap tmDH, const RowsParams p) {
  using C = RowsSwigluCfg<MODE, RP>;
  constexpr int S = C::STAGES;
  const int tile = blockIdx.x;
  if (tile >= *p.n_tiles) return;
  const TileInfo ti = p.tiles[tile];

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint64_t* infull = bars;          // [S] input tiles and L chunk landed
  uint64_t* afull = bars + S;       // [S] workers wrote the MMA operand
  uint64_t* sfree = bars + 2 * S;   // [S] the stage's MMAs completed
  uint64_t* acc_done = bars + 3 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&infull[s]), 1);
      mbar_init(smem_u32(&afull[s]), C::WORKERS);
      mbar_init(smem_u32(&sfree[s]), 1);
    }
    mbar_init(smem_u32(acc_done), 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmL);
    tma_prefetch_desc(&tmGU);
    if constexpr (MODE == ROWS_SWIGLU_BWD) tma_prefetch_desc(&tmDH);
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_it = (p.n + C::BK - 1) / C::BK;
  bool ok = true;

  if (warp < 8) {
    // ------------------------------------------------------------ workers
    const int cv = tid & 7;        // 16-byte column group of the 64-column stage
    const int rb = tid >> 3;       // rows rb + 32 j
    for (int it = 0; it < n_it; ++it) {
      const int s = it % S;
      if (ok) ok = mbar_wait(smem_u32(&infull[s]), (it / S) & 1, p.err);   // skip after a failure
      uint8_t* st = smem + s * C::STAGE_BYTES;
      const int col = it * C::BK + cv * 8;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = rb + 32 * j;
        // 128-byte swizzle: 16-byte group cv of row r sits at group cv ^ (r & 7)
        const uint32_t off = r * 128 + ((cv ^ (r & 7)) << 4);
        uint4* pg = reinterpret_cast<uint4*>(st + off);
        uint4* pu = reinterpret_cast<uint4*>(st + C::TILE_BYTES + off);
        const int q = ti.row0 + r;
        const bool valid = q < ti.row_end && col < p.n;
        float g[8], u[8];
        unpack8(*pg, g);
        unpack8(*pu, u);
        if constexpr (MODE == ROWS_SWIGLU) {
          float h[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) h[i] = __fdividef(g[i], 1.0f + __expf(-g[i])) * u[i];
          const uint4 o = pack8(h);
          *pg = o;
          if (valid) *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * p.n + col) = o;
        } else {
          float d[8], dg[8], du[8];
          unpack8(*reinterpret_cast<const uint4*>(st + 2 * C::TILE_BYTES + off), d);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float sg = __fdividef(1.0f, 1.0f + __expf(-g[i]));
            dg[i] = d[i] * u[i] * sg * (1.0f + g[i] * (1.0f - sg));
            du[i] = d[i] * g[i] * sg;
          }
          const uint4 o0 = pack8(dg), o1 = pack8(du);
          *pg = o0;
          *pu = o1;
          if (valid) {
            *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * p.n + col) = o0;
            *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * p.n + p.n + col) = o1;
          }
        }
      }
      mbar_arrive(smem_u32(&afull[s]));
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ control thread
    constexpr bool L_MN = MODE == ROWS_SWIGLU;   // A_d [E][n][rp]; B_gu [E][rp][2n]
    const uint32_t idesc = idesc_bf16(128, RP, 0, L_MN ? 1 : 0);
    auto load = [&](int it) {
      const int s = it % S;
      uint8_t* st = smem + s * C::STAGE_BYTES;
      const uint32_t fb = smem_u32(&infull[s]);
      const int c0 = it * C::BK;
      mbar_arrive_expect_tx(fb, C::NT * C::TILE_BYTES + C::L_BYTES);
      tma_load_2d(&tmGU, fb, smem_u32(st), c0, ti.row0);
      tma_load_2d(&tmGU, fb, smem_u32(st + C::TILE_BYTES), p.n + c0, ti.row0);
      if constexpr (MODE == ROWS_SWIGLU_BWD) tma_load_2d(&tmDH, fb, smem_u32(st + 2 * C::TILE_BYTES), c0, ti.row0);
      const uint32_t lb = smem_u32(st + C::NT * C::TILE_BYTES);
      if constexpr (L_MN) {
        tma_load_3d(&tmL, fb, lb, 0, c0, ti.e);
      } else {
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_3d(&tmL, fb, lb + h * (RP * C::BK * 2), (h == 0 ? 0 : p.n) + c0, 0, ti.e);
      }
    };
    for (int it = 0; it < S && it < n_it; ++it) load(it);
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it % S;
      ok = mbar_wait(smem_u32(&afull[s]), (it / S) & 1, p.err);
      if (!ok) break;
      fence_proxy_async_smem();     // worker smem writes -> tcgen05 reads (and later TMA writes)
      tc_fence_after();
      uint8_t* st = smem + s * C::STAGE_BYTES;
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h) {
        const uint32_t sa = smem_u32(st + h * C::TILE_BYTES);
        const uint32_t sl = smem_u32(st + C::NT * C::TILE_BYTES) + h * (RP * C::BK * 2);
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk) {
          const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024, kSw128);
          uint64_t bd;
          if constexpr (L_MN) {
            bd = (RP == 16) ? smem_desc(sl + kk * 16 * 32, RP * C::BK * 2, 256, kSw32)
                            : smem_desc(sl + kk * 16 * 64, RP * C::BK * 2, 512, kSw64);
          } else {
            bd = smem_desc(sl + kk * 32, 16, 1024, kSw128);
          }
          umma_bf16(tmem, ad, bd, idesc, (it | kk | h) ? 1u : 0u);
        }
      }
      umma_commit(smem_u32(&sfree[s]));
      // refill the slot of the previous iteration once its MMAs are done
      const int pv = it - 1;
      if (pv >= 0 && pv + S < n_it) {
        ok = mbar_wait(smem_u32(&sfree[pv % S]), (pv / S) & 1, p.err);
        if (ok) load(pv + S);
      }
    }
    umma_commit(smem_u32(acc_done));
  }

  // ---- epilogue: warps 0-3 read their TMEM lane quarter (row = tile row)
  if (warp < 4) {
    ok = mbar_wait(smem_u32(acc_done), 0, p.err) && ok;
    ok = __all_sync(0xffffffffu, ok);
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
        float x[8], xc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) { x[i] = v[8 * g + i]; xc[i] = p.scale * x[i]; }
        if (g * 8 < p.r_save) *reinterpret_cast<uint4*>(sv + 8 * g) = pack8(x);
        oc[g] = pack8(xc);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace moe
