// Row producers of the grouped GEMMs fused with the rank-r products of the
// Split-LoRA reordering ("Accelerating Mixture-of-Experts Fine-Tuning",
// Mathematical Formulation section 2, step 1: the compact [s, r] intermediate).
//
// One CTA owns a 128-row tile of one expert's sorted rows.  For each 64-column
// K-chunk the CTA's threads build the rows in registers, write them to HBM (they
// are the next grouped GEMM's token operand) and into shared memory in the UMMA
// K-major 128-byte-swizzled layout; one thread then issues the tcgen05 MMAs
//     LR[128 x RP] += Rows[128 x 64] L[e][64 x RP]
// while the threads build the next chunk (double-buffered).  Modes:
//   ROWS_GATHER     rows = src[p / k] (optionally times w[p]), p = sorted_pairs[q]:
//                   X for the gate_up GEMM (L = A_gu), w * dY for the down backward (L = B_d^T)
//   ROWS_SWIGLU     rows = silu(g) * u from GU = [g | u]: H for the down GEMM (L = A_d)
//   ROWS_SWIGLU_BWD rows = [dH u s (1 + g (1 - s)) | dH g s], s = sigmoid(g): dGU for the
//                   gate_up backward (L = B_gu^T)
// The epilogue writes LR unscaled (kept for the adapter gradients) and
// bf16(c * LR) (the LoRA operand of the grouped GEMM).
#pragma once

#include "common.cuh"

namespace moe {

enum RowsMode : int { ROWS_GATHER = 0, ROWS_SWIGLU = 1, ROWS_SWIGLU_BWD = 2 };

struct RowsParams {
  const TileInfo* tiles;   // 128-row tiles {e, row0, row_end}
  const int* n_tiles;
  int K;                   // columns of the rows (m, n or 2n)
  int nk;                  // K chunks of 64
  // ROWS_GATHER
  const __nv_bfloat16* src;   // [T, K]
  const int32_t* sorted_pairs;
  const float* w;             // [P] or nullptr
  int k;
  // ROWS_SWIGLU / ROWS_SWIGLU_BWD
  const __nv_bfloat16* gu;    // [P, 2n]
  const __nv_bfloat16* dh;    // [P, n]
  int n;
  // outputs
  __nv_bfloat16* rows_out;    // [P, K] (or nullptr)
  float scale;
  __nv_bfloat16* save;        // [P, ld_save]: first r_save columns of LR
  int ld_save;
  int r_save;
  __nv_bfloat16* outc;        // [P, RP]: bf16(scale * LR)
  int* err;
};

template <int MODE, int RP, bool L_MN>
struct RowsCfg {
  static constexpr int BM = 128, BK = 64, THREADS = 512, PASSES = BM * 8 / THREADS;
  static constexpr int HALVES = MODE == ROWS_SWIGLU_BWD ? 2 : 1;   // dg and du chunks together
  static constexpr int A_BYTES = HALVES * BM * BK * 2;
  static constexpr int L_BYTES = HALVES * RP * BK * 2;
  static constexpr int L_RING = 4;                     // L chunks loaded two iterations ahead
  static constexpr int BUF_BYTES = A_BYTES;
  static constexpr int NT = MODE == ROWS_GATHER ? 1 : (MODE == ROWS_SWIGLU ? 2 : 3);  // input tensors
  static constexpr int TILE_BYTES = BM * BK * 2;
  static constexpr int IN_STAGES = 2;
  static_assert(IN_STAGES >= 2, "input ring");
  static constexpr int IN_BYTES = IN_STAGES * NT * TILE_BYTES;
  static constexpr int SMEM_BYTES = 2 * A_BYTES + L_RING * L_BYTES + IN_BYTES + 256 + 1024;
  static constexpr int TMEM_COLS = 32;
};

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint4 o;
  o.x = pack_bf16x2(x[0], x[1]);
  o.y = pack_bf16x2(x[2], x[3]);
  o.z = pack_bf16x2(x[4], x[5]);
  o.w = pack_bf16x2(x[6], x[7]);
  return o;
}
__device__ __forceinline__ void unpack8(uint4 v, float (&x)[8]) {
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x);
  x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z);
  x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}

template <int MODE, int RP, bool L_MN>
__global__ void __launch_bounds__(512)
    rows_lowrank_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmGU,
                        const __grid_constant__ CUtensorMap tmDH, const RowsParams p) {
  using C = RowsCfg<MODE, RP, L_MN>;
  const int tile = blockIdx.x;
  if (tile >= *p.n_tiles) return;
  const TileInfo ti = p.tiles[tile];

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* lring = smem + 2 * C::A_BYTES;
  uint8_t* in_ring = lring + C::L_RING * C::L_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(in_ring + C::IN_BYTES);
  uint64_t* lfull = bars;        // [L_RING] L chunk landed
  uint64_t* mdone = bars + C::L_RING;    // [2] MMAs of iteration it (parity it/2) finished
  uint64_t* infull = bars + C::L_RING + 2;  // [IN_STAGES] input tiles landed (TMA modes)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::L_RING + 2 + C::IN_STAGES);

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  if (tid == 0) {
    for (int b = 0; b < C::L_RING; ++b) mbar_init(smem_u32(&lfull[b]), 1);
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&mdone[b]), 1);
    for (int b = 0; b < C::IN_STAGES; ++b) mbar_init(smem_u32(&infull[b]), 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmL);
    if constexpr (MODE != ROWS_GATHER) tma_prefetch_desc(&tmGU);
    if constexpr (MODE == ROWS_SWIGLU_BWD) tma_prefetch_desc(&tmDH);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_bf16(128, RP, 0, L_MN ? 1 : 0);

  // thread -> (row, 16-byte column group) of the 128 x 64 chunk, PASSES passes of 64 rows
  const int cv = tid & 7;
  const int rbase = tid >> 3;
  bool ok = true;
  // iterations: 64 columns each (SWIGLU_BWD: 64 gate + the matching 64 up columns)
  const int n_it = MODE == ROWS_SWIGLU_BWD ? (p.n + C::BK - 1) / C::BK : p.nk;

  // source rows of this thread's rows (hoisted out of the column loop)
  const __nv_bfloat16* srow[C::PASSES];
  float wrow[C::PASSES];
  bool rvalid[C::PASSES];
#pragma unroll
  for (int pass = 0; pass < C::PASSES; ++pass) {
    const int q = ti.row0 + rbase + pass * 64;
    rvalid[pass] = q < ti.row_end;
    wrow[pass] = 1.0f;
    srow[pass] = p.gu != nullptr ? p.gu : p.src;
    if constexpr (MODE == ROWS_GATHER) {
      if (rvalid[pass]) {
        const int pr = p.sorted_pairs[q];
        srow[pass] = p.src + (size_t)(pr / p.k) * p.K;
        if (p.w != nullptr) wrow[pass] = p.w[pr];
      }
    }
  }

  auto load_l = [&](int it) {   // L chunk(s) of iteration it into ring slot it % L_RING (thread 0)
    const int b = it % C::L_RING;
    const uint32_t lb = smem_u32(lring + b * C::L_BYTES);
    mbar_arrive_expect_tx(smem_u32(&lfull[b]), C::L_BYTES);
#pragma unroll
    for (int h = 0; h < C::HALVES; ++h) {
      const int k0 = (h == 0 ? 0 : p.n) + it * C::BK;
      const uint32_t dst = lb + h * (RP * C::BK * 2);
      if constexpr (L_MN) tma_load_3d(&tmL, smem_u32(&lfull[b]), dst, 0, k0, ti.e);
      else tma_load_3d(&tmL, smem_u32(&lfull[b]), dst, k0, 0, ti.e);
    }
  };

  // Input ring: IN_STAGES x NT tensors x [128 rows][64 columns] (no swizzle); each
  // thread copies and later reads back only its own 16-byte pieces, so its
  // cp.async groups need no block-level synchronisation.
  auto issue_loads = [&](int it) {
    const int col = it * C::BK + cv * 8;
    uint8_t* st = in_ring + (it % C::IN_STAGES) * (C::NT * C::TILE_BYTES);
    if constexpr (MODE == ROWS_GATHER) {
#pragma unroll
      for (int pass = 0; pass < C::PASSES; ++pass) {
        const int r = rbase + pass * 64;
        const uint32_t off = r * 128 + cv * 16;
        const bool v = rvalid[pass] && col < p.K;
        cp_async_16(smem_u32(st + off), v ? (const void*)(srow[pass] + col) : (const void*)p.src, v ? 16u : 0u);
      }
    } else if (tid == 0) {
      // whole 128 x 64 tiles of the expert-sorted rows (rows past P read as zero)
      const uint32_t fb = smem_u32(&infull[it % C::IN_STAGES]);
      const int c0 = it * C::BK;
      mbar_arrive_expect_tx(fb, C::NT * C::TILE_BYTES);
      if constexpr (MODE == ROWS_SWIGLU) {
        tma_load_2d(&tmGU, fb, smem_u32(st), c0, ti.row0);
        tma_load_2d(&tmGU, fb, smem_u32(st + C::TILE_BYTES), p.n + c0, ti.row0);
      } else {
        tma_load_2d(&tmDH, fb, smem_u32(st), c0, ti.row0);
        tma_load_2d(&tmGU, fb, smem_u32(st + C::TILE_BYTES), c0, ti.row0);
        tma_load_2d(&tmGU, fb, smem_u32(st + 2 * C::TILE_BYTES), p.n + c0, ti.row0);
      }
    }
  };

  if (tid == 0) {
    load_l(0);
    if (n_it > 1) load_l(1);
  }
#pragma unroll
  for (int j = 0; j < C::IN_STAGES - 1; ++j) {
    if (j < n_it) issue_loads(j);
    if constexpr (MODE == ROWS_GATHER) cp_async_commit();
  }

  for (int it = 0; it < n_it; ++it) {
    const int b = it & 1;
    uint8_t* abuf = smem + b * C::A_BYTES;
    if (it + C::IN_STAGES - 1 < n_it) issue_loads(it + C::IN_STAGES - 1);
    if constexpr (MODE == ROWS_GATHER) {
      cp_async_commit();
      cp_async_wait<C::IN_STAGES - 1>();               // this thread's pieces have landed
    } else {
      ok = mbar_wait(smem_u32(&infull[it % C::IN_STAGES]), (it / C::IN_STAGES) & 1, p.err) && ok;
    }
    // A buffer b and L slot (it + 2) % L_RING were last read by the MMAs of iteration it - 2
    if (it >= 2) ok = mbar_wait(smem_u32(&mdone[b]), ((it - 2) >> 1) & 1, p.err) && ok;
    if (tid == 0 && it + 2 < n_it) load_l(it + 2);
    const int col = it * C::BK + cv * 8;
    const uint8_t* st = in_ring + (it % C::IN_STAGES) * (C::NT * C::TILE_BYTES);
    uint4 out0[C::PASSES], out1[C::PASSES];
#pragma unroll
    for (int pass = 0; pass < C::PASSES; ++pass) {
      const int r = rbase + pass * 64;
      const uint32_t off = r * 128 + cv * 16;
      uint4 o0 = make_uint4(0, 0, 0, 0), o1 = make_uint4(0, 0, 0, 0);
      if constexpr (MODE == ROWS_GATHER) {
        o0 = *reinterpret_cast<const uint4*>(st + off);
        if (wrow[pass] != 1.0f) {
          float x[8];
          unpack8(o0, x);
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] *= wrow[pass];
          o0 = pack8(x);
        }
      } else if constexpr (MODE == ROWS_SWIGLU) {
        float g[8], u[8], h[8];
        unpack8(*reinterpret_cast<const uint4*>(st + off), g);
        unpack8(*reinterpret_cast<const uint4*>(st + C::TILE_BYTES + off), u);
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = __fdividef(g[i], 1.0f + __expf(-g[i])) * u[i];
        o0 = pack8(h);
      } else {
        float d[8], g[8], u[8], dg[8], du[8];
        unpack8(*reinterpret_cast<const uint4*>(st + off), d);
        unpack8(*reinterpret_cast<const uint4*>(st + C::TILE_BYTES + off), g);
        unpack8(*reinterpret_cast<const uint4*>(st + 2 * C::TILE_BYTES + off), u);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float s = __fdividef(1.0f, 1.0f + __expf(-g[i]));
          dg[i] = d[i] * u[i] * s * (1.0f + g[i] * (1.0f - s));
          du[i] = d[i] * g[i] * s;
        }
        o0 = pack8(dg);
        o1 = pack8(du);
      }
      out0[pass] = o0;
      out1[pass] = o1;
      // K-major, 128-byte swizzle: 16-byte group cv of row r lands at group cv ^ (r & 7)
      *reinterpret_cast<uint4*>(abuf + r * 128 + ((cv ^ (r & 7)) << 4)) = o0;
      if constexpr (C::HALVES == 2)
        *reinterpret_cast<uint4*>(abuf + C::BM * C::BK * 2 + r * 128 + ((cv ^ (r & 7)) << 4)) = o1;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      ok = mbar_wait(smem_u32(&lfull[it % C::L_RING]), (it / C::L_RING) & 1, p.err) && ok;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h) {
        const uint32_t sa = smem_u32(abuf) + h * (C::BM * C::BK * 2);
        const uint32_t sl = smem_u32(lring + (it % C::L_RING) * C::L_BYTES) + h * (RP * C::BK * 2);
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
      umma_commit(smem_u32(&mdone[b]));
    }
    // the rows themselves go to HBM after the shared-memory hand-off
#pragma unroll
    for (int pass = 0; pass < C::PASSES; ++pass) {
      const int q = ti.row0 + rbase + pass * 64;
      if constexpr (MODE == ROWS_GATHER) {
        if (rvalid[pass] && col < p.K && p.rows_out != nullptr)
          *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * p.K + col) = out0[pass];
      } else if constexpr (MODE == ROWS_SWIGLU) {
        if (rvalid[pass] && col < p.n) *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * p.n + col) = out0[pass];
      } else {
        if (rvalid[pass] && col < p.n) {
          *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * p.n + col) = out0[pass];
          *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * p.n + p.n + col) = out1[pass];
        }
      }
    }
  }

  // ---- epilogue: warps 0-3 read their TMEM lane quarter
  const int last = n_it - 1;
  ok = mbar_wait(smem_u32(&mdone[last & 1]), (last >> 1) & 1, p.err) && ok;
  if (warp < 4) {
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
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace moe
