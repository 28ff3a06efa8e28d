// SwiGLU row kernels of the layer fused with the rank-r products of the Split-LoRA
// reordering ("Accelerating Mixture-of-Experts Fine-Tuning", Mathematical
// Formulation section 2; gate = first n columns of GU, h = silu(g) * u):
//   ROWS_SWIGLU      H = silu(g) u                                   -> H,   HA = H A_d
//   ROWS_SWIGLU_BWD  dGU = [dH u s (1 + g (1 - s)), dH g s], s = sigmoid(g)
//                                                                    -> dGU, T2 = dGU B_gu^T
// Persistent: the (128-row tile, 64-column stage) units of the launch are split
// into equal contiguous ranges, one per CTA (rows_common.cuh), and each CTA walks
// its range through one ring of shared-memory stages:
//   * the control warp loads each stage's input tiles (g, u and for the backward
//     dH) with TMA in the 128-byte-swizzled K-major layout, with the stage's
//     adapter chunk, and issues the rank-r MMAs once the workers are done;
//   * 8 worker warps compute the activation (or its derivative) in place in the
//     swizzled tiles, which thereby become the MMA operand, and write the rows to
//     HBM;
//   * 4 epilogue warps drain the double-buffered TMEM accumulator of each tile
//     segment and write LR (unscaled, kept for the adapter gradients) and
//     bf16(c * LR) (the LoRA operand of the next grouped GEMM).
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
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 512 + 1024;
  static constexpr int CTAS_PER_SM = MODE == ROWS_SWIGLU ? 2 : 1;
  static constexpr int TMEM_COLS = 64;                           // 2 x RP accumulators
  static constexpr int WORKERS = 256;
  static constexpr int THREADS = WORKERS + 32 + 128;             // + control + epilogue warps
};

// Stage layout: [tile g][tile u][tile dH (backward)][L chunk(s)]
template <int MODE, int RP>
__global__ void __launch_bounds__(RowsSwigluCfg<MODE, RP>::THREADS, RowsSwigluCfg<MODE, RP>::CTAS_PER_SM)
    rows_swiglu_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmGU,
                       const __grid_constant__ CUtensorMap tmDH, const RowsParams p) {
  using C = RowsSwigluCfg<MODE, RP>;
  pdl_begin();          // predecessors' outputs (tile table, rows) visible from here
  constexpr int S = C::STAGES;
  const int n_it = (p.n + C::BK - 1) / C::BK;
  const int64_t U = (int64_t)(*p.n_tiles) * n_it;
  const int G = (int)(U < (int64_t)gridDim.x ? U : (int64_t)gridDim.x);
  const int cta = blockIdx.x;
  if (cta >= G) return;                         // every CTA below G owns at least one unit
  const int64_t beg = split_beg(U, G, cta), end = split_beg(U, G, cta + 1);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint64_t* infull = bars;            // [S] input tiles and L chunk landed
  uint64_t* afull = bars + S;         // [S] workers wrote the MMA operand
  uint64_t* sfree = bars + 2 * S;     // [S] the stage's MMAs completed
  uint64_t* acc_full = bars + 3 * S;  // [2] a segment's accumulation completed
  uint64_t* acc_empty = acc_full + 2; // [2] the epilogue read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 4);
  volatile int* flag = reinterpret_cast<volatile int*>(acc_full + 5);
  uint64_t* drain = acc_full + 6;     // all MMAs done (teardown)
  int4* slot_tile = reinterpret_cast<int4*>(bars + 32);      // [S] {row0, row_end, e, col0}

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&infull[s]), 1);
      mbar_init(smem_u32(&afull[s]), C::WORKERS);
      mbar_init(smem_u32(&sfree[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    mbar_init(smem_u32(drain), 1);
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

  if (warp < 8) {
    // ------------------------------------------------------------ workers
    const int cv = tid & 7;        // 16-byte column group of the 64-column stage
    const int rb = tid >> 3;       // rows rb + 32 j
    bool ok = true;
    for (int64_t u = beg; u < end; ++u) {
      const int gi = (int)(u - beg), s = gi % S;
      if (ok) ok = mbar_wait(smem_u32(&infull[s]), (gi / S) & 1, p.err);   // skip after a failure
      const int4 inf = slot_tile[s];
      uint8_t* st = smem + s * C::STAGE_BYTES;
      const int col = inf.w + cv * 8;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = rb + 32 * j;
        // 128-byte swizzle: 16-byte group cv of row r sits at group cv ^ (r & 7)
        const uint32_t off = r * 128 + ((cv ^ (r & 7)) << 4);
        uint4* pg = reinterpret_cast<uint4*>(st + off);
        uint4* pu = reinterpret_cast<uint4*>(st + C::TILE_BYTES + off);
        const int q = inf.x + r;
        // rows past the tile's end are left as loaded: their rank-r results are never
        // stored.  Columns past n are computed: with dH (or u) read as zero there they
        // become the zeros the rank-r product needs against the adapter's next columns.
        if (q >= inf.y) continue;
        const bool in_n = col < p.n;
        float g[8], uu[8];
        unpack8(*pg, g);
        unpack8(*pu, uu);
        if constexpr (MODE == ROWS_SWIGLU) {
          float h[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = 0.5f * g[i];          // silu(g) = a (1 + tanh(a)), a = g / 2
            h[i] = fmaf(a, tanh_approx(a), a) * uu[i];
          }
          const uint4 o = pack8(h);
          *pg = o;
          if (in_n) *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * p.n + col) = o;
        } else {
          float d[8], dg[8], du[8];
          unpack8(*reinterpret_cast<const uint4*>(st + 2 * C::TILE_BYTES + off), d);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float sg = fmaf(0.5f, tanh_approx(0.5f * g[i]), 0.5f);   // sigmoid(g)
            dg[i] = d[i] * uu[i] * sg * (1.0f + g[i] * (1.0f - sg));
            du[i] = d[i] * g[i] * sg;
          }
          const uint4 o0 = pack8(dg), o1 = pack8(du);
          *pg = o0;
          *pu = o1;
          if (in_n) {
            *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * p.n + col) = o0;
            *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * p.n + p.n + col) = o1;
          }
        }
      }
      mbar_arrive(smem_u32(&afull[s]));
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ control thread
    if (lane == 0) {
      constexpr bool L_MN = MODE == ROWS_SWIGLU;   // A_d [E][n][rp]; B_gu [E][rp][2n]
      const uint32_t idesc = idesc_bf16(128, RP, 0, L_MN ? 1 : 0);
      int ct = -1;
      TileInfo cti{};
      auto load = [&](int64_t u) {
        const int gi = (int)(u - beg), s = gi % S;
        const int t = (int)(u / n_it), c0 = (int)(u % n_it) * C::BK;
        if (t != ct) { cti = p.tiles[t]; ct = t; }
        slot_tile[s] = make_int4(cti.row0, cti.row_end, cti.e, c0);
        uint8_t* st = smem + s * C::STAGE_BYTES;
        const uint32_t fb = smem_u32(&infull[s]);
        mbar_arrive_expect_tx(fb, C::NT * C::TILE_BYTES + C::L_BYTES);
        tma_load_2d(&tmGU, fb, smem_u32(st), c0, cti.row0);
        tma_load_2d(&tmGU, fb, smem_u32(st + C::TILE_BYTES), p.n + c0, cti.row0);
        if constexpr (MODE == ROWS_SWIGLU_BWD)
          tma_load_2d(&tmDH, fb, smem_u32(st + 2 * C::TILE_BYTES), c0, cti.row0);
        const uint32_t lb = smem_u32(st + C::NT * C::TILE_BYTES);
        if constexpr (L_MN) {
          tma_load_3d(&tmL, fb, lb, 0, c0, cti.e);
        } else {
#pragma unroll
          for (int h = 0; h < C::HALVES; ++h)
            tma_load_3d(&tmL, fb, lb + h * (RP * C::BK * 2), (h == 0 ? 0 : p.n) + c0, 0, cti.e);
        }
      };
      for (int64_t u = beg; u < end && u < beg + S; ++u) load(u);
      int sidx = 0;
      bool ok = true, issued = false;
      for (int64_t u = beg; u < end && ok; ++u) {
        const int gi = (int)(u - beg), s = gi % S;
        const int it = (int)(u % n_it);
        const bool first = u == beg || it == 0, last = u == end - 1 || it == n_it - 1;
        const int b = sidx & 1;
        if (first) {
          ok = mbar_wait(smem_u32(&acc_empty[b]), ((sidx >> 1) & 1) ^ 1, p.err);
          tc_fence_after();
        }
        ok = ok && mbar_wait(smem_u32(&afull[s]), (gi / S) & 1, p.err);
        if (!ok) break;
        fence_proxy_async_smem();     // worker smem writes -> tcgen05 reads (and later TMA writes)
        tc_fence_after();
        uint8_t* st = smem + s * C::STAGE_BYTES;
        const uint32_t d = tmem + b * 32;
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
            umma_bf16(d, ad, bd, idesc, (first && h == 0 && kk == 0) ? 0u : 1u);
          }
        }
        issued = true;
        umma_commit(smem_u32(&sfree[s]));
        if (last) {
          umma_commit(smem_u32(&acc_full[b]));
          ++sidx;
        }
        // refill the slot of the previous unit once its MMAs are done
        const int pv = gi - 1;
        if (pv >= 0 && beg + pv + S < end) {
          ok = mbar_wait(smem_u32(&sfree[pv % S]), (pv / S) & 1, p.err);
          if (ok) load(beg + pv + S);
        }
      }
      if (issued) {                   // every MMA done before the teardown frees TMEM
        umma_commit(smem_u32(drain));
        mbar_wait(smem_u32(drain), 0, p.err);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps 9..12
    const int q4 = warp & 3;                  // TMEM lane quarter
    const int et = (warp - 9) * 32 + lane;    // 0..127
    const int rin = q4 * 32 + lane;           // tile row of this thread
    const int t_beg = (int)(beg / n_it), t_end = (int)((end - 1) / n_it);
    int sidx = 0;
    for (int t = t_beg; t <= t_end; ++t, ++sidx) {
      const int64_t sb = beg > (int64_t)t * n_it ? beg : (int64_t)t * n_it;
      const int64_t se = end < (int64_t)(t + 1) * n_it ? end : (int64_t)(t + 1) * n_it;
      const bool whole = sb == (int64_t)t * n_it && se == (int64_t)(t + 1) * n_it;
      const int b = sidx & 1;
      const bool ok = mbar_wait(smem_u32(&acc_full[b]), (sidx >> 1) & 1, p.err);
      if (named_bar_or(1, 128, !ok)) break;     // the same branch in every epilogue warp
      tc_fence_after();
      float v[RP];
      if constexpr (RP == 16) {
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(q4 * 32) << 16) + b * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
      } else {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + b * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
      rows_segment_epilogue<RP>(p, v, et, rin, t, whole, cta, t == t_beg ? 0 : 1, U, G, n_it, 2, flag);
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
