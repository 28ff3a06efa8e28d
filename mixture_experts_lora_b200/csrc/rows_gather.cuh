// Row gather of the grouped GEMM's token operand fused with the rank-r product of
// the Split-LoRA reordering ("Accelerating Mixture-of-Experts Fine-Tuning",
// Mathematical Formulation section 2, step 1: the compact [s, r] intermediate):
//     rows[q] = w[p] * src[p / k]   (w = 1 when no weights),  p = sorted_pairs[q]
//     LR[q]   = rows[q] L[e]        (L = A_gu for X forward, B_d^T for w * dY backward)
// One CTA owns a 128-row tile of one expert's sorted rows and walks K in 64-column
// stages through a ring of RG_STAGES shared-memory tiles:
//   * 256 worker threads copy their 16-byte pieces of the gathered rows with
//     cp.async straight into the UMMA K-major 128-byte-swizzled layout, two stages
//     ahead; once a stage has landed each worker scales its pieces (weighted mode),
//     writes them to rows_out and arrives on the stage's barrier;
//   * one control thread loads the stage's L chunk with TMA, issues the rank-r
//     MMAs LR[128 x RP] += rows[128 x 64] L[64 x RP] into TMEM and commits them,
//     which frees the stage.
// The epilogue writes LR unscaled (kept for the adapter gradients) and
// bf16(c * LR) (the LoRA operand of the grouped GEMM).
#pragma once

#include "common.cuh"
#include "rows_common.cuh"

namespace moe {

constexpr int RG_STAGES = 4;
constexpr int RG_LOOK = 2;      // stages of copies in flight ahead of the one being consumed
constexpr int RG_WORKERS = 256;
constexpr int RG_THREADS = RG_WORKERS + 32;   // + the control warp

template <int RP>
struct RowsGatherCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int TILE_BYTES = BM * BK * 2;   // 16 KB
  static constexpr int L_BYTES = RP * BK * 2;
  static constexpr int SMEM_BYTES = RG_STAGES * (TILE_BYTES + L_BYTES) + 256 + 1024;
  static constexpr int TMEM_COLS = 32;
};

template <int RP, bool L_MN>
__global__ void __launch_bounds__(RG_THREADS)
    rows_gather_kernel(const __grid_constant__ CUtensorMap tmL, const RowsParams p) {
  using C = RowsGatherCfg<RP>;
  pdl_begin();          // predecessors' outputs (tile table, rows) visible from here
  const int tile = blockIdx.x;
  if (tile >= *p.n_tiles) return;
  const TileInfo ti = p.tiles[tile];

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* lring = smem + RG_STAGES * C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(lring + RG_STAGES * C::L_BYTES);
  uint64_t* sfull = bars;                    // [S] all workers' pieces of the stage are in place
  uint64_t* sfree = bars + RG_STAGES;        // [S] the stage's MMAs completed
  uint64_t* lfull = bars + 2 * RG_STAGES;    // [S] L chunk landed
  uint64_t* acc_done = bars + 3 * RG_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  if (tid == 0) {
    for (int s = 0; s < RG_STAGES; ++s) {
      mbar_init(smem_u32(&sfull[s]), RG_WORKERS);
      mbar_init(smem_u32(&sfree[s]), 1);
      mbar_init(smem_u32(&lfull[s]), 1);
    }
    mbar_init(smem_u32(acc_done), 1);
    mbar_fence_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_it = p.nk;
  bool ok = true;

  if (warp < 8) {
    // ------------------------------------------------------------ workers
    const int cv = tid & 7;        // 16-byte column group of the 64-column stage
    const int rb = tid >> 3;       // rows rb + 32 j
    const __nv_bfloat16* srow[4];
    float wrow[4];
    int qrow[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = ti.row0 + rb + 32 * j;
      qrow[j] = q < ti.row_end ? q : -1;
      srow[j] = p.src;
      wrow[j] = 1.0f;
      if (qrow[j] >= 0) {
        const int pr = p.sorted_pairs[q];
        srow[j] = p.src + (size_t)(pr / p.k) * p.K;
        if (p.w != nullptr) wrow[j] = p.w[pr];
      }
    }
    // Rows past the tile's end are not copied: each MMA row depends on its own A row
    // only, and the rank-r rows of those rows are never stored.  Columns past K of a
    // real row are zero-filled: they meet the adapter chunk's zero rows, and stale
    // shared-memory bits there could be non-finite (NaN x 0 = NaN).
    auto issue = [&](int it) {
      uint8_t* st = smem + (it % RG_STAGES) * C::TILE_BYTES;
      const int col = it * C::BK + cv * 8;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (qrow[j] < 0) continue;
        const int r = rb + 32 * j;
        const bool v = col < p.K;
        // K-major, 128-byte swizzle: 16-byte group cv of row r lands at group cv ^ (r & 7)
        cp_async_16(smem_u32(st + r * 128 + ((cv ^ (r & 7)) << 4)),
                    v ? (const void*)(srow[j] + col) : (const void*)p.src, v ? 16u : 0u);
      }
    };
    // RG_LOOK stages ahead: the stage refilled at iteration it was last read by the
    // MMAs of iteration it + RG_LOOK - RG_STAGES, which have had time to complete
#pragma unroll
    for (int j = 0; j < RG_LOOK; ++j) {
      if (j < n_it) issue(j);
      cp_async_commit();
    }
    for (int it = 0; it < n_it; ++it) {
      const int nx = it + RG_LOOK;
      if (nx < n_it) {
        // after a failed wait the tile's results are discarded: stop waiting
        if (ok && nx >= RG_STAGES)
          ok = mbar_wait(smem_u32(&sfree[nx % RG_STAGES]), ((nx - RG_STAGES) / RG_STAGES) & 1, p.err);
        issue(nx);
      }
      cp_async_commit();
      cp_async_wait<RG_LOOK>();                  // this thread's pieces of stage it landed
      uint8_t* st = smem + (it % RG_STAGES) * C::TILE_BYTES;
      const int col = it * C::BK + cv * 8;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (qrow[j] < 0) continue;
        const int r = rb + 32 * j;
        uint4* sp = reinterpret_cast<uint4*>(st + r * 128 + ((cv ^ (r & 7)) << 4));
        uint4 v = *sp;
        if (wrow[j] != 1.0f) {
          float x[8];
          unpack8(v, x);
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] *= wrow[j];
          v = pack8(x);
          *sp = v;
        }
        if (col < p.K && p.rows_out != nullptr)
          *reinterpret_cast<uint4*>(p.rows_out + (size_t)qrow[j] * p.K + col) = v;
      }
      mbar_arrive(smem_u32(&sfull[it % RG_STAGES]));
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ control thread
    const uint32_t idesc = idesc_bf16(128, RP, 0, L_MN ? 1 : 0);
    auto load_l = [&](int it) {
      const int s = it % RG_STAGES;
      const uint32_t lb = smem_u32(lring + s * C::L_BYTES);
      mbar_arrive_expect_tx(smem_u32(&lfull[s]), C::L_BYTES);
      if constexpr (L_MN) tma_load_3d(&tmL, smem_u32(&lfull[s]), lb, 0, it * C::BK, ti.e);
      else tma_load_3d(&tmL, smem_u32(&lfull[s]), lb, it * C::BK, 0, ti.e);
    };
    for (int it = 0; it < RG_STAGES && it < n_it; ++it) load_l(it);
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it % RG_STAGES;
      const uint32_t par = (it / RG_STAGES) & 1;
      ok = mbar_wait(smem_u32(&sfull[s]), par, p.err) && mbar_wait(smem_u32(&lfull[s]), par, p.err);
      if (!ok) break;
      fence_proxy_async_smem();     // worker smem writes -> tcgen05 reads
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * C::TILE_BYTES);
      const uint32_t sl = smem_u32(lring + s * C::L_BYTES);
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
        umma_bf16(tmem, ad, bd, idesc, (it | kk) ? 1u : 0u);
      }
      umma_commit(smem_u32(&sfree[s]));
      // refill the L slot of the previous iteration once its MMAs are done
      const int pv = it - 1;
      if (pv >= 0 && pv + RG_STAGES < n_it) {
        ok = mbar_wait(smem_u32(&sfree[pv % RG_STAGES]), (pv / RG_STAGES) & 1, p.err);
        if (ok) load_l(pv + RG_STAGES);
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
