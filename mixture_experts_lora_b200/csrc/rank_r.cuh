// Rank-r products of the Split-LoRA reordering: the compact [rows, r] intermediates
// that replace the E x K x N adapter delta ("Accelerating Mixture-of-Experts
// Fine-Tuning", Mathematical Formulation section 2, step 1):
//     LR[q] = Rows[q] L[e]        for every sorted row q of expert e,
// with, in this layer,
//     XA  = X A_gu      (rows gathered from X:  Rows[q] = X[sorted_pairs[q] / k])
//     HA  = H A_d       (sorted rows of H)
//     T1' = dY B_d^T    (rows gathered from dY; the routing weight is applied after)
//     T2  = dGU B_gu^T  (sorted rows of dGU)
// L is stored either [E][K][r] (A_gu, A_d: rank innermost, "MN-major" as the MMA's B
// operand) or [E][r][K] (B_d, B_gu: K innermost, "K-major").  Ranks below RP read as
// zero (the tensor map's out-of-range fill), so the padded columns of every output
// are exact zeros.
//
// One CTA per 128-row tile of one expert (the size-class-ordered tile table), K in
// 64-column stages through a ring of shared-memory slots:
//   * gathered rows: 256 worker threads copy 16-byte pieces of the tile's rows with
//     cp.async straight into the UMMA K-major 128-byte-swizzled layout, LOOK stages
//     ahead, wait for their own pieces, fence them to the async proxy and arrive;
//   * sorted rows: the control thread loads each stage's row tile with TMA;
//   * the control thread loads the stage's L chunk with TMA, issues the MMAs
//     LR[128 x RP] += Rows[128 x 64] L[64 x RP] into TMEM and commits them, which
//     frees the slot.
// The epilogue (warps 0-3, one tile row per thread) writes
//     out_save[q, 0:r_save] = bf16(v)      or bf16(w v) with save_w
//     out_c[q, 0:RP]        = bf16(scale v)
//     out_w[q, 0:RP]        = bf16(w wsrc[q])   (optional; wsrc has r_wsrc columns)
// where w is the routing weight of the row's pair.
#pragma once

#include "common.cuh"

namespace moe {

struct RankParams {
  const TileInfo* tiles;        // 128-row tiles {e, row0, row_end}
  const int* n_tiles;
  int K;                        // columns of the rows (multiple of 8)
  int n_it;                     // 64-column stages
  const __nv_bfloat16* src;     // gathered rows: [T, K]
  const int32_t* sorted_pairs;  // [P]
  int k;
  const float* w;               // [P] routing weights in pair order (save_w / out_w)
  __nv_bfloat16* out_save;      // [P, ld_save] or nullptr
  int ld_save, r_save;
  bool save_w;
  __nv_bfloat16* out_c;         // [P, RP]
  float scale;
  const __nv_bfloat16* wsrc;    // [P, r_wsrc] or nullptr
  int r_wsrc;
  __nv_bfloat16* out_w;         // [P, RP] or nullptr
  int* err;
};

template <int RP_, bool GATHER_, bool L_MN_>
struct RankCfg {
  static constexpr int RP = RP_;
  static constexpr bool GATHER = GATHER_, L_MN = L_MN_;
  static constexpr int BM = 128, BK = 64;
  static constexpr int TILE_BYTES = BM * BK * 2;           // 16 KB
  static constexpr int L_BYTES = RP * BK * 2;              // 2-16 KB
  static constexpr int STAGE_BYTES = TILE_BYTES + L_BYTES;
  static constexpr int STAGES = GATHER ? 6 : 4;
  static constexpr int LOOK = GATHER ? 4 : 0;              // gathered stages in flight
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
  static constexpr int TMEM_COLS = RP < 32 ? 32 : RP;
  static constexpr int WORKERS = 256;
  static constexpr int THREADS = WORKERS + 32;
  // L chunk as the MMA's B operand.  MN-major [64 K][RP]: rows of RP * 2 bytes up to
  // one 128-byte swizzle atom (RP <= 64), else two 64-rank atoms 8 KB apart.
  // K-major [RP][64 K]: 128-byte rows, one atom.
  static constexpr uint32_t LMN_SW = RP == 16 ? kSw32 : RP == 32 ? kSw64 : kSw128;
  static constexpr int LMN_ROWB = (RP < 64 ? RP : 64) * 2;
  static constexpr int LMN_ATOMS = RP > 64 ? 2 : 1;
  static constexpr int LMN_ATOM_BYTES = BK * LMN_ROWB;
  static_assert(RP == 16 || RP == 32 || RP == 64 || RP == 128, "RP");
  static_assert(LOOK < STAGES, "look-ahead");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C>
__global__ void __launch_bounds__(C::THREADS)
    rank_r_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmRows,
                  const RankParams p) {
  constexpr int RP = C::RP, S = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint64_t* rfull = bars;              // [S] gathered rows of the stage in place (8 warps)
  uint64_t* lfull = bars + S;          // [S] TMA bytes of the stage landed
  uint64_t* sfree = bars + 2 * S;      // [S] the stage's MMAs completed
  uint64_t* acc_done = bars + 3 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&rfull[s]), C::WORKERS / 32);
      mbar_init(smem_u32(&lfull[s]), 1);
      mbar_init(smem_u32(&sfree[s]), 1);
    }
    mbar_init(smem_u32(acc_done), 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmL);
    if constexpr (!C::GATHER) tma_prefetch_desc(&tmRows);
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();          // predecessors' outputs (tile table, rows) visible from here
  const int tile = blockIdx.x;
  const bool active = tile < *p.n_tiles;
  TileInfo ti{};
  if (active) ti = p.tiles[tile];
  const int n_it = p.n_it;
  bool ok = true;

  if (active && warp < 8) {
    if constexpr (C::GATHER) {
      // ---------------------------------------------------------- workers: gathered rows
      const int cv = tid & 7;        // 16-byte group of the 64-column stage
      const int rb = tid >> 3;       // rows rb + 32 j
      const __nv_bfloat16* srow[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = ti.row0 + rb + 32 * j;
        srow[j] = q < ti.row_end ? p.src + (size_t)(p.sorted_pairs[q] / p.k) * p.K : nullptr;
      }
      // Rows past the tile's end are not copied: each MMA row depends on its own row
      // only and those rows are never stored.  Columns past K of a real row are zero
      // (they meet the L chunk's zero rows; stale bits there could be NaN).
      auto issue = [&](int it) {
        uint8_t* st = smem + (it % S) * C::STAGE_BYTES;
        const int col = it * C::BK + cv * 8;
        const bool v = col < p.K;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (srow[j] == nullptr) continue;
          const int r = rb + 32 * j;
          cp_async_16(smem_u32(st + r * 128 + ((cv ^ (r & 7)) << 4)),
                      v ? (const void*)(srow[j] + col) : (const void*)p.src, v ? 16u : 0u);
        }
      };
#pragma unroll 1
      for (int j = 0; j < C::LOOK; ++j) {
        if (j < n_it) issue(j);
        cp_async_commit();
      }
#pragma unroll 1
      for (int it = 0; it < n_it; ++it) {
        const int nx = it + C::LOOK;
        if (nx < n_it) {
          // the slot was last read by the MMAs of stage nx - S
          if (ok && nx >= S) ok = mbar_wait(smem_u32(&sfree[nx % S]), ((nx - S) / S) & 1, p.err);
          if (ok) issue(nx);
        }
        cp_async_commit();
        cp_async_wait<C::LOOK>();                 // this thread's pieces of stage it landed
        fence_proxy_async_smem();                 // generic-proxy writes -> tcgen05 reads
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&rfull[it % S]));
      }
      cp_async_wait<0>();
    }
  } else if (active && warp == 8 && lane == 0) {
    // ------------------------------------------------------------ control thread
    const uint32_t idesc = idesc_bf16(128, RP, 0, C::L_MN ? 1 : 0);
    auto load = [&](int it) {
      const int s = it % S;
      uint8_t* st = smem + s * C::STAGE_BYTES;
      const uint32_t lb = smem_u32(st + C::TILE_BYTES);
      const uint32_t fb = smem_u32(&lfull[s]);
      mbar_arrive_expect_tx(fb, C::L_BYTES + (C::GATHER ? 0 : C::TILE_BYTES));
      if constexpr (C::L_MN) {
#pragma unroll
        for (int a = 0; a < C::LMN_ATOMS; ++a)
          tma_load_3d(&tmL, fb, lb + a * C::LMN_ATOM_BYTES, a * 64, it * C::BK, ti.e);
      } else {
        tma_load_3d(&tmL, fb, lb, it * C::BK, 0, ti.e);
      }
      if constexpr (!C::GATHER) tma_load_2d(&tmRows, fb, smem_u32(st), it * C::BK, ti.row0);
    };
    for (int it = 0; it < S && it < n_it; ++it) load(it);
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it % S;
      const uint32_t par = (it / S) & 1;
      ok = mbar_wait(smem_u32(&lfull[s]), par, p.err);
      if (ok && C::GATHER) ok = mbar_wait(smem_u32(&rfull[s]), par, p.err);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
      const uint32_t sl = sa + C::TILE_BYTES;
#pragma unroll
      for (int kk = 0; kk < C::BK / 16; ++kk) {
        const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024, kSw128);
        uint64_t bd;
        if constexpr (C::L_MN)
          bd = smem_desc(sl + kk * 16 * C::LMN_ROWB, C::LMN_ATOM_BYTES, 8 * C::LMN_ROWB, C::LMN_SW);
        else
          bd = smem_desc(sl + kk * 32, 16, 1024, kSw128);
        umma_bf16(tmem, ad, bd, idesc, (it | kk) ? 1u : 0u);
      }
      umma_commit(smem_u32(&sfree[s]));
      // refill the slot of the previous stage once its MMAs are done
      const int pv = it - 1;
      if (pv >= 0 && pv + S < n_it) {
        ok = mbar_wait(smem_u32(&sfree[pv % S]), (pv / S) & 1, p.err);
        if (ok) load(pv + S);
      }
    }
    umma_commit(smem_u32(acc_done));
  }

  // ---- epilogue: warps 0-3 read their TMEM lane quarter (row = tile row)
  if (active && warp < 4) {
    ok = mbar_wait(smem_u32(acc_done), 0, p.err) && ok;
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    const int row = ti.row0 + warp * 32 + lane;
    const bool live = ok && row < ti.row_end;
    float wq = 1.0f;
    if (live && (p.save_w || p.out_w != nullptr)) wq = p.w[p.sorted_pairs[row]];
#pragma unroll
    for (int c0 = 0; c0 < RP; c0 += 16) {
      uint32_t r16[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, r16);
      tmem_wait_ld();
      if (!live) continue;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int col = c0 + 8 * g;
        float x[8], xs[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[i] = __uint_as_float(r16[8 * g + i]);
          xs[i] = p.scale * x[i];
        }
        *reinterpret_cast<uint4*>(p.out_c + (size_t)row * RP + col) = pack8(xs);
        if (p.out_save != nullptr && col < p.r_save) {
          if (p.save_w) {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] *= wq;
          }
          *reinterpret_cast<uint4*>(p.out_save + (size_t)row * p.ld_save + col) = pack8(x);
        }
      }
    }
    if (live && p.out_w != nullptr) {
#pragma unroll
      for (int col = 0; col < RP; col += 8) {
        float x[8];
        if (col < p.r_wsrc) {
          unpack8(*reinterpret_cast<const uint4*>(p.wsrc + (size_t)row * p.r_wsrc + col), x);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] *= wq;
        *reinterpret_cast<uint4*>(p.out_w + (size_t)row * RP + col) = pack8(x);
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
