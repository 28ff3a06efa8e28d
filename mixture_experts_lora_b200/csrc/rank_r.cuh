// Rank-r products of the Split-LoRA reordering: the compact [rows, r] intermediates
// that replace the E x K x N adapter delta ("Accelerating Mixture-of-Experts
// Fine-Tuning", Mathematical Formulation section 2, step 1):
//     LR[q] = Rows[q] L[e]        for every sorted row q of expert e,
// in three modes:
//   RK_GATHER   Rows[q] = s_q src[sorted_pairs[q] / k] gathered from a token matrix
//               (s_q the routing weight of the row's pair when w is given, else 1),
//               and written out as the expert-ordered operand of the grouped GEMMs:
//               XA = X A_gu with the sorted X, T1 = (w dY) B_d^T with the sorted w dY
//   RK_SORTED   Rows = a sorted [P, K] matrix: HA = H A_d
//   RK_DSWIGLU  the SwiGLU backward, written out, with T2 = dGU B_gu^T:
//               dGU = [dH u s (1 + g (1 - s)), dH g s], s = sigmoid(g), [g | u] = GU
// L is stored either [E][K][r] (A_gu, A_d: rank innermost, "MN-major" as the MMA's B
// operand) or [E][r][K] (B_d, B_gu: K innermost, "K-major").  Ranks below RP read as
// zero (the tensor map's out-of-range fill), so the padded columns of every output
// are exact zeros.
//
// One CTA per 128-row tile of one expert (the size-class-ordered tile table), K in
// 64-column stages through a ring of shared-memory slots:
//   * RK_GATHER: 256 worker threads copy 16-byte pieces of the tile's rows with
//     cp.async straight into the UMMA K-major 128-byte-swizzled layout, LOOK stages
//     ahead; once its pieces of a stage have landed a worker scales them (weighted
//     rows) and arrives; thread 0 also loads each stage's L chunk with TMA.  The
//     staged rows go to the sorted output as one TMA tensor store per stage (full
//     tiles; the workers store a ragged tile's rows themselves);
//   * RK_SORTED: one thread loads each stage's row tile and L chunk with TMA;
//   * RK_DSWIGLU: a loader thread brings each stage's dH, g and u tiles and the two
//     L chunks (gate and up columns) with TMA; the workers compute dg and du in place
//     in the swizzled tiles, which thereby become the MMA operands and go to dGU as
//     two TMA tensor stores (the workers store a ragged tile's rows themselves);
//   * the control thread waits for the stage, issues the MMAs
//     LR[128 x RP] += Rows[128 x 64] L[64 x RP] into TMEM and commits them, which
//     frees the slot.
// The epilogue (warps 0-3, one tile row per thread) writes
//     out_save[q, 0:r_save] = bf16(v)
//     out_c[q, 0:RP]        = bf16(scale v)
#pragma once

#include "common.cuh"

namespace moe {

enum RankMode : int { RK_SORTED = 0, RK_GATHER = 1, RK_DSWIGLU = 2 };

struct RankParams {
  const TileInfo* tiles;        // 128-row tiles {e, row0, row_end}
  const int* n_tiles;
  int K;                        // columns of the rows (RK_DSWIGLU: n); multiple of 8
  int n_it;                     // 64-column stages
  const __nv_bfloat16* src;     // RK_GATHER: [T, K]
  const int32_t* sorted_pairs;  // [P]
  int k;
  const float* w;               // RK_GATHER: [P] routing weights in pair order, or nullptr
  __nv_bfloat16* rows_out;      // RK_GATHER: [P, K] sorted rows; RK_DSWIGLU: dGU [P, 2K]
  __nv_bfloat16* out_save;      // [P, ld_save] or nullptr
  int ld_save, r_save;
  __nv_bfloat16* out_c;         // [P, RP]
  float scale;
  int* err;
  TableBuild tb;                // RK_GATHER: tb.offsets set when this launch builds the
                                // call's tables (then its own tile comes from them)
};

template <int RP_, int MODE_, bool L_MN_>
struct RankCfg {
  static constexpr int RP = RP_, MODE = MODE_;
  static constexpr bool L_MN = L_MN_;
  static constexpr int BM = 128, BK = 64;
  static constexpr int TILE_BYTES = BM * BK * 2;           // 16 KB
  static constexpr int NT = MODE == RK_DSWIGLU ? 3 : 1;    // input tiles per stage
  static constexpr int HALVES = MODE == RK_DSWIGLU ? 2 : 1;  // MMA operand tiles per stage
  static constexpr int L_CHUNK = RP * BK * 2;              // 2-16 KB
  static constexpr int L_BYTES = HALVES * L_CHUNK;
  static constexpr int STAGE_BYTES = NT * TILE_BYTES + L_BYTES;
  // RK_GATHER: four stages (two of copies in flight) keep three CTAs on an SM at rank
  // 16; deeper rings cost that third CTA and were slower, three stages were no faster.
  // RK_DSWIGLU: two stages of three tiles keep two CTAs on an SM (one CTA of three or
  // four stages was 7-12% slower)
  static constexpr int STAGES_WANT = MODE == RK_DSWIGLU ? 2 : 4;
  static constexpr int STAGES_FIT = (232448 - 2048) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT < STAGES_WANT ? STAGES_FIT : STAGES_WANT;
  static constexpr int LOOK = MODE == RK_GATHER ? STAGES - 2 : 0;   // gathered stages in flight
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
  static constexpr int TMEM_COLS = RP < 32 ? 32 : RP;
  static constexpr int WORKERS = 256;
  static constexpr int THREADS = WORKERS + 64;             // + control warp + loader warp
  // L chunk as the MMA's B operand.  MN-major [64 K][RP]: rows of RP * 2 bytes up to
  // one 128-byte swizzle atom (RP <= 64), else two 64-rank atoms 8 KB apart.
  // K-major [RP][64 K]: 128-byte rows, one atom.
  static constexpr uint32_t LMN_SW = RP == 16 ? kSw32 : RP == 32 ? kSw64 : kSw128;
  static constexpr int LMN_ROWB = (RP < 64 ? RP : 64) * 2;
  static constexpr int LMN_ATOMS = RP > 64 ? 2 : 1;
  static constexpr int LMN_ATOM_BYTES = BK * LMN_ROWB;
  static_assert(RP == 16 || RP == 32 || RP == 64 || RP == 128, "RP");
  static_assert(MODE != RK_DSWIGLU || !L_MN, "the SwiGLU backward takes B_gu [E][r][2n]");
  static_assert(STAGES >= 2 && (MODE != RK_GATHER || STAGES >= 3), "pipeline depth");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C>
__global__ void __launch_bounds__(C::THREADS)
    rank_r_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmRows,
                  const __grid_constant__ CUtensorMap tmGU, const __grid_constant__ CUtensorMap tmOutG,
                  const __grid_constant__ CUtensorMap tmOutU, const RankParams p) {
  constexpr int RP = C::RP, S = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint64_t* rfull = bars;              // [S] workers' part of the stage in place
  uint64_t* lfull = bars + S;          // [S] TMA bytes of the stage landed
  uint64_t* sfree = bars + 2 * S;      // [S] the stage's MMAs completed
  uint64_t* acc_done = bars + 3 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&rfull[s]), C::WORKERS);
      mbar_init(smem_u32(&lfull[s]), 1);
      mbar_init(smem_u32(&sfree[s]), 1);
    }
    mbar_init(smem_u32(acc_done), 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmL);
    tma_prefetch_desc(&tmRows);
    if constexpr (C::MODE == RK_DSWIGLU) {
      tma_prefetch_desc(&tmGU);
      tma_prefetch_desc(&tmOutG);
      tma_prefetch_desc(&tmOutU);
    }
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();          // predecessors' outputs (offsets, tile table, rows) visible from here
  const int tile = blockIdx.x;
  bool active;
  TileInfo ti{};
  if (C::MODE == RK_GATHER && p.tb.offsets != nullptr) {
    __shared__ int s_scan[33];
    __shared__ unsigned long long s_scan64[33];
    __shared__ TileInfo s_tile;
    active = tile < build_tables_cta(p.tb, tile, (int)gridDim.x, &ti, s_scan, s_scan64, &s_tile);
  } else {
    active = tile < *p.n_tiles;
    if (active) ti = p.tiles[tile];
  }
  const int n_it = p.n_it;
  bool ok = true;
  // RK_GATHER and RK_DSWIGLU: a full tile's stages go out to rows_out as TMA tensor
  // stores issued by the control thread (the staged tiles are already in the store's
  // swizzled layout); the rows of a ragged last tile, whose neighbours belong to the
  // next tile, are stored by the workers
  const bool tma_rows = C::MODE != RK_SORTED && ti.row_end - ti.row0 == C::BM;

  // TMA bytes of stage it into slot it % S: the L chunk(s), plus the row tile(s) in the
  // TMA-fed modes
  auto load = [&](int it) {
    const int s = it % S;
    uint8_t* st = smem + s * C::STAGE_BYTES;
    const uint32_t fb = smem_u32(&lfull[s]);
    const uint32_t lb = smem_u32(st + C::NT * C::TILE_BYTES);
    const int c0 = it * C::BK;
    mbar_arrive_expect_tx(fb, C::L_BYTES + (C::MODE == RK_GATHER ? 0 : C::NT * C::TILE_BYTES));
    if constexpr (C::MODE == RK_DSWIGLU) {
      // dH [P, n] at column c0; g and u from GU [P, 2n] at columns c0 and n + c0
      tma_load_2d(&tmRows, fb, smem_u32(st + 2 * C::TILE_BYTES), c0, ti.row0);
      tma_load_2d(&tmGU, fb, smem_u32(st), c0, ti.row0);
      tma_load_2d(&tmGU, fb, smem_u32(st + C::TILE_BYTES), p.K + c0, ti.row0);
      // B_gu [E][r][2n]: rows of the gate columns, then of the up columns
      tma_load_3d(&tmL, fb, lb, c0, 0, ti.e);
      tma_load_3d(&tmL, fb, lb + C::L_CHUNK, p.K + c0, 0, ti.e);
    } else {
      if constexpr (C::L_MN) {
#pragma unroll
        for (int a = 0; a < C::LMN_ATOMS; ++a)
          tma_load_3d(&tmL, fb, lb + a * C::LMN_ATOM_BYTES, a * 64, c0, ti.e);
      } else {
        tma_load_3d(&tmL, fb, lb, c0, 0, ti.e);
      }
      if constexpr (C::MODE == RK_SORTED) tma_load_2d(&tmRows, fb, smem_u32(st), c0, ti.row0);
    }
  };

  if (active && warp < 8) {
    const int cv = tid & 7;        // 16-byte group of the 64-column stage
    const int rb = tid >> 3;       // rows rb + 32 j
    if constexpr (C::MODE == RK_GATHER) {
      // ---------------------------------------------------------- workers: gathered rows
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
      // Rows past the tile's end are not copied: each MMA row depends on its own row
      // only and those rows are never stored.  Columns past K of a real row are zero
      // (they meet the L chunk's zero rows; stale bits there could be NaN).
      auto issue = [&](int it) {
        uint8_t* st = smem + (it % S) * C::STAGE_BYTES;
        const int col = it * C::BK + cv * 8;
        const bool v = col < p.K;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (qrow[j] < 0) continue;
          const int r = rb + 32 * j;
          cp_async_16(smem_u32(st + r * 128 + ((cv ^ (r & 7)) << 4)),
                      v ? (const void*)(srow[j] + col) : (const void*)p.src, v ? 16u : 0u);
        }
      };
#pragma unroll 1
      for (int j = 0; j < C::LOOK; ++j) {
        if (j < n_it) {
          if (tid == 0) load(j);
          issue(j);
        }
        cp_async_commit();
      }
#pragma unroll 1
      for (int it = 0; it < n_it; ++it) {
        const int nx = it + C::LOOK;
        if (nx < n_it) {
          // the slot was last read by the MMAs of stage nx - S (after a failed wait
          // the tile's results are discarded: stop waiting)
          if (ok && nx >= S) ok = mbar_wait(smem_u32(&sfree[nx % S]), ((nx - S) / S) & 1, p.err);
          if (tid == 0) load(nx);
          issue(nx);
        }
        cp_async_commit();
        cp_async_wait<C::LOOK>();                 // this thread's pieces of stage it landed
        uint8_t* st = smem + (it % S) * C::STAGE_BYTES;
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
          if (!tma_rows && col < p.K)
            *reinterpret_cast<uint4*>(p.rows_out + (size_t)qrow[j] * p.K + col) = v;
        }
        fence_proxy_async_smem();                 // generic-proxy writes -> tcgen05 reads
        mbar_arrive(smem_u32(&rfull[it % S]));
      }
    } else if constexpr (C::MODE == RK_DSWIGLU) {
      // ---------------------------------------------------------- workers: SwiGLU backward
      const int n = p.K;
#pragma unroll 1
      for (int it = 0; it < n_it; ++it) {
        const int s = it % S;
        if (ok) ok = mbar_wait(smem_u32(&lfull[s]), (it / S) & 1, p.err);
        uint8_t* st = smem + s * C::STAGE_BYTES;
        const int col = it * C::BK + cv * 8;
        const bool in_n = col < n;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = rb + 32 * j;
          const int q = ti.row0 + r;
          // rows past the tile's end stay as loaded: their rank-r rows are never stored.
          // Columns past n are computed: dH reads as zero there, so dg and du are the
          // zeros the MMA needs against the adapter's columns beyond the gate (up) half.
          if (q >= ti.row_end) continue;
          // 128-byte swizzle: 16-byte group cv of row r sits at group cv ^ (r & 7)
          const uint32_t off = r * 128 + ((cv ^ (r & 7)) << 4);
          uint4* pg = reinterpret_cast<uint4*>(st + off);
          uint4* pu = reinterpret_cast<uint4*>(st + C::TILE_BYTES + off);
          float g[8], uu[8], d[8], dg[8], du[8];
          unpack8(*pg, g);
          unpack8(*pu, uu);
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
          if (in_n && !tma_rows) {
            *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * n + col) = o0;
            *reinterpret_cast<uint4*>(p.rows_out + (size_t)q * 2 * n + n + col) = o1;
          }
        }
        fence_proxy_async_smem();                 // generic-proxy writes -> tcgen05 reads
        mbar_arrive(smem_u32(&rfull[s]));
      }
    }
  } else if (active && warp == 9 && C::MODE != RK_GATHER) {
    // ------------------------------------------------------------ loader (TMA-fed modes)
    if (lane == 0) {
#pragma unroll 1
      for (int it = 0; it < n_it; ++it) {
        // the slot was last read by the MMAs of stage it - S
        if (it >= S && ok) ok = mbar_wait(smem_u32(&sfree[it % S]), ((it - S) / S) & 1, p.err);
        load(it);
      }
    }
    __syncwarp();
  } else if (active && warp == 8 && lane == 0) {
    // ------------------------------------------------------------ control thread
    const uint32_t idesc = idesc_bf16(128, RP, 0, C::L_MN ? 1 : 0);
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it % S;
      const uint32_t par = (it / S) & 1;
      ok = mbar_wait(smem_u32(&lfull[s]), par, p.err);
      if (ok && C::MODE != RK_SORTED) ok = mbar_wait(smem_u32(&rfull[s]), par, p.err);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
      const uint32_t sl = sa + C::NT * C::TILE_BYTES;
      if (tma_rows) {
        // columns past K (past n in each half of dGU) are clipped by the maps
        if constexpr (C::MODE == RK_GATHER) {
          tma_store_2d(&tmRows, sa, it * C::BK, ti.row0);
        } else if constexpr (C::MODE == RK_DSWIGLU) {
          tma_store_2d(&tmOutG, sa, it * C::BK, ti.row0);
          tma_store_2d(&tmOutU, sa + C::TILE_BYTES, it * C::BK, ti.row0);
        }
        bulk_commit_group();
      }
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h) {
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk) {
          const uint64_t ad = smem_desc(sa + h * C::TILE_BYTES + kk * 32, 16, 1024, kSw128);
          uint64_t bd;
          if constexpr (C::L_MN)
            bd = smem_desc(sl + kk * 16 * C::LMN_ROWB, C::LMN_ATOM_BYTES, 8 * C::LMN_ROWB, C::LMN_SW);
          else
            bd = smem_desc(sl + h * C::L_CHUNK + kk * 32, 16, 1024, kSw128);
          umma_bf16(tmem, ad, bd, idesc, (it | h | kk) ? 1u : 0u);
        }
      }
      // the slot is refilled once sfree fires: the store must have read it by then
      if (tma_rows) bulk_wait_read<0>();
      umma_commit(smem_u32(&sfree[s]));
    }
    umma_commit(smem_u32(acc_done));
    if (tma_rows) bulk_wait<0>();
  }

  // ---- epilogue: warps 0-3 read their TMEM lane quarter (row = tile row)
  if (active && warp < 4) {
    ok = mbar_wait(smem_u32(acc_done), 0, p.err) && ok;
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    const int row = ti.row0 + warp * 32 + lane;
    const bool live = ok && row < ti.row_end;
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
        if (p.out_save != nullptr && col < p.r_save)
          *reinterpret_cast<uint4*>(p.out_save + (size_t)row * p.ld_save + col) = pack8(x);
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
