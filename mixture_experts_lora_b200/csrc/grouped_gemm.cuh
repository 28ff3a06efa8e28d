// Persistent grouped GEMM with fused Split-LoRA for sm_100a: CTA pairs
// (tcgen05 cta_group::2), TMEM accumulators, TMA loads and TMA stores.
//
// Orientation: output features on the MMA's M side, the expert's tokens on the N
// side.  A pair of CTAs computes 256 features (128 per CTA, each CTA's own TMEM)
// for a token chunk of at most 256 rows of one expert (granularity 16, each CTA
// holds half of the token rows, so a token row is read once per pair).  Each
// expert's rows are cut into balanced chunks, so the ragged end of an expert
// wastes at most 15 columns.  For a tile (token chunk of expert e, feature tile w):
//
//   D[f, t] = sum_k Wt[e][f, k] Act[t, k]  +  sum_j Lt[e][f, j] LRc[t, j]
//
// where Act is the activation matrix in expert order, Wt the weight oriented
// feature-major and LRc = bf16(c * Act L_A[e]) the rank-r product from the rank-r
// kernel; the second sum is one more K-block of the same accumulation.  This is
// Y = XW + (alpha/r)(XA)B of the Split-LoRA reordering ("Accelerating
// Mixture-of-Experts Fine-Tuning", Mathematical Formulation section 2) with no
// K x N adapter delta.
//
// The token operand is the expert-ordered [P, K] matrix (sorted X, H, w dY or dGU)
// loaded with TMA.
//
// Epilogues (EPI):
//   EPI_PLAIN    out[q, f] = bf16(D)
//   EPI_SWIGLU   the gate_up projection with the SwiGLU fused (h = silu(g) u, gate = first
//                n columns; Unsloth docs "What is torch._grouped_mm?", the expert's
//                gate_up output split in two): each CTA's 128 features are 64 gate
//                features and the 64 up features of the same indices, so g and u of a
//                token meet in one CTA; it writes GU (kept for the backward) and H.
//
// Roles (320 threads per CTA): warp 0 issues TMA loads (each CTA its own half,
// completing on the leader's barriers), warp 1 allocates TMEM and, in the leader CTA,
// issues tcgen05.mma for the pair; warps 2-9 drain TMEM (two warps per TMEM lane
// quarter, alternating 32-token blocks), transpose each 32 x 32 block through shared
// memory and store it with one TMA tensor store (16-byte stores for a chunk's ragged
// last block).  The accumulator is double buffered (2 x 256 fp32 columns) so the
// epilogue of one tile overlaps the K-loop of the next.
//
// Shared-memory operands (canonical UMMA layouts, per CTA):
//   A (weights)  forward, W stored [K][F]: MN-major, two 64-feature atoms of 128 K
//                rows, 128-byte swizzle; backward, W stored [F][K]: K-major,
//                [128 features][64 K] atoms, 128-byte swizzle
//   B (tokens)   two K atoms of [128 rows][64 K], K-major, 128-byte swizzle
//   LoRA block   A: L_B^T (forward [r][F]: MN-major; backward [F][r]: K-major), B: LRc
//                [N/2 rows][r], K-major; 32/64/128-byte swizzle by rank width, two
//                64-wide K atoms at rank 128.  At rank 16 the block has a double
//                buffer of its own; wider ranks take one ring stage per tile.
#pragma once

#include "common.cuh"

namespace moe {

enum GemmEpi : int { EPI_PLAIN = 0, EPI_SWIGLU = 1 };

struct GemmParams {
  const TileInfo* chunks;  // token chunks {e, row0, row_end}, at most 256 rows each
  const int* n_chunks;
  int F;                   // output features (EPI_SWIGLU: h-features n)
  int n_ftiles;            // feature tiles per chunk
  int nk;                  // K steps of 128 (the LoRA block follows them)
  int n;                   // expert intermediate size (SwiGLU epilogue)
  // outputs, for the ragged stores (the full blocks go through the tensor maps)
  __nv_bfloat16* out;      // PLAIN: [P, F]; SWIGLU: GU [P, 2n]
  __nv_bfloat16* out_h;    // SWIGLU: H [P, n]
  int* err;
};

// A_MN: weights stored [K][F] (MN-major A).  V: operands through atom views, one TMA
// copy per operand and stage; needs whole 64-wide atoms.  Otherwise two copies per
// operand.
template <bool A_MN_, int RP_, bool V_, int EPI_>
struct GemmCfg {
  static constexpr int RP = RP_;
  static constexpr bool A_MN = A_MN_, V = V_;
  static constexpr int EPI = EPI_;
  // BK = 128 per stage as two 64-wide K atoms (one 128-byte swizzle row each): a
  // stage carries 8 MMAs per wait and commit.  BOXR: token rows per LoRA-block copy.
  static constexpr int BM = 128, BK = 128, KA = 64, NMAX = 256, NHALF = NMAX / 2, BOXR = 64;
  static constexpr int A_BYTES = BM * BK * 2;          // 32 KB
  static constexpr int B_BYTES = NHALF * BK * 2;       // 32 KB
  static constexpr int ATOM_A = BM * KA * 2;           // 16 KB: one K atom of a K-major A
  static constexpr int ATOM_B = NHALF * KA * 2;        // 16 KB: one K atom of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BLK_BYTES = 32 * 32 * 2;        // one 32 x 32 bf16 staging block
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 32 * (2 + EPI_WARPS);
  static constexpr int EPI_BYTES = EPI_WARPS * BLK_BYTES;   // one transpose block per warp
  static constexpr int SMEM_LIMIT = 232448;
  // LoRA operands.  K-major atoms are LK_W ranks wide.
  static constexpr int LK_W = RP < 64 ? RP : 64;
  static constexpr int LK_ATOMS = RP > 64 ? 2 : 1;
  static constexpr uint32_t LK_SW = LK_W == 16 ? kSw32 : LK_W == 32 ? kSw64 : kSw128;
  static constexpr uint32_t LK_SBO = 8 * LK_W * 2;
  static constexpr int LA_ATOM = BM * LK_W * 2;             // K-major A atom (128 features)
  static constexpr int LR_ATOM = NHALF * LK_W * 2;          // K-major B atom (128 token rows)
  static constexpr int LA_BOX_BYTES = RP * 64 * 2;          // forward: RP rows x 64 features
  static constexpr int LA_BYTES = A_MN ? 2 * LA_BOX_BYTES : LK_ATOMS * LA_ATOM;
  static constexpr int LR_BOX_BYTES = BOXR * LK_W * 2;      // 64 token rows x LK_W ranks
  // LSIDE: at rank 16 the LoRA block's operands live in a double buffer of their own,
  // loaded at the start of a tile, instead of taking a whole ring stage per tile
  static constexpr bool LSIDE = RP == 16;
  static constexpr int LS_BYTES = LA_BYTES + LK_ATOMS * LR_ATOM;
  static constexpr int LS_TOTAL = LSIDE ? 2 * LS_BYTES : 0;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - EPI_BYTES - LS_TOTAL - 2048) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + LS_TOTAL + EPI_BYTES + 2048;
  static constexpr int TMEM_COLS = 512;
  static_assert(RP == 16 || RP == 32 || RP == 64 || RP == 128, "RP");
  static_assert(LA_BYTES <= A_BYTES && LK_ATOMS * LR_ATOM <= B_BYTES, "LoRA block fits a stage");
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory");
  static_assert(!(EPI == EPI_SWIGLU) || A_MN, "SwiGLU epilogue is the gate_up forward");
};

// Descriptor offset (in 16-byte units) of 16-wide K step kk inside K-major LoRA
// operand atoms of `atom_bytes` bytes, LK_W ranks wide.
template <class C>
__device__ __forceinline__ uint32_t lk_step(int kk, int atom_bytes) {
  const int k0 = kk * 16;
  return (uint32_t)((k0 / C::LK_W) * atom_bytes + (k0 % C::LK_W) * 2) >> 4;
}

// Stores one 32-token x 32-feature staging block (token-major rows of 64 bytes) at
// (column fcol of the tensor map, row grow).  A block with all 32 rows inside the
// chunk goes out as one TMA tensor store (columns past the map's width and rows past
// P clipped); the chunk's ragged last block, whose rows past the end belong to the
// next chunk, as 16-byte stores of its rows_left rows and columns below fmax, at
// base + row * ld + fcol.
__device__ __forceinline__ void epi_store_block(const CUtensorMap* tm, uint8_t* blk, int fcol,
                                                int grow, int rows_left, __nv_bfloat16* base,
                                                size_t ld, int fmax) {
  const int lane = lane_id();
  if (rows_left >= 32) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tm, smem_u32(blk), fcol, grow);
      bulk_commit_group();
    }
  } else {
    __syncwarp();
    const int rrow = lane >> 2, rpart = lane & 3;   // 8 rows x 4 parts per pass
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int rr = rrow + 8 * j;
      const int f = fcol + rpart * 8;
      if (rr < rows_left && f < fmax) {
        const uint4 x = *reinterpret_cast<const uint4*>(blk + rr * 64 + rpart * 16);
        *reinterpret_cast<uint4*>(base + (size_t)(grow + rr) * ld + f) = x;
      }
    }
  }
  __syncwarp();
}

// First feature (global column of W) of this CTA's 64-feature A box i for feature
// tile w (pair rank r): plain tiles cover 256 output features per pair; SwiGLU tiles
// cover 128 h-features per pair, each CTA 64 gate columns (box 0) and the 64 up
// columns n later (box 1).
template <class C>
__device__ __forceinline__ int feat_box(int w, int r, int i, int n) {
  if constexpr (C::EPI == EPI_SWIGLU) return w * 128 + r * 64 + i * n;
  else return w * 256 + r * 128 + i * 64;
}

// Token rows each CTA of the pair copies per K atom for a chunk whose half (rows per
// CTA, rounded up to 8) is `half`: with atom views the copy is cut to the chunk in
// steps of 32 rows (the MMA reads only the chunk's columns), else whole 128-row boxes.
template <class C>
__device__ __forceinline__ int act_box_rows(int half) {
  if constexpr (C::V) return half > 96 ? 128 : (half + 31) & ~31;
  else return C::NHALF;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmAct,
                    const __grid_constant__ CUtensorMap tmLW, const __grid_constant__ CUtensorMap tmLR,
                    const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmOut2,
                    const __grid_constant__ CUtensorMap tmOut3, const __grid_constant__ CUtensorMap tmAct32,
                    const __grid_constant__ CUtensorMap tmAct64, const __grid_constant__ CUtensorMap tmAct96,
                    const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t side_off = C::STAGES * C::STAGE_BYTES;   // LoRA side buffers (LSIDE)
  uint8_t* epi = smem + C::STAGES * C::STAGE_BYTES + C::LS_TOTAL;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi + C::EPI_BYTES);
  uint64_t* full = bars;                       // [STAGES] (used in the leader)
  uint64_t* empty = bars + C::STAGES;          // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2] (used in the leader)
  uint64_t* drain = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(acc_full + 6);
  uint64_t* lfull = acc_full + 8;              // [2] LoRA side buffer loaded (leader)
  uint64_t* lempty = acc_full + 10;            // [2] LoRA side buffer consumed

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  constexpr int NST = C::LSIDE ? 0 : 1;        // ring stages of the LoRA block per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 2 * C::EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&lfull[b]), 1);
      mbar_init(smem_u32(&lempty[b]), 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmLW);
    tma_prefetch_desc(&tmLR);
    if constexpr (C::V) {
      tma_prefetch_desc(&tmAct32);
      tma_prefetch_desc(&tmAct64);
      tma_prefetch_desc(&tmAct96);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();       // barriers of both CTAs exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();          // predecessors' outputs (chunk tables, operands) visible from here
  const int total = (*p.n_chunks) * p.n_ftiles;

  // Issue the LoRA block's copies (L_B^T rows of this CTA's features and its half of
  // the LRc rows) into the A and B areas at la / lr, completing on the leader's bar.
  auto load_lora = [&](uint32_t bar, uint32_t la, uint32_t lr, int w, int e, int r0, int nbh) {
    if constexpr (C::A_MN) {
      tma_load_3d_pair(&tmLW, bar, la, feat_box<C>(w, rank, 0, p.n), 0, e);
      tma_load_3d_pair(&tmLW, bar, la + C::LA_BOX_BYTES, feat_box<C>(w, rank, 1, p.n), 0, e);
    } else {
#pragma unroll
      for (int a = 0; a < C::LK_ATOMS; ++a)
        tma_load_3d_pair(&tmLW, bar, la + a * C::LA_ATOM, a * 64, feat_box<C>(w, rank, 0, p.n), e);
    }
#pragma unroll
    for (int a = 0; a < C::LK_ATOMS; ++a)
      for (int j = 0; j < nbh; ++j)
        tma_load_2d_pair(&tmLR, bar, lr + a * C::LR_ATOM + j * C::LR_BOX_BYTES, a * 64, r0 + j * C::BOXR);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // The whole warp waits (converged), lane 0 issues the copies.
    const uint32_t full_leader = mapa_smem(smem_u32(full), 0);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int it = 0;
    for (int t = pair; t < total && ok; t += npairs, ++it) {
      const int c = t / p.n_ftiles, w = t % p.n_ftiles;
      const TileInfo ch = p.chunks[c];
      const int half = ((((ch.row_end - ch.row0) + 15) & ~15) >> 1);
      const int nbh = (half + C::BOXR - 1) / C::BOXR;
      const int r0 = ch.row0 + (int)rank * half;
      const uint32_t lbytes = C::LA_BYTES + C::LK_ATOMS * nbh * C::LR_BOX_BYTES;
      const int brows = act_box_rows<C>(half);
      const CUtensorMap* tact = brows == 32 ? &tmAct32 : brows == 64 ? &tmAct64
                              : brows == 96 ? &tmAct96 : &tmAct;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      if constexpr (C::LSIDE) {
        // LoRA operands of this tile into side buffer it & 1
        const int lb = it & 1;
        const bool lok = mbar_wait(smem_u32(&lempty[lb]), ((it >> 1) & 1) ^ 1, p.err);
        if (!__all_sync(0xffffffffu, lok)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t la = s_base + side_off + lb * C::LS_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&lfull[lb]), 2 * lbytes);
          load_lora(mapa_smem(smem_u32(&lfull[lb]), 0), la, la + C::LA_BYTES, w, ch.e, r0, nbh);
        }
        __syncwarp();
      }
      for (int ks = 0; ks < p.nk + NST; ++ks) {
        const bool wok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err);
        if (!__all_sync(0xffffffffu, wok)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t fb = full_leader + stage * 8;
          const uint32_t sa = s_base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          if (ks < p.nk) {
            // the token copy covers the CTA's half of the chunk rounded up to its box
            // (rows past the chunk are loaded and ignored, rows past P and K past the
            // end read as zero)
            const int k0 = ks * C::BK;
            if (rank == 0)
              mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * (C::A_BYTES + brows * C::BK * 2));
            if constexpr (C::V) {
              if constexpr (C::EPI == EPI_SWIGLU)
                tma_load_5d_pair(&tmW, fb, sa, 0, k0, feat_box<C>(w, rank, 0, p.n) / 64, 0, ch.e);
              else if constexpr (C::A_MN)
                tma_load_4d_pair(&tmW, fb, sa, 0, k0, feat_box<C>(w, rank, 0, p.n) / 64, ch.e);
              else
                tma_load_4d_pair(&tmW, fb, sa, 0, feat_box<C>(w, rank, 0, p.n), k0 / C::KA, ch.e);
              tma_load_3d_pair(tact, fb, sb, 0, r0, k0 / C::KA);
            } else {
              if constexpr (C::A_MN) {
                tma_load_3d_pair(&tmW, fb, sa, feat_box<C>(w, rank, 0, p.n), k0, ch.e);
                tma_load_3d_pair(&tmW, fb, sa + C::A_BYTES / 2, feat_box<C>(w, rank, 1, p.n), k0, ch.e);
              } else {
                tma_load_3d_pair(&tmW, fb, sa, k0, feat_box<C>(w, rank, 0, p.n), ch.e);
                tma_load_3d_pair(&tmW, fb, sa + C::ATOM_A, k0 + C::KA, feat_box<C>(w, rank, 0, p.n), ch.e);
              }
              tma_load_2d_pair(&tmAct, fb, sb, k0, r0);
              tma_load_2d_pair(&tmAct, fb, sb + C::ATOM_B, k0 + C::KA, r0);
            }
          } else {
            if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * lbytes);
            load_lora(fb, sa, sb, w, ch.e, r0, nbh);
          }
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    // The whole warp waits (converged); lane 0 issues every MMA and commit, so each
    // commit tracks all MMAs issued before it.
    if (rank == 0) {
      // descriptors of stage 0, k-step 0 (A at the stage base, B after A)
      const uint64_t a_desc0 = C::A_MN ? smem_desc(s_base, C::A_BYTES / 2, 1024, kSw128)
                                       : smem_desc(s_base, 16, 1024, kSw128);
      const uint64_t b_desc0 = smem_desc(s_base + C::A_BYTES, 16, 1024, kSw128);
      const uint64_t la_desc0 = C::A_MN ? smem_desc(s_base, C::LA_BOX_BYTES, 1024, kSw128)
                                        : smem_desc(s_base, 16, C::LK_SBO, C::LK_SW);
      const uint64_t lr_desc0 = smem_desc(s_base + C::A_BYTES, 16, C::LK_SBO, C::LK_SW);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued_any = false;
      // the LoRA block's K steps at LoRA operands la (A) / lr (B) + offsets
      auto lora_mmas = [&](uint32_t d, uint64_t la0, uint64_t lr0, uint32_t idesc, bool first) {
#pragma unroll
        for (int kk = 0; kk < C::RP / 16; ++kk) {
          const uint32_t ao = C::A_MN ? (uint32_t)(kk * 2048) >> 4 : lk_step<C>(kk, C::LA_ATOM);
          umma_bf16_pair(d, la0 + ao, lr0 + lk_step<C>(kk, C::LR_ATOM), idesc,
                         (first && kk == 0) ? 0u : 1u);
        }
      };
      for (int t = pair; t < total && ok; t += npairs, ++it) {
        const int c = t / p.n_ftiles;
        const TileInfo ch = p.chunks[c];
        const int ncols = ((ch.row_end - ch.row0) + 15) & ~15;
        const uint32_t idesc = idesc_bf16(256, ncols, C::A_MN ? 1 : 0, 0);
        const int atom_b = act_box_rows<C>(ncols >> 1) * C::KA * 2;   // bytes between B's K atoms
        const int b = it & 1;
        const bool aok = mbar_wait(smem_u32(&acc_empty[b]), ((it >> 1) & 1) ^ 1, p.err);
        if (!__all_sync(0xffffffffu, aok)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + b * C::NMAX;
        if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
        for (int ks = 0; ks < p.nk + NST; ++ks) {
          const bool fok = mbar_wait(smem_u32(&full[stage]), phase, p.err);
          if (!__all_sync(0xffffffffu, fok)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            // descriptors: the 14-bit start-address field advances by (byte offset >> 4)
            const uint32_t so = (uint32_t)(stage * C::STAGE_BYTES) >> 4;
            if (ks < p.nk) {
#pragma unroll
              for (int kk = 0; kk < C::BK / 16; ++kk) {
                // K step kk: MN-major A advances 16 rows of 128 B; K-major operands
                // advance 32 B inside a K atom, atoms ATOM_* bytes apart
                const uint32_t ka = (uint32_t)((kk >> 2) * C::ATOM_A + (kk & 3) * 32) >> 4;
                const uint32_t kb = (uint32_t)((kk >> 2) * atom_b + (kk & 3) * 32) >> 4;
                umma_bf16_pair(d, a_desc0 + so + (C::A_MN ? kk * (2048 / 16) : ka), b_desc0 + so + kb,
                               idesc, (ks | kk) ? 1u : 0u);
              }
            } else {
              lora_mmas(d, la_desc0 + so, lr_desc0 + so, idesc, false);
            }
            umma_commit_pair(smem_u32(&empty[stage]), 0x3);
          }
          __syncwarp();
          issued_any = true;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if constexpr (C::LSIDE) {
          // the LoRA block last, from side buffer it & 1 (loaded when the tile's copies
          // began, so the tile starts on K stages already in the ring)
          const int lb = it & 1;
          const bool lok = mbar_wait(smem_u32(&lfull[lb]), (it >> 1) & 1, p.err);
          if (!__all_sync(0xffffffffu, lok)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t la = s_base + side_off + lb * C::LS_BYTES;
            const uint64_t la0 = C::A_MN ? smem_desc(la, C::LA_BOX_BYTES, 1024, kSw128)
                                         : smem_desc(la, 16, C::LK_SBO, C::LK_SW);
            lora_mmas(d, la0, smem_desc(la + C::LA_BYTES, 16, C::LK_SBO, C::LK_SW), idesc, false);
            umma_commit_pair(smem_u32(&lempty[lb]), 0x3);
          }
          __syncwarp();
        }
        if (lane == 0) umma_commit_pair(smem_u32(&acc_full[b]), 0x3);
        __syncwarp();
      }
      if (!ok && lane == 0) *abort_flag = 1;
      if (issued_any) {
        if (lane == 0) umma_commit_pair(smem_u32(drain), 0x1);
        __syncwarp();
        mbar_wait(smem_u32(drain), 0, p.err);
      }
    }
    __syncwarp();
  } else if (warp < 2 + C::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue (warps 2..9, both CTAs)
    const int q = warp & 3;                         // TMEM lane quarter of this warp
    const int hsel = (warp - 2) >> 2;               // which alternate 32-token blocks
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const uint32_t acc_empty_leader = mapa_smem(smem_u32(acc_empty), 0);
    uint8_t* blk = epi + (warp - 2) * C::BLK_BYTES; // 32 tokens x 32 features bf16, 64-byte rows
    // SwiGLU: lane quarters 0-1 hold gate features, 2-3 the up features of the same
    // indices; each gate warp pairs with the up warp two below it (same token blocks).
    const bool gate_w = q < 2;
    uint8_t* blk_up = epi + (warp - 4) * C::BLK_BYTES;              // gate warps only
    const int pbar = 2 + 2 * ((q & 1) + 2 * hsel);                  // 2,4,6,8 and +1
    if constexpr (C::EPI == EPI_SWIGLU) {
      if (gate_w) named_bar_arrive(pbar + 1, 64);   // the up warp may stage its first block
    }
    const size_t ldo = C::EPI == EPI_PLAIN ? (size_t)p.F : (size_t)2 * p.n;
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const int c = t / p.n_ftiles, w = t % p.n_ftiles;
      const TileInfo ch = p.chunks[c];
      const int nrows = ch.row_end - ch.row0;
      const int b = it & 1;
      // first feature of this warp: SwiGLU h-feature index, else the output column
      const int fq = C::EPI == EPI_SWIGLU ? w * 128 + (int)rank * 64 + (q & 1) * 32
                                          : w * 256 + (int)rank * 128 + q * 32;
      const bool ok = mbar_wait(smem_u32(&acc_full[b]), (it >> 1) & 1, p.err);
      if (named_bar_or(1, 32 * C::EPI_WARPS, !ok || *abort_flag != 0)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + b * C::NMAX;
      uint32_t v[32];
      for (int c0 = hsel * 32; c0 < nrows; c0 += 64) {
        tmem_ld32(acc + c0, v);
        tmem_wait_ld();
        const int grow = ch.row0 + c0;
        const int rows_left = nrows - c0;
        if (lane == 0) bulk_wait_read<0>();         // the last store from blk has read it
        __syncwarp();
        if constexpr (C::EPI == EPI_PLAIN) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            *reinterpret_cast<__nv_bfloat16*>(blk + i * 64 + lane * 2) = __float2bfloat16_rn(__uint_as_float(v[i]));
          epi_store_block(&tmOut, blk, fq, grow, rows_left, p.out, ldo, p.F);
        } else {
          if (!gate_w) {
            // u: stage it once the gate warp has read the previous block, store it
            // (GU columns n + f), then hand the staging block to the gate warp
            named_bar(pbar + 1, 64);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              *reinterpret_cast<__nv_bfloat16*>(blk + i * 64 + lane * 2) = __float2bfloat16_rn(__uint_as_float(v[i]));
            epi_store_block(&tmOut2, blk, fq, grow, rows_left, p.out + p.n, ldo, p.n);
            named_bar_arrive(pbar, 64);
          } else {
            // g: store it (GU columns f), then h = silu(g) u from the bf16-rounded g and
            // the up warp's staged u, stored to H
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const __nv_bfloat16 gb = __float2bfloat16_rn(__uint_as_float(v[i]));
              *reinterpret_cast<__nv_bfloat16*>(blk + i * 64 + lane * 2) = gb;
              v[i] = __float_as_uint(__bfloat162float(gb));
            }
            epi_store_block(&tmOut, blk, fq, grow, rows_left, p.out, ldo, p.n);
            named_bar(pbar, 64);                     // u staged
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float u = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(blk_up + i * 64 + lane * 2));
              const float a = 0.5f * __uint_as_float(v[i]);   // silu(g) = a (1 + tanh(a)), a = g / 2
              v[i] = __float_as_uint(fmaf(a, tanh_approx(a), a) * u);
            }
            named_bar_arrive(pbar + 1, 64);          // done with the up block
            if (lane == 0) bulk_wait_read<0>();      // the g store has read blk
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              *reinterpret_cast<__nv_bfloat16*>(blk + i * 64 + lane * 2) = __float2bfloat16_rn(__uint_as_float(v[i]));
            epi_store_block(&tmOut3, blk, fq, grow, rows_left, p.out_h, (size_t)p.n, p.n);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + b * 8);
    }
    if constexpr (C::EPI == EPI_SWIGLU) {
      if (!gate_w) named_bar(pbar + 1, 64);   // the gate warp's last hand-back
    }
    if (lane == 0) bulk_wait<0>();                        // every store of this warp complete
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();       // the peer's TMEM and barriers outlive every use by the leader
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

}  // namespace moe
