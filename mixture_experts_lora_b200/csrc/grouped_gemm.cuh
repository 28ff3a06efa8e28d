// Persistent grouped GEMM with fused Split-LoRA for sm_100a: CTA pairs
// (tcgen05 cta_group::2), TMEM accumulators, TMA loads and TMA stores.
//
// Orientation: output features on the MMA's M side, the expert's tokens on the N
// side.  A pair of CTAs computes 256 features (128 per CTA, each CTA's own TMEM)
// for a token chunk of at most 256 rows of one expert (granularity 16, each CTA
// loads half of the token rows, so a token row is read once per pair).  Each
// expert's rows are cut into balanced chunks, so the ragged end of an expert
// wastes at most 15 columns.  For a tile (token chunk of expert e, feature tile w):
//
//   D[f, t] = sum_k Wt[e][f, k] Act[t, k]  +  sum_r Lt[e][f, r] LRc[t, r]
//
// where Act is the expert-sorted activation matrix, Wt the weight oriented
// feature-major and LRc = bf16(c * Act L_A[e]) the rank-r product from the
// row kernel; the second sum is one extra K-block of the same pipeline.
// This is Y = XW + (alpha/r)(XA)B of the Split-LoRA reordering ("Accelerating
// Mixture-of-Experts Fine-Tuning", Mathematical Formulation section 2) with no
// K x N adapter delta.
//
// Roles (320 threads per CTA): warp 0 issues TMA loads (each CTA its own half,
// completing on the leader's barriers), warp 1 allocates TMEM and, in the leader
// CTA, issues tcgen05.mma for the pair; warps 2-9 drain TMEM (two warps per TMEM
// lane quarter, alternating 32-token chunks), transpose each 32 x 32 block through
// shared memory and write it to the [tokens, features] output with one TMA tensor
// store (16-byte stores for a chunk's ragged last block).  The
// accumulator is double buffered (2 x 256 fp32 columns) so the epilogue of one
// tile overlaps the K-loop of the next.
//
// Shared-memory operands (canonical UMMA layouts, per CTA):
//   A (weights)  forward, W stored [K][F]: MN-major, two 64-feature atoms of 64 K
//                rows, 128-byte swizzle (one TMA copy through a 4-D view when
//                F % 64 == 0); backward, W stored [F][K]: K-major,
//                [128 features][64 K], 128-byte swizzle
//   B (tokens)   two K atoms of [128 rows][64 K], K-major, 128-byte swizzle
// Each stage costs the two issuing threads a fixed number of instructions
// (waits, TMA copies, MMAs, a commit), so the loaders use as few copies per stage
// as the layouts allow and the MMA descriptors are advanced by offsets.
//   LoRA block   A: L_B^T (forward [r][F]: MN-major; backward [F][r]: K-major,
//                32/64-byte swizzle); B: LRc [N/2 rows][r], K-major, 32/64-byte swizzle
#pragma once

#include "common.cuh"

namespace moe {

struct GemmParams {
  const TileInfo* chunks;  // token chunks {e, row0, row_end}, at most 256 rows each
  const int* n_chunks;
  int F;                   // output features
  int n_ftiles;            // feature tiles (256 features per pair) per chunk
  int nk;                  // K steps of 128 (the LoRA block is step nk)
  __nv_bfloat16* out;      // [P, F] in sorted token order
  int* err;
};

// A_MN: weights stored [K][F] (MN-major A).  V: operands through atom views, one
// TMA copy per operand and stage: the weight tile via a 4-D view (64-wide atom,
// rows, atom index, expert) and the token tile via a 3-D view (64-wide K atom,
// rows, atom index); needs K % 64 == 0 (and F % 64 == 0 for MN-major weights).
// Otherwise two copies per operand.
template <bool A_MN_, int RP_, bool V_ = false>
struct GemmCfg {
  static constexpr int RP = RP_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool V = V_;
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
  static constexpr int EPI_BYTES = EPI_WARPS * BLK_BYTES;   // one transpose block per warp
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int LA_BOX_BYTES = RP * 64 * 2;          // forward: 64 features x RP rows
  static constexpr int LA_BYTES = A_MN ? 2 * LA_BOX_BYTES : BM * RP * 2;
  static constexpr int LR_BOX_BYTES = BOXR * RP * 2;        // 64 token rows x RP
  // LSIDE: the LoRA block's operands (LA: L_B^T, LR: c*LR rows) live in a double
  // buffer of their own, loaded at the start of a tile, instead of taking a whole
  // ring stage per tile (fits beside three stages for RP = 16)
  static constexpr bool LSIDE = RP == 16;
  static constexpr int LS_BYTES = LA_BYTES + NHALF * RP * 2;
  static constexpr int LS_TOTAL = LSIDE ? 2 * LS_BYTES : 0;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - EPI_BYTES - LS_TOTAL - 2048) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + LS_TOTAL + EPI_BYTES + 2048;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t LR_SWZ = RP == 16 ? kSw32 : kSw64;
  static constexpr uint32_t LR_SBO = RP == 16 ? 256 : 512;
  static_assert(RP == 16 || RP == 32, "RP");
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory");
};

// First feature of this CTA's 64-feature A box i for feature tile w (pair rank r).
__device__ __forceinline__ int feat_box(int w, int r, int i) { return w * 256 + r * 128 + i * 64; }

template <class C>
__global__ void __launch_bounds__(320, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmAct,
                    const __grid_constant__ CUtensorMap tmLW, const __grid_constant__ CUtensorMap tmLR,
                    const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
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
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      if constexpr (C::LSIDE) {
        // LoRA operands of this tile into side buffer it & 1
        const int lb = it & 1;
        const bool lok = mbar_wait(smem_u32(&lempty[lb]), ((it >> 1) & 1) ^ 1, p.err);
        if (!__all_sync(0xffffffffu, lok)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t lfb = mapa_smem(smem_u32(&lfull[lb]), 0);
          const uint32_t la = s_base + side_off + lb * C::LS_BYTES;
          const uint32_t lr = la + C::LA_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&lfull[lb]), 2 * (C::LA_BYTES + nbh * C::LR_BOX_BYTES));
          if constexpr (C::A_MN) {
            tma_load_3d_pair(&tmLW, lfb, la, feat_box(w, rank, 0), 0, ch.e);
            tma_load_3d_pair(&tmLW, lfb, la + C::LA_BOX_BYTES, feat_box(w, rank, 1), 0, ch.e);
          } else {
            tma_load_3d_pair(&tmLW, lfb, la, 0, feat_box(w, rank, 0), ch.e);
          }
          for (int j = 0; j < nbh; ++j)
            tma_load_2d_pair(&tmLR, lfb, lr + j * C::LR_BOX_BYTES, 0, r0 + j * C::BOXR);
        }
        __syncwarp();
      }
      for (int ks = 0; ks < p.nk + (C::LSIDE ? 0 : 1); ++ks) {
        const bool wok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err);
        if (!__all_sync(0xffffffffu, wok)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t fb = full_leader + stage * 8;
          const uint32_t sa = s_base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          if (ks < p.nk) {
            // every copy is full-size (rows past the chunk are loaded and ignored,
            // rows past P and K past the end read as zero)
            const int k0 = ks * C::BK;
            if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * (C::A_BYTES + C::B_BYTES));
            if constexpr (C::V) {
              if constexpr (C::A_MN)
                tma_load_4d_pair(&tmW, fb, sa, 0, k0, feat_box(w, rank, 0) / 64, ch.e);
              else
                tma_load_4d_pair(&tmW, fb, sa, 0, feat_box(w, rank, 0), k0 / C::KA, ch.e);
              tma_load_3d_pair(&tmAct, fb, sb, 0, r0, k0 / C::KA);
            } else {
              if constexpr (C::A_MN) {
                tma_load_3d_pair(&tmW, fb, sa, feat_box(w, rank, 0), k0, ch.e);
                tma_load_3d_pair(&tmW, fb, sa + C::A_BYTES / 2, feat_box(w, rank, 1), k0, ch.e);
              } else {
                tma_load_3d_pair(&tmW, fb, sa, k0, feat_box(w, rank, 0), ch.e);
                tma_load_3d_pair(&tmW, fb, sa + C::ATOM_A, k0 + C::KA, feat_box(w, rank, 0), ch.e);
              }
              tma_load_2d_pair(&tmAct, fb, sb, k0, r0);
              tma_load_2d_pair(&tmAct, fb, sb + C::ATOM_B, k0 + C::KA, r0);
            }
          } else {
            const uint32_t bytes = C::LA_BYTES + nbh * C::LR_BOX_BYTES;
            if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * bytes);
            if constexpr (C::A_MN) {
              tma_load_3d_pair(&tmLW, fb, sa, feat_box(w, rank, 0), 0, ch.e);
              tma_load_3d_pair(&tmLW, fb, sa + C::LA_BOX_BYTES, feat_box(w, rank, 1), 0, ch.e);
            } else {
              tma_load_3d_pair(&tmLW, fb, sa, 0, feat_box(w, rank, 0), ch.e);
            }
            for (int j = 0; j < nbh; ++j)
              tma_load_2d_pair(&tmLR, fb, sb + j * C::LR_BOX_BYTES, 0, r0 + j * C::BOXR);
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
                                        : smem_desc(s_base, 16, C::LR_SBO, C::LR_SWZ);
      const uint64_t lr_desc0 = smem_desc(s_base + C::A_BYTES, 16, C::LR_SBO, C::LR_SWZ);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued_any = false;
      for (int t = pair; t < total && ok; t += npairs, ++it) {
        const int c = t / p.n_ftiles;
        const TileInfo ch = p.chunks[c];
        const int ncols = ((ch.row_end - ch.row0) + 15) & ~15;
        const uint32_t idesc = idesc_bf16(256, ncols, C::A_MN ? 1 : 0, 0);
        const int b = it & 1;
        const bool aok = mbar_wait(smem_u32(&acc_empty[b]), ((it >> 1) & 1) ^ 1, p.err);
        if (!__all_sync(0xffffffffu, aok)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + b * C::NMAX;
        if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
        if constexpr (C::LSIDE) {
          // the LoRA block first (it starts the accumulation), from side buffer it & 1
          const int lb = it & 1;
          const bool lok = mbar_wait(smem_u32(&lfull[lb]), (it >> 1) & 1, p.err);
          if (!__all_sync(0xffffffffu, lok)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t la = s_base + side_off + lb * C::LS_BYTES;
            const uint32_t lr = la + C::LA_BYTES;
#pragma unroll
            for (int kk = 0; kk < C::RP / 16; ++kk) {
              const uint64_t ad = C::A_MN ? smem_desc(la + kk * 2048, C::LA_BOX_BYTES, 1024, kSw128)
                                          : smem_desc(la + kk * 32, 16, C::LR_SBO, C::LR_SWZ);
              umma_bf16_pair(d, ad, smem_desc(lr + kk * 32, 16, C::LR_SBO, C::LR_SWZ), idesc,
                             kk ? 1u : 0u);
            }
            umma_commit_pair(smem_u32(&lempty[lb]), 0x3);
          }
          __syncwarp();
        }
        for (int ks = 0; ks < p.nk + (C::LSIDE ? 0 : 1); ++ks) {
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
                const uint32_t kb = (uint32_t)((kk >> 2) * C::ATOM_B + (kk & 3) * 32) >> 4;
                umma_bf16_pair(d, a_desc0 + so + (C::A_MN ? kk * (2048 / 16) : ka), b_desc0 + so + kb,
                               idesc, (C::LSIDE || (ks | kk)) ? 1u : 0u);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < C::RP / 16; ++kk)
                umma_bf16_pair(d, la_desc0 + so + kk * (C::A_MN ? 2048 / 16 : 32 / 16),
                               lr_desc0 + so + kk * (32 / 16), idesc, 1u);
            }
            umma_commit_pair(smem_u32(&empty[stage]), 0x3);
          }
          __syncwarp();
          issued_any = true;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
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
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9, both CTAs)
    const int q = warp & 3;                         // TMEM lane quarter of this warp
    const int hsel = (warp - 2) >> 2;               // which alternate 32-token chunks
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const uint32_t acc_empty_leader = mapa_smem(smem_u32(acc_empty), 0);
    uint8_t* blk = epi + (warp - 2) * C::BLK_BYTES; // 32 tokens x 32 features bf16, 64-byte rows
    const int rrow = lane >> 2, rpart = lane & 3;   // transposed read: 8 rows x 4 parts per pass
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const int c = t / p.n_ftiles, w = t % p.n_ftiles;
      const TileInfo ch = p.chunks[c];
      const int nrows = ch.row_end - ch.row0;
      const int b = it & 1;
      const int fq = w * 256 + (int)rank * 128 + q * 32;   // first feature of this warp
      const bool ok = mbar_wait(smem_u32(&acc_full[b]), (it >> 1) & 1, p.err);
      if (named_bar_or(1, 32 * C::EPI_WARPS, !ok || *abort_flag != 0)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + b * C::NMAX;
      uint32_t v[32], vn[32];
      int c0 = hsel * 32;
      if (c0 < nrows) { tmem_ld32(acc + c0, v); tmem_wait_ld(); }
      for (; c0 < nrows; c0 += 64) {
        const bool more = c0 + 64 < nrows;
        if (more) tmem_ld32(acc + c0 + 64, vn);          // next chunk, in flight meanwhile
        if (lane == 0) bulk_wait_read<0>();               // the last store from blk has read it
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          *reinterpret_cast<__nv_bfloat16*>(blk + i * 64 + lane * 2) = __float2bfloat16_rn(__uint_as_float(v[i]));
        const int grow = ch.row0 + c0;
        if (c0 + 32 <= nrows) {
          // 32 rows inside the chunk: one TMA tensor store of the block (features past F
          // are clipped by the tensor map)
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmOut, smem_u32(blk), fq, grow);
            bulk_commit_group();
          }
        } else {
          // the chunk's ragged last block: its rows past the end belong to the next
          // chunk, so 16-byte stores of the rows inside only
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int rr = rrow + 8 * j;
            const int f = fq + rpart * 8;
            if (c0 + rr < nrows && f < p.F) {
              const uint4 x = *reinterpret_cast<const uint4*>(blk + rr * 64 + rpart * 16);
              *reinterpret_cast<uint4*>(p.out + (size_t)(grow + rr) * p.F + f) = x;
            }
          }
        }
        __syncwarp();
        if (more) {
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = vn[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + b * 8);
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
