// Gradients of the expert weights themselves (full fine-tuning): a grouped GEMM whose
// contraction runs over each expert's rows of the expert-sorted matrices,
//     G[e] = L_e^T R_e,   L [P, Mdim], R [P, Ndim] -> G [E, Mdim, Ndim] (bf16, fp32 sums)
// with L_e, R_e the rows [offsets[e], offsets[e+1]) - a count that differs per
// expert and may be zero.  dW_gu[e] = X_e^T dGU_e and dW_d[e] = H_e^T (w dY)_e: the
// layer sees W only through x W, so training it (the full fine-tuning mode of
// "GPT-5.6-Terraに触れてみたよ", section on full fine-tuning, W' = W0 + delta W)
// needs exactly these products.
//
// One CTA (tcgen05 cta_group::1, persistent) owns 128 x 256 output tiles of one
// expert: Mdim on the MMA's M side (TMEM lane = output row), Ndim on N.  Tiles are
// taken expert-major, so the CTAs that run together read one expert's rows from L2.
// Both operands sit MN-major in shared memory: a stage holds 64 rows of L as two
// 64-column atoms and 64 rows of R as four atoms, 128-byte swizzled, one TMA copy
// each through atom views (or one per atom when a width is not a multiple of 64).
//
// The ragged end: every copy starts at the expert's first row and is full-size, so
// the stage that crosses the end of the segment also holds rows of the next expert.
// The MMA warp issues only the 16-row K steps that reach into the segment and, in
// the last of them, zeroes L's rows past the end in shared memory before the MMA
// (a 128-byte row of a swizzled MN-major atom is one K row whatever the swizzle).
// Rows past P read as zero from TMA.  Experts without rows get a zero tile written
// straight by the epilogue.
//
// Roles (320 threads): warp 0 issues the TMA copies, warp 1 owns TMEM, zeroes tails
// and issues the MMAs, warps 2-9 drain TMEM (two warps per lane quarter, alternate
// 32-column chunks): each 32 x 32 block goes to bf16 in a 64-byte-swizzled staging
// buffer of the warp (two per warp, alternating) and out with one TMA tensor store,
// which writes whole row segments and clips rows and columns past the matrix.  TMEM
// holds two 256-column accumulators, so a tile's epilogue overlaps the next tile's MMAs.
#pragma once

#include "common.cuh"

namespace moe {

struct DwParams {
  const int32_t* offsets;   // [E + 1] expert segments of the sorted rows
  int E, Mdim, Ndim;
  int n_mt, n_nt;           // 128-row and 256-column tiles per expert
  __nv_bfloat16* out;       // [E, Mdim, Ndim]
  int* err;
};

// V: one copy per operand and stage through atom views (Mdim, Ndim multiples of 64);
// otherwise one copy per 64-column atom.
template <bool V_>
struct DwCfg {
  static constexpr bool V = V_;
  static constexpr int BM = 128, BN = 256, BK = 64;     // BK: rows (K) per stage
  static constexpr int ATOM = BK * 64 * 2;              // 8 KB: 64 rows x 64 columns
  static constexpr int L_BYTES = 2 * ATOM;              // 16 KB
  static constexpr int R_BYTES = 4 * ATOM;              // 32 KB
  static constexpr int STAGE_BYTES = L_BYTES + R_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int STG_BYTES = 32 * 32 * 2;         // one 32 x 32 bf16 output block
  static constexpr int STG_TOTAL = EPI_WARPS * 2 * STG_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STG_TOTAL + 256 + 1024;
  static constexpr int TMEM_COLS = 2 * BN;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    moe_dw_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmR,
                  const __grid_constant__ CUtensorMap tmO, const DwParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint8_t* stg_all = smem + C::STAGES * C::STAGE_BYTES;   // epilogue staging blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg_all + C::STG_TOTAL);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = bars + C::STAGES;          // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* drain = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(acc_full + 6);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), C::EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmL);
    tma_prefetch_desc(&tmR);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();          // predecessors' outputs visible from here
  const int per_e = p.n_mt * p.n_nt;
  const int total = p.E * per_e;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int e = t / per_e, rem = t % per_e;
      const int nt = rem / p.n_mt, mt = rem % p.n_mt;
      const int lo = p.offsets[e], rows = p.offsets[e + 1] - lo;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      for (int k0 = 0; k0 < rows; k0 += C::BK) {
        const bool wok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err);
        if (!__all_sync(0xffffffffu, wok)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t sl = s_base + stage * C::STAGE_BYTES;
          const uint32_t sr = sl + C::L_BYTES;
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          if constexpr (C::V) {
            tma_load_3d(&tmL, fb, sl, 0, lo + k0, mt * 2);
            tma_load_3d(&tmR, fb, sr, 0, lo + k0, nt * 4);
          } else {
#pragma unroll
            for (int a = 0; a < 2; ++a) tma_load_2d(&tmL, fb, sl + a * C::ATOM, (mt * 2 + a) * 64, lo + k0);
#pragma unroll
            for (int a = 0; a < 4; ++a) tma_load_2d(&tmR, fb, sr + a * C::ATOM, (nt * 4 + a) * 64, lo + k0);
          }
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // MN-major operands, 128-byte swizzle: LBO = stride between 64-wide atoms, SBO =
    // stride between 8-row groups; a 16-row K step advances 2048 bytes.
    const uint64_t a_desc0 = smem_desc(s_base, C::ATOM, 1024, kSw128);
    const uint64_t b_desc0 = smem_desc(s_base + C::L_BYTES, C::ATOM, 1024, kSw128);
    const uint32_t idesc = idesc_bf16(C::BM, C::BN, 1, 1);
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    bool issued_any = false;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int e = t / per_e;
      const int rows = p.offsets[e + 1] - p.offsets[e];
      if (rows <= 0) continue;
      const int b = it & 1;
      const bool aok = mbar_wait(smem_u32(&acc_empty[b]), ((it >> 1) & 1) ^ 1, p.err);
      if (!__all_sync(0xffffffffu, aok)) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      const uint32_t d = tmem + b * C::BN;
      for (int k0 = 0; k0 < rows; k0 += C::BK) {
        const bool fok = mbar_wait(smem_u32(&full[stage]), phase, p.err);
        if (!__all_sync(0xffffffffu, fok)) { ok = false; break; }
        const int kv = rows - k0 < C::BK ? rows - k0 : C::BK;   // rows of this expert
        const int nsteps = (kv + 15) >> 4;
        const int z = nsteps * 16 - kv;                          // rows of the next expert
        if (z > 0) {
          // zero L rows kv .. 16 * nsteps - 1 of both atoms (z lines of 128 bytes each)
          uint8_t* lz = smem + stage * C::STAGE_BYTES + kv * 128;
          for (int i = lane; i < 2 * z * 8; i += 32) {
            const int a = i / (z * 8), o = i - a * z * 8;
            *reinterpret_cast<uint4*>(lz + a * C::ATOM + o * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t so = (uint32_t)(stage * C::STAGE_BYTES) >> 4;
          for (int kk = 0; kk < nsteps; ++kk)
            umma_bf16(d, a_desc0 + so + kk * (2048 / 16), b_desc0 + so + kk * (2048 / 16), idesc,
                      (k0 | kk) ? 1u : 0u);
          umma_commit(smem_u32(&empty[stage]));
        }
        __syncwarp();
        issued_any = true;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(&acc_full[b]));
      __syncwarp();
      ++it;
    }
    if (!ok && lane == 0) *abort_flag = 1;
    if (issued_any) {
      if (lane == 0) umma_commit(smem_u32(drain));
      __syncwarp();
      mbar_wait(smem_u32(drain), 0, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;                         // TMEM lane quarter of this warp
    const int hsel = (warp - 2) >> 2;               // which alternate 32-column chunks
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint8_t* stg = stg_all + (warp - 2) * 2 * C::STG_BYTES;
    int sel = 0;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const int e = t / per_e, rem = t % per_e;
      const int nt = rem / p.n_mt, mt = rem % p.n_mt;
      const int rows = p.offsets[e + 1] - p.offsets[e];
      const int row = mt * C::BM + q * 32 + lane;
      __nv_bfloat16* orow = p.out + ((size_t)e * p.Mdim + row) * p.Ndim;
      const int col0 = nt * C::BN;
      if (rows <= 0) {
        if (row < p.Mdim) {
          for (int c0 = hsel * 32; c0 < C::BN; c0 += 64)
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int col = col0 + c0 + 8 * g;
              if (col < p.Ndim) *reinterpret_cast<uint4*>(orow + col) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        continue;
      }
      const int b = it & 1;
      const bool ok = mbar_wait(smem_u32(&acc_full[b]), (it >> 1) & 1, p.err);
      if (named_bar_or(1, 32 * C::EPI_WARPS, !ok || *abort_flag != 0)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + b * C::BN;
      uint32_t v[32], vn[32];
      int c0 = hsel * 32;
      tmem_ld32(acc + c0, v);
      tmem_wait_ld();
      for (; c0 < C::BN; c0 += 64) {
        const bool more = c0 + 64 < C::BN;
        if (more) tmem_ld32(acc + c0 + 64, vn);     // next chunk, in flight meanwhile
        if (col0 + c0 < p.Ndim) {
          // staging buffer `sel` was last handed to a store two blocks ago: wait
          // until that store has read it
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          uint8_t* blk = stg + sel * C::STG_BYTES;
          // row `lane` of the block: four 16-byte chunks, 64-byte swizzle (chunk j of
          // row r sits at chunk j ^ ((r >> 1) & 3)), conflict-free for the warp
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * g + 0]), __uint_as_float(v[8 * g + 1]));
            o.y = pack_bf16x2(__uint_as_float(v[8 * g + 2]), __uint_as_float(v[8 * g + 3]));
            o.z = pack_bf16x2(__uint_as_float(v[8 * g + 4]), __uint_as_float(v[8 * g + 5]));
            o.w = pack_bf16x2(__uint_as_float(v[8 * g + 6]), __uint_as_float(v[8 * g + 7]));
            *reinterpret_cast<uint4*>(blk + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) = o;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmO, smem_u32(blk), col0 + c0, mt * C::BM + q * 32, e);
            bulk_commit_group();
          }
          sel ^= 1;
        }
        if (more) {
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = vn[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
      ++it;
    }
    if (lane == 0) bulk_wait<0>();                // every store of this warp complete
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace moe
