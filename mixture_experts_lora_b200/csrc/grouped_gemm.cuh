// Persistent grouped GEMM with fused Split-LoRA for sm_100a (tcgen05 + TMEM + TMA).
//
// One launch covers every expert.  The row operand A is an expert-sorted
// activation matrix [P, K] (rows of expert e are [offsets[e], offsets[e+1]));
// a row tile never straddles two experts, so the weight operand of a tile is
// W[e].  For each (row tile, column tile) the kernel computes
//
//     acc = A_tile W[e][:, cols]  +  bf16(c * (A_tile LA[e])) LB[e][:, cols]
//
// which is Y = XW + (alpha/r)(XA)B of the Split-LoRA reordering ("Accelerating
// Mixture-of-Experts Fine-Tuning", Mathematical Formulation section 2): the
// rank-r product A_tile LA[e] accumulates in its own small TMEM accumulator in
// the same K-loop (it reuses the A tile already in shared memory), is rounded
// to bf16 by the epilogue warps and staged back to shared memory, and one
// extra MMA with K = r adds its product with LB[e] into the main accumulator.
// No K x N adapter delta is formed.
//
// Roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and issues
// tcgen05.mma, warps 2-5 run the epilogue (TMEM -> registers -> global).
// The main accumulator and the low-rank accumulator are double buffered in TMEM
// so the epilogue of one tile overlaps the K-loop of the next; the LoRA-B MMA
// of a tile is issued a few K-steps into the next tile, after the epilogue has
// staged bf16(c * XA).
//
// Operand layouts in shared memory (all canonical UMMA layouts):
//   A      [128 rows][64 K]  K-major, 128-byte swizzle (one TMA box)
//   B      forward  (W stored [K][N]): MN-major, boxes of 32 columns x 64 K rows,
//                    64-byte swizzle; backward (W^T, stored [N][K]): K-major,
//                    [BN rows][64 K], 128-byte swizzle
//   LA     forward  ([K][RP]): MN-major, 32/64-byte swizzle; backward ([RP][K]):
//                    K-major, 128-byte swizzle
//   LB     forward  ([RP][N]): MN-major boxes like B; backward ([N][RP]): K-major,
//                    32/64-byte swizzle
//   XS     staged bf16(c*XA) [128][RP], K-major, no swizzle (written by threads)
#pragma once

#include "common.cuh"

namespace moe {

enum EpiKind : int {
  EPI_GATEUP_FWD = 0,  // write GU (bf16) and H = silu(g) * u
  EPI_STORE = 1,       // write acc as bf16
  EPI_SWIGLU_BWD = 2   // acc = dH; read GU; write dGU = [dg | du]
};

struct GemmParams {
  const TileInfo* tiles;   // row tiles of 128 rows
  const int* n_row_tiles;  // number of valid entries in `tiles` (device)
  int N;                   // output columns (EPI_GATEUP_FWD: n, the gate width)
  int K;
  int n_tiles;             // column tiles
  int nk;                  // K steps of 64
  float scale;             // LoRA scale c
  int n_half;              // offset of the up half in GU / dGU (= n)
  __nv_bfloat16* out0;     // GATEUP: GU [P,2n]; STORE: out [P,N]; SWIGLU_BWD: dGU [P,2n]
  int ld0;
  __nv_bfloat16* out1;     // GATEUP: H [P,n]
  int ld1;
  const __nv_bfloat16* in0;  // SWIGLU_BWD: GU [P,2n]
  int ldi0;
  __nv_bfloat16* save_lr;  // low-rank product [P, ld_lr]; first r_lr columns (column tile 0)
  int ld_lr;
  int r_lr;
  int* err;
};

template <int BN_, bool B_MN_, int RP_, int EPI_>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64, BN = BN_, RP = RP_, EPI = EPI_;
  static constexpr bool B_MN = B_MN_;
  static constexpr int WB = 32;                      // MN-major box width (64 B rows)
  static constexpr int NBOX = BN / WB;               // MN-major boxes per B tile
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int LA_BYTES = RP * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + LA_BYTES;
  static constexpr int LB_BYTES = RP * BN * 2;
  static constexpr int XS_BYTES = BM * RP * 2;
  static constexpr int FIXED_BYTES = 2 * LB_BYTES + 2 * XS_BYTES + 1024 /*barriers*/ + 1024 /*align*/;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int STAGES = (SMEM_LIMIT - FIXED_BYTES) / STAGE_BYTES > 4
                                    ? 4
                                    : (SMEM_LIMIT - FIXED_BYTES) / STAGE_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED_BYTES;
  static constexpr int TMEM_COLS = 512;
  static constexpr int XA_COL0 = 2 * BN;             // low-rank accumulators after the two mains
  static constexpr int LORA_DEFER = 2;               // K-step of the next tile that issues LoRA-B
  static_assert(BN % WB == 0 && BN % 32 == 0 && BN <= 256, "BN");
  static_assert(RP == 16 || RP == 32, "RP");
  static_assert(2 * BN + 2 * RP <= TMEM_COLS, "TMEM budget");
  static_assert(STAGES >= 2, "shared memory");
  static_assert(EPI != EPI_GATEUP_FWD || (BN / 2) % 32 == 0, "gate/up halves");
};

// Column coordinate (in W's N dimension) of MN-major box i of column tile nt.
template <class C>
__device__ __forceinline__ int mn_box_col(int nt, int i, int n_half) {
  if constexpr (C::EPI == EPI_GATEUP_FWD) {
    constexpr int half = C::NBOX / 2;
    const int j0 = nt * (C::BN / 2);
    return i < half ? j0 + i * C::WB : n_half + j0 + (i - half) * C::WB;
  } else {
    return nt * C::BN + i * C::WB;
  }
}

// Columns of the MMA for column tile nt (multiple of 16, at most BN).
template <class C>
__device__ __forceinline__ int tile_cols(const GemmParams& p, int nt) {
  if constexpr (C::EPI == EPI_GATEUP_FWD) {
    return C::BN;
  } else {
    int c = p.N - nt * C::BN;
    c = c < C::BN ? c : C::BN;
    return (c + 15) & ~15;
  }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <class C>
__global__ void __launch_bounds__(192, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmLA,
                    const __grid_constant__ CUtensorMap tmLB, const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_stage0 = s_base;
  const uint32_t s_lb0 = s_base + C::STAGES * C::STAGE_BYTES;
  const uint32_t s_xs0 = s_lb0 + 2 * C::LB_BYTES;
  uint8_t* xs_ptr0 = smem + C::STAGES * C::STAGE_BYTES + 2 * C::LB_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(xs_ptr0 + 2 * C::XS_BYTES);
  // barrier slots
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = bars + C::STAGES;          // [STAGES]
  uint64_t* lb_full = bars + 2 * C::STAGES;    // [2]
  uint64_t* lb_empty = lb_full + 2;            // [2]
  uint64_t* xa_full = lb_full + 4;             // [2]
  uint64_t* xa_staged = lb_full + 6;           // [2]
  uint64_t* acc_full = lb_full + 8;            // [2]
  uint64_t* acc_empty = lb_full + 10;          // [2]
  uint64_t* drain = lb_full + 12;              // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lb_full + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(lb_full + 14);

  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&lb_full[b]), 1);
      mbar_init(smem_u32(&lb_empty[b]), 1);
      mbar_init(smem_u32(&xa_full[b]), 1);
      mbar_init(smem_u32(&xa_staged[b]), 4);
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmLA);
    tma_prefetch_desc(&tmLB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = (*p.n_row_tiles) * p.n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const int mt = t / p.n_tiles, nt = t % p.n_tiles;
        const TileInfo ti = p.tiles[mt];
        const int b = it & 1;
        const uint32_t bpar = (it >> 1) & 1;
        // LoRA-B operand of this tile
        if (!mbar_wait(smem_u32(&lb_empty[b]), bpar ^ 1, p.err)) { ok = false; break; }
        const uint32_t lbb = smem_u32(&lb_full[b]);
        const uint32_t lb_dst = s_lb0 + b * C::LB_BYTES;
        mbar_arrive_expect_tx(lbb, C::LB_BYTES);
        if constexpr (C::B_MN) {
#pragma unroll
          for (int i = 0; i < C::NBOX; ++i)
            tma_load_3d(&tmLB, lbb, lb_dst + i * (C::RP * C::WB * 2), mn_box_col<C>(nt, i, p.n_half),
                        0, ti.e);
        } else {
          tma_load_3d(&tmLB, lbb, lb_dst, 0, nt * C::BN, ti.e);
        }
        for (int ks = 0; ks < p.nk; ++ks) {
          if (*abort_flag) { ok = false; break; }
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t sa = s_stage0 + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          const uint32_t sl = sb + C::B_BYTES;
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          tma_load_2d(&tmA, fb, sa, ks * C::BK, ti.row0);
          if constexpr (C::B_MN) {
#pragma unroll
            for (int i = 0; i < C::NBOX; ++i)
              tma_load_3d(&tmB, fb, sb + i * (C::BK * C::WB * 2), mn_box_col<C>(nt, i, p.n_half),
                          ks * C::BK, ti.e);
            tma_load_3d(&tmLA, fb, sl, 0, ks * C::BK, ti.e);
          } else {
            tma_load_3d(&tmB, fb, sb, ks * C::BK, nt * C::BN, ti.e);
            tma_load_3d(&tmLA, fb, sl, ks * C::BK, 0, ti.e);
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        // let copies already issued land before the block can exit
        for (int s = 0; s < C::STAGES; ++s) mbar_wait(smem_u32(&full[s]), phase ^ (s < stage ? 0u : 1u), nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_lr = idesc_bf16(128, C::RP, 0, C::B_MN ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool pending = false;
      int pend_b = 0, pend_it = 0, pend_cols = 0;
      bool issued_any = false;

      auto lora_b = [&](int pb, int pit, int cols) -> bool {
        const uint32_t par = (pit >> 1) & 1;
        if (!mbar_wait(smem_u32(&xa_staged[pb]), par, p.err)) return false;
        if (!mbar_wait(smem_u32(&lb_full[pb]), par, p.err)) return false;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, cols, 0, C::B_MN ? 1 : 0);
        const uint32_t xs = s_xs0 + pb * C::XS_BYTES;
        const uint32_t lb = s_lb0 + pb * C::LB_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::RP / 16; ++kk) {
          // staged XA: K-major, no swizzle, core matrices 8 rows x 16 B;
          // K-chunks of 8 at 128 B, 8-row groups at RP*16 B
          const uint64_t ad = smem_desc(xs + kk * 256, 128, C::RP * 16, kSwNone);
          uint64_t bd;
          if constexpr (C::B_MN) {
            bd = smem_desc(lb + kk * 16 * 64, C::RP * 64, 512, kSw64);
          } else {
            bd = (C::RP == 16) ? smem_desc(lb, 16, 256, kSw32)
                               : smem_desc(lb + kk * 32, 16, 512, kSw64);
          }
          umma_bf16(tmem + pb * C::BN, ad, bd, idesc, 1u);
        }
        umma_commit(smem_u32(&acc_full[pb]));
        umma_commit(smem_u32(&lb_empty[pb]));
        return true;
      };

      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const int nt = t % p.n_tiles;
        const int b = it & 1;
        const uint32_t bpar = (it >> 1) & 1;
        const int cols = tile_cols<C>(p, nt);
        const uint32_t idesc = idesc_bf16(128, cols, 0, C::B_MN ? 1 : 0);
        if (!mbar_wait(smem_u32(&acc_empty[b]), bpar ^ 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_main = tmem + b * C::BN;
        const uint32_t d_lr = tmem + C::XA_COL0 + b * C::RP;
        const int defer_at = p.nk - 1 < C::LORA_DEFER ? p.nk - 1 : C::LORA_DEFER;
        for (int ks = 0; ks < p.nk; ++ks) {
          if (*abort_flag) { ok = false; break; }
          if (!mbar_wait(smem_u32(&full[stage]), phase, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = s_stage0 + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          const uint32_t sl = sb + C::B_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024, kSw128);
            uint64_t bd, ld;
            if constexpr (C::B_MN) {
              bd = smem_desc(sb + kk * 16 * 64, C::BK * C::WB * 2, 512, kSw64);
              ld = (C::RP == 16) ? smem_desc(sl + kk * 16 * 32, C::LA_BYTES, 256, kSw32)
                                 : smem_desc(sl + kk * 16 * 64, C::LA_BYTES, 512, kSw64);
            } else {
              bd = smem_desc(sb + kk * 32, 16, 1024, kSw128);
              ld = smem_desc(sl + kk * 32, 16, 1024, kSw128);
            }
            const uint32_t acc = (ks | kk) ? 1u : 0u;
            umma_bf16(d_main, ad, bd, idesc, acc);
            umma_bf16(d_lr, ad, ld, idesc_lr, acc);
          }
          umma_commit(smem_u32(&empty[stage]));
          issued_any = true;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
          if (pending && ks == defer_at) {
            if (!lora_b(pend_b, pend_it, pend_cols)) { ok = false; break; }
            pending = false;
          }
        }
        if (!ok) break;
        umma_commit(smem_u32(&xa_full[b]));
        if (pending) {  // only when the K loop was shorter than the deferral point
          if (!lora_b(pend_b, pend_it, pend_cols)) { ok = false; break; }
          pending = false;
        }
        pending = true;
        pend_b = b;
        pend_it = it;
        pend_cols = cols;
      }
      if (ok && pending) ok = lora_b(pend_b, pend_it, pend_cols);
      if (!ok) *abort_flag = 1;
      if (issued_any) {
        // every MMA issued by this thread has finished before the block exits
        umma_commit(smem_u32(drain));
        mbar_wait(smem_u32(drain), 0, p.err);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int mt = t / p.n_tiles, nt = t % p.n_tiles;
      const TileInfo ti = p.tiles[mt];
      const int row = ti.row0 + row_in_tile;
      const bool valid = row < ti.row_end;
      const int b = it & 1;
      const uint32_t bpar = (it >> 1) & 1;

      // ---- 1. low-rank product: save it, stage bf16(c * XA) for the LoRA-B MMA
      bool ok = mbar_wait(smem_u32(&xa_full[b]), bpar, p.err);
      if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; break; }
      tc_fence_after();
      {
        float v[C::RP];
        if constexpr (C::RP == 16) {
          uint32_t r[16];
          tmem_ld16(tmem + lane_base + C::XA_COL0 + b * C::RP, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
        } else {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + C::XA_COL0 + b * C::RP, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        }
        if (nt == 0 && valid && p.save_lr != nullptr) {
          __nv_bfloat16* dst = p.save_lr + (size_t)row * p.ld_lr;
#pragma unroll
          for (int g = 0; g < C::RP / 8; ++g) {
            if (g * 8 < p.r_lr) {
              uint4 w;
              w.x = pack_bf16x2(v[g * 8 + 0], v[g * 8 + 1]);
              w.y = pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]);
              w.z = pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]);
              w.w = pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]);
              *reinterpret_cast<uint4*>(dst + g * 8) = w;
            }
          }
        }
        uint8_t* xs = xs_ptr0 + b * C::XS_BYTES + (row_in_tile & 7) * 16 +
                      (row_in_tile >> 3) * (C::RP * 16);
#pragma unroll
        for (int g = 0; g < C::RP / 8; ++g) {
          uint4 w;
          w.x = pack_bf16x2(p.scale * v[g * 8 + 0], p.scale * v[g * 8 + 1]);
          w.y = pack_bf16x2(p.scale * v[g * 8 + 2], p.scale * v[g * 8 + 3]);
          w.z = pack_bf16x2(p.scale * v[g * 8 + 4], p.scale * v[g * 8 + 5]);
          w.w = pack_bf16x2(p.scale * v[g * 8 + 6], p.scale * v[g * 8 + 7]);
          *reinterpret_cast<uint4*>(xs + g * 128) = w;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&xa_staged[b]));

      // ---- 2. main accumulator
      ok = mbar_wait(smem_u32(&acc_full[b]), bpar, p.err);
      if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + b * C::BN;

      if constexpr (C::EPI == EPI_STORE) {
        const int n0 = nt * C::BN;
        const int ncols = tile_cols<C>(p, nt);
        for (int c = 0; c < ncols; c += 32) {
          uint32_t r[32];
          tmem_ld32(acc + c, r);
          tmem_wait_ld();
          if (valid) {
            __nv_bfloat16* dst = p.out0 + (size_t)row * p.ld0;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int col = n0 + c + g * 8;
              if (col < p.N) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(r[g * 8 + 0]), __uint_as_float(r[g * 8 + 1]));
                w.y = pack_bf16x2(__uint_as_float(r[g * 8 + 2]), __uint_as_float(r[g * 8 + 3]));
                w.z = pack_bf16x2(__uint_as_float(r[g * 8 + 4]), __uint_as_float(r[g * 8 + 5]));
                w.w = pack_bf16x2(__uint_as_float(r[g * 8 + 6]), __uint_as_float(r[g * 8 + 7]));
                *reinterpret_cast<uint4*>(dst + col) = w;
              }
            }
          }
        }
      } else if constexpr (C::EPI == EPI_GATEUP_FWD) {
        constexpr int NJ = C::BN / 2;
        const int j0 = nt * NJ;
#pragma unroll 1
        for (int c = 0; c < NJ; c += 32) {
          uint32_t gr[32], ur[32];
          tmem_ld32(acc + c, gr);
          tmem_ld32(acc + NJ + c, ur);
          tmem_wait_ld();
          if (valid) {
            __nv_bfloat16* gu = p.out0 + (size_t)row * p.ld0;
            __nv_bfloat16* h = p.out1 + (size_t)row * p.ld1;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int j = j0 + c + g * 8;
              if (j < p.n_half) {
                float gv[8], uv[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  gv[i] = __uint_as_float(gr[g * 8 + i]);
                  uv[i] = __uint_as_float(ur[g * 8 + i]);
                }
                uint4 wg, wu, wh;
                wg.x = pack_bf16x2(gv[0], gv[1]); wg.y = pack_bf16x2(gv[2], gv[3]);
                wg.z = pack_bf16x2(gv[4], gv[5]); wg.w = pack_bf16x2(gv[6], gv[7]);
                wu.x = pack_bf16x2(uv[0], uv[1]); wu.y = pack_bf16x2(uv[2], uv[3]);
                wu.z = pack_bf16x2(uv[4], uv[5]); wu.w = pack_bf16x2(uv[6], uv[7]);
                wh.x = pack_bf16x2(silu_f(gv[0]) * uv[0], silu_f(gv[1]) * uv[1]);
                wh.y = pack_bf16x2(silu_f(gv[2]) * uv[2], silu_f(gv[3]) * uv[3]);
                wh.z = pack_bf16x2(silu_f(gv[4]) * uv[4], silu_f(gv[5]) * uv[5]);
                wh.w = pack_bf16x2(silu_f(gv[6]) * uv[6], silu_f(gv[7]) * uv[7]);
                *reinterpret_cast<uint4*>(gu + j) = wg;
                *reinterpret_cast<uint4*>(gu + p.n_half + j) = wu;
                *reinterpret_cast<uint4*>(h + j) = wh;
              }
            }
          }
        }
      } else {  // EPI_SWIGLU_BWD
        const int n0 = nt * C::BN;
        const int ncols = tile_cols<C>(p, nt);
#pragma unroll 1
        for (int c = 0; c < ncols; c += 32) {
          uint32_t r[32];
          tmem_ld32(acc + c, r);
          tmem_wait_ld();
          if (valid) {
            const __nv_bfloat16* gu = p.in0 + (size_t)row * p.ldi0;
            __nv_bfloat16* dgu = p.out0 + (size_t)row * p.ld0;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int j = n0 + c + g * 8;
              if (j < p.N) {
                const uint4 gw = *reinterpret_cast<const uint4*>(gu + j);
                const uint4 uw = *reinterpret_cast<const uint4*>(gu + p.n_half + j);
                const uint32_t ga[4] = {gw.x, gw.y, gw.z, gw.w};
                const uint32_t ua[4] = {uw.x, uw.y, uw.z, uw.w};
                uint32_t dgo[4], duo[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  float d0 = __uint_as_float(r[g * 8 + 2 * i]);
                  float d1 = __uint_as_float(r[g * 8 + 2 * i + 1]);
                  float g0 = bf16_lo(ga[i]), g1 = bf16_hi(ga[i]);
                  float u0 = bf16_lo(ua[i]), u1 = bf16_hi(ua[i]);
                  float s0 = 1.0f / (1.0f + __expf(-g0));
                  float s1 = 1.0f / (1.0f + __expf(-g1));
                  dgo[i] = pack_bf16x2(d0 * u0 * s0 * (1.0f + g0 * (1.0f - s0)),
                                       d1 * u1 * s1 * (1.0f + g1 * (1.0f - s1)));
                  duo[i] = pack_bf16x2(d0 * g0 * s0, d1 * g1 * s1);
                }
                *reinterpret_cast<uint4*>(dgu + j) = make_uint4(dgo[0], dgo[1], dgo[2], dgo[3]);
                *reinterpret_cast<uint4*>(dgu + p.n_half + j) =
                    make_uint4(duo[0], duo[1], duo[2], duo[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
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
