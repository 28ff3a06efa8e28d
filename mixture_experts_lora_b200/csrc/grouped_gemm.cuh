// Persistent grouped GEMM with fused Split-LoRA for sm_100a (tcgen05 + TMEM + TMA).
//
// Orientation: output features on the MMA's M side (128 per tile, dense), the
// expert's tokens on the N side (up to 256 per tile, granularity 16).  Each
// expert's rows are cut into token chunks of at most 256 rows, so the ragged end
// of an expert costs at most 15 wasted columns instead of a partly empty
// 128-row tile.  For a tile (token chunk of expert e, feature tile w):
//
//   D[f, t] = sum_k Wt[e][f, k] Act[t, k]  +  sum_r Lt[e][f, r] LRc[t, r]
//
// where Act is the expert-sorted activation matrix, Wt the weight oriented
// feature-major and LRc = bf16(c * Act L_A[e]) the rank-r product computed by
// the low-rank kernel.  The second sum is one extra K-block of the same
// pipeline: Y = XW + (alpha/r)(XA)B of the Split-LoRA reordering
// ("Accelerating Mixture-of-Experts Fine-Tuning", Mathematical Formulation
// section 2) without any K x N adapter delta.
//
// Roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and
// issues tcgen05.mma, warps 2-5 run the epilogue (TMEM -> registers -> global).
// The accumulator is double buffered in TMEM (2 x 256 fp32 columns) so the
// epilogue of one tile overlaps the K-loop of the next.
//
// Shared-memory operands (canonical UMMA layouts):
//   A (weights)  forward, W stored [K][F]: MN-major, two 64-feature boxes of 64 K
//                rows, 128-byte swizzle; backward, W stored [F][K]: K-major,
//                [128 features][64 K], 128-byte swizzle
//   B (tokens)   [N rows][64 K], K-major, 128-byte swizzle, boxes of 32 rows
//   LoRA block   A: L_B^T (forward [r][F]: MN-major; backward [F][r]: K-major,
//                32/64-byte swizzle); B: LRc [N rows][r], K-major, 32/64-byte swizzle
#pragma once

#include "common.cuh"

namespace moe {

enum EpiKind : int {
  EPI_GATEUP_FWD = 0,  // features = 64 gate + 64 up; write GU and H = silu(g) * u
  EPI_STORE = 1,       // write D^T as bf16
  EPI_SWIGLU_BWD = 2   // D = dH; read GU; write dGU = [dg | du]
};

struct GemmParams {
  const TileInfo* chunks;  // token chunks {e, row0, row_end}, at most 256 rows each
  const int* n_chunks;
  int F;                   // output features (EPI_GATEUP_FWD: n, the gate width)
  int K;
  int n_ftiles;            // feature tiles per chunk
  int nk;                  // K steps of 64 (the LoRA block is step nk)
  int n_half;              // offset of the up half in W / GU / dGU (= n)
  __nv_bfloat16* out0;     // GATEUP: GU [P,2n]; STORE: out [P,F]; SWIGLU_BWD: dGU [P,2n]
  int ld0;
  __nv_bfloat16* out1;     // GATEUP: H [P,n]
  int ld1;
  const __nv_bfloat16* in0;  // SWIGLU_BWD: GU [P,2n]
  int ldi0;
  int* err;
};

template <int EPI_, bool A_MN_, int RP_>
struct GemmCfg {
  static constexpr int EPI = EPI_, RP = RP_;
  static constexpr bool A_MN = A_MN_;
  static constexpr int BM = 128, BK = 64, NMAX = 256, BOXR = 32;
  static constexpr int A_BYTES = BM * BK * 2;        // 16 KB
  static constexpr int B_BYTES = NMAX * BK * 2;      // 32 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int XCH_BYTES = (EPI == EPI_GATEUP_FWD) ? 64 * 33 * 4 : 0;
  static constexpr int STAGES = 4;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + XCH_BYTES + 1024 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int LA_BOX_BYTES = A_MN ? RP * 64 * 2 : 0;   // forward: 64 features x RP rows
  static constexpr int LR_BOX_BYTES = BOXR * RP * 2;            // 32 token rows x RP
  static constexpr uint32_t LR_SWZ = RP == 16 ? kSw32 : kSw64;
  static constexpr uint32_t LR_SBO = RP == 16 ? 256 : 512;
  static_assert(RP == 16 || RP == 32, "RP");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Feature coordinate (column of W stored [K][F], row of W stored [F][K]) of the
// 64-feature box i of feature tile w.
template <class C>
__device__ __forceinline__ int feat_box(int w, int i, int n_half) {
  if constexpr (C::EPI == EPI_GATEUP_FWD) return (i == 0 ? 0 : n_half) + w * 64;
  else return w * 128 + i * 64;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Barrier over `n` threads that also ORs a predicate across them, so that every
// participating warp takes the same branch afterwards.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

template <class C>
__global__ void __launch_bounds__(192, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmAct,
                    const __grid_constant__ CUtensorMap tmLW, const __grid_constant__ CUtensorMap tmLR,
                    const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  float* xch = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::XCH_BYTES);
  uint64_t* full = bars;                   // [STAGES]
  uint64_t* empty = bars + C::STAGES;      // [STAGES]
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
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmLW);
    tma_prefetch_desc(&tmLR);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = (*p.n_chunks) * p.n_ftiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int c = t / p.n_ftiles, w = t % p.n_ftiles;
        const TileInfo ch = p.chunks[c];
        const int nb = (ch.row_end - ch.row0 + C::BOXR - 1) / C::BOXR;
        for (int ks = 0; ks <= p.nk; ++ks) {
          if (*abort_flag) { ok = false; break; }
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t sa = s_base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          if (ks < p.nk) {
            mbar_arrive_expect_tx(fb, C::A_BYTES + nb * (C::BOXR * C::BK * 2));
            if constexpr (C::A_MN) {
              tma_load_3d(&tmW, fb, sa, feat_box<C>(w, 0, p.n_half), ks * C::BK, ch.e);
              tma_load_3d(&tmW, fb, sa + C::A_BYTES / 2, feat_box<C>(w, 1, p.n_half), ks * C::BK, ch.e);
            } else {
              tma_load_3d(&tmW, fb, sa, ks * C::BK, w * C::BM, ch.e);
            }
            for (int j = 0; j < nb; ++j)
              tma_load_2d(&tmAct, fb, sb + j * (C::BOXR * C::BK * 2), ks * C::BK, ch.row0 + j * C::BOXR);
          } else {
            // LoRA block: A = L_B^T (RP K-rows), B = LRc (RP columns)
            constexpr int la_bytes = C::A_MN ? 2 * C::LA_BOX_BYTES : C::BM * C::RP * 2;
            mbar_arrive_expect_tx(fb, la_bytes + nb * C::LR_BOX_BYTES);
            if constexpr (C::A_MN) {
              tma_load_3d(&tmLW, fb, sa, feat_box<C>(w, 0, p.n_half), 0, ch.e);
              tma_load_3d(&tmLW, fb, sa + C::LA_BOX_BYTES, feat_box<C>(w, 1, p.n_half), 0, ch.e);
            } else {
              tma_load_3d(&tmLW, fb, sa, 0, w * C::BM, ch.e);
            }
            for (int j = 0; j < nb; ++j)
              tma_load_2d(&tmLR, fb, sb + j * C::LR_BOX_BYTES, 0, ch.row0 + j * C::BOXR);
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        for (int s = 0; s < C::STAGES; ++s)
          mbar_wait(smem_u32(&full[s]), phase ^ (s < stage ? 0u : 1u), nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued_any = false;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const int c = t / p.n_ftiles;
        const TileInfo ch = p.chunks[c];
        const int ncols = ((ch.row_end - ch.row0) + 15) & ~15;
        const uint32_t idesc = idesc_bf16(128, ncols, C::A_MN ? 1 : 0, 0);
        const int b = it & 1;
        if (!mbar_wait(smem_u32(&acc_empty[b]), ((it >> 1) & 1) ^ 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + b * C::NMAX;
        for (int ks = 0; ks <= p.nk; ++ks) {
          if (*abort_flag) { ok = false; break; }
          if (!mbar_wait(smem_u32(&full[stage]), phase, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = s_base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          if (ks < p.nk) {
#pragma unroll
            for (int kk = 0; kk < C::BK / 16; ++kk) {
              const uint64_t ad = C::A_MN ? smem_desc(sa + kk * 2048, C::A_BYTES / 2, 1024, kSw128)
                                          : smem_desc(sa + kk * 32, 16, 1024, kSw128);
              const uint64_t bd = smem_desc(sb + kk * 32, 16, 1024, kSw128);
              umma_bf16(d, ad, bd, idesc, (ks | kk) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < C::RP / 16; ++kk) {
              const uint64_t ad = C::A_MN ? smem_desc(sa + kk * 2048, C::LA_BOX_BYTES, 1024, kSw128)
                                          : smem_desc(sa + kk * 32, 16, C::LR_SBO, C::LR_SWZ);
              const uint64_t bd = smem_desc(sb + kk * 32, 16, C::LR_SBO, C::LR_SWZ);
              umma_bf16(d, ad, bd, idesc, 1u);
            }
          }
          umma_commit(smem_u32(&empty[stage]));
          issued_any = true;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(smem_u32(&acc_full[b]));
      }
      if (!ok) *abort_flag = 1;
      if (issued_any) {
        umma_commit(smem_u32(drain));
        mbar_wait(smem_u32(drain), 0, p.err);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                       // TMEM lane quarter of this warp
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const int c = t / p.n_ftiles, w = t % p.n_ftiles;
      const TileInfo ch = p.chunks[c];
      const int nrows = ch.row_end - ch.row0;
      const int b = it & 1;
      const bool ok = mbar_wait(smem_u32(&acc_full[b]), (it >> 1) & 1, p.err);
      // one decision for all four epilogue warps (they meet at named barriers below)
      if (named_bar_or(1, 128, !ok || *abort_flag != 0)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + b * C::NMAX;

      if constexpr (C::EPI == EPI_STORE) {
        const int f = w * 128 + q * 32 + lane;
        const bool fok = f < p.F;
        __nv_bfloat16* dst = p.out0 + (size_t)ch.row0 * p.ld0 + f;
        for (int c0 = 0; c0 < nrows; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(acc + c0, v);
          tmem_wait_ld();
          if (fok) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c0 + i < nrows) dst[(size_t)(c0 + i) * p.ld0] = __float2bfloat16_rn(__uint_as_float(v[i]));
          }
        }
      } else if constexpr (C::EPI == EPI_GATEUP_FWD) {
        // lanes 0-63: gate features w*64 + (0..63); lanes 64-127: the matching up features
        const bool is_gate = q < 2;
        const int j = w * 64 + (q & 1) * 32 + lane;     // gate-feature index of this lane's pair
        const bool fok = j < p.n_half;
        __nv_bfloat16* gu = p.out0 + (size_t)ch.row0 * p.ld0 + (is_gate ? j : p.n_half + j);
        __nv_bfloat16* h = p.out1 + (size_t)ch.row0 * p.ld1 + j;
        float* xrow = xch + ((q & 1) * 32 + lane) * 33;
        for (int c0 = 0; c0 < nrows; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(acc + c0, v);
          tmem_wait_ld();
          if (!is_gate) {
#pragma unroll
            for (int i = 0; i < 32; ++i) xrow[i] = __uint_as_float(v[i]);
          }
          named_bar(1, 128);
          if (fok) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (c0 + i < nrows) {
                const float x = __uint_as_float(v[i]);
                gu[(size_t)(c0 + i) * p.ld0] = __float2bfloat16_rn(x);
                if (is_gate) h[(size_t)(c0 + i) * p.ld1] = __float2bfloat16_rn(silu_f(x) * xrow[i]);
              }
            }
          }
          named_bar(1, 128);
        }
      } else {  // EPI_SWIGLU_BWD
        const int f = w * 128 + q * 32 + lane;
        const bool fok = f < p.F;
        const __nv_bfloat16* gsrc = p.in0 + (size_t)ch.row0 * p.ldi0 + f;
        __nv_bfloat16* dst = p.out0 + (size_t)ch.row0 * p.ld0 + f;
        for (int c0 = 0; c0 < nrows; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(acc + c0, v);
          tmem_wait_ld();
          if (fok) {
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
              if (c0 + i < nrows) {
                const size_t ro = (size_t)(c0 + i);
                const float dh = __uint_as_float(v[i]);
                const float g = __bfloat162float(gsrc[ro * p.ldi0]);
                const float u = __bfloat162float(gsrc[ro * p.ldi0 + p.n_half]);
                const float s = 1.0f / (1.0f + __expf(-g));
                dst[ro * p.ld0] = __float2bfloat16_rn(dh * u * s * (1.0f + g * (1.0f - s)));
                dst[ro * p.ld0 + p.n_half] = __float2bfloat16_rn(dh * g * s);
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
