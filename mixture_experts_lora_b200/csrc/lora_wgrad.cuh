// Adapter weight gradients as a ragged-K grouped GEMM on tcgen05.
//
// For expert e with sorted rows R_e the four adapter gradients all have the form
//     G_e [D, r] = sum_{q in R_e} Big[q, :]^T Small[q, :]
// dA_d = c G (Big = H, Small = T1), dB_d = c G^T (Big = w*dY, Small = HA),
// dA_gu = c G (Big = X, Small = T2), dB_gu = c G^T (Big = dGU, Small = XA):
// the chain rule through Y = XW + (alpha/r)(XA)B with W frozen ("Accelerating
// Mixture-of-Experts Fine-Tuning", Mathematical Formulation section 2; Unsloth
// docs "Implementation details": only the m*r + r*n adapter parameters train).
//
// One launch computes up to two such problems (the two gradients that become
// computable at the same point of the backward).  Units are (problem, row chunk
// of one expert, 128-wide D tile); a persistent CTA walks its units with one
// continuous TMA/MMA pipeline:
//   M = 128 columns of Big (MN-major A operand, 128-byte swizzle),
//   N = RP (Small, MN-major, no swizzle),
//   K = rows of the chunk, 128 per stage,
// with one TMA copy per operand and stage (Big through a view of 64-column atoms
// when D % 64 == 0, Small through a view of 8-column groups that lands in the
// core-matrix layout).  Every copy is full-size from the chunk's first row, so the
// stage that crosses the chunk's end also holds rows of the next chunk: the MMA
// warp issues only the 16-row K steps that reach into the chunk and zeroes Small's
// rows past its end in the last of them, so a ragged tail contributes nothing.
// The loader and MMA threads each spend a fixed number of instructions per stage
// (two copies; precomputed descriptors advanced by offsets).
// The accumulator is double buffered in TMEM.  A unit of an expert whose rows fit
// in one chunk writes the final bf16 gradient (scaled, in its output orientation).
// Otherwise each unit writes an fp32 partial and counts itself in a per-(expert,
// D tile) arrival counter; the unit that arrives last sums the expert's partials
// in chunk order (deterministic, whatever the arrival order) and writes the
// gradient.  Gradients of experts without rows are written as zeros by the same
// launch.
#pragma once

#include "common.cuh"

namespace moe {

struct WgradProblem {
  const __nv_bfloat16* small;  // [P, ld_small]
  int ld_small;
  int r_small;                 // columns of `small` to read (rest zero)
  int D;
  int n_dtiles;
  bool transpose;              // out [E, r, D] instead of [E, D, r]
  __nv_bfloat16* out;
  float* partial;              // [max_chunks, D, RP]
  int* counters;               // [E, n_dtiles] arrival counters, zero on entry and exit
};

struct WgradParams {
  WgradProblem pr[2];
  int n_problems;
  const TileInfo* chunks;      // row chunks {e, row0, row_end}
  const int* n_chunks;
  const int32_t* chunk_start;  // [E+1]
  int E;
  int r;                       // output rank
  float scale;
  int* err;
};

template <int RP, bool V_ = true>
struct WgradCfg {
  static constexpr bool V = V_;             // Big through the atom view (D % 64 == 0)
  // 128 rows per stage: 8 MMAs per wait and commit (the per-stage issue cost of the
  // loader and MMA threads, not the bytes, bounded 64-row stages)
  static constexpr int BM = 128, BK = 128;
  static constexpr int BIG_BYTES = BM * BK * 2;   // two 64-column atoms of BK rows
  static constexpr int SMALL_BYTES = RP * BK * 2;
  static constexpr int SMALL_NG = BK * 16;        // bytes between 8-column groups of Small
  static constexpr int STAGE_BYTES = BIG_BYTES + SMALL_BYTES;
  static constexpr int STAGES_FIT = (232448 - 2048) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 1024;
  static constexpr int TMEM_COLS = 64;            // 2 x RP fp32 columns (RP <= 32)
  static constexpr int EPI_THREADS = 128;         // warps 2..5
};

// Unit t of the launch -> (problem, chunk, D tile).
struct WgradUnit {
  int prob, c, dt;
};
__device__ __forceinline__ WgradUnit wgrad_unit(const WgradParams& p, int nch, int t) {
  WgradUnit u;
  const int t0 = nch * p.pr[0].n_dtiles;
  u.prob = t < t0 ? 0 : 1;
  const int tt = u.prob == 0 ? t : t - t0;
  const int nd = p.pr[u.prob].n_dtiles;
  u.c = tt / nd;
  u.dt = tt - u.c * nd;
  return u;
}

// Scaled bf16 gradient row d of expert e from fp32 values v[0..RP).
template <int RP>
__device__ __forceinline__ void wgrad_store(const WgradProblem& q, int r, float scale, int e, int d,
                                            const float (&v)[RP]) {
  if (q.transpose) {
#pragma unroll
    for (int i = 0; i < RP; ++i)
      if (i < r) q.out[((size_t)e * r + i) * q.D + d] = __float2bfloat16_rn(scale * v[i]);
  } else {
    __nv_bfloat16* dst = q.out + ((size_t)e * q.D + d) * r;
#pragma unroll
    for (int g = 0; g < RP / 8; ++g) {
      if (g * 8 < r) {
        uint4 o;
        o.x = pack_bf16x2(scale * v[8 * g + 0], scale * v[8 * g + 1]);
        o.y = pack_bf16x2(scale * v[8 * g + 2], scale * v[8 * g + 3]);
        o.z = pack_bf16x2(scale * v[8 * g + 4], scale * v[8 * g + 5]);
        o.w = pack_bf16x2(scale * v[8 * g + 6], scale * v[8 * g + 7]);
        *reinterpret_cast<uint4*>(dst + 8 * g) = o;
      }
    }
  }
}

template <int RP, bool V>
__global__ void __launch_bounds__(192, 1)
    lora_wgrad_kernel(const __grid_constant__ CUtensorMap tmBig0,
                      const __grid_constant__ CUtensorMap tmBig1,
                      const __grid_constant__ CUtensorMap tmSmall0,
                      const __grid_constant__ CUtensorMap tmSmall1, const WgradParams p) {
  using C = WgradCfg<RP, V>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                     // [STAGES]: TMA bytes + producer stores
  uint64_t* empty = bars + C::STAGES;        // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES; // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* drain = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(acc_full + 6);
  volatile int* last_flag = abort_flag + 1;

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
    *last_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmBig0);
    tma_prefetch_desc(&tmSmall0);
    if (p.n_problems > 1) {
      tma_prefetch_desc(&tmBig1);
      tma_prefetch_desc(&tmSmall1);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nch = *p.n_chunks;
  const int total = nch * (p.pr[0].n_dtiles + (p.n_problems > 1 ? p.pr[1].n_dtiles : 0));

  if (warp == 0) {
    // ---------------------------------------------------------- producer (whole warp)
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const WgradUnit u = wgrad_unit(p, nch, t);
      const CUtensorMap* tb = u.prob == 0 ? &tmBig0 : &tmBig1;
      const CUtensorMap* ts = u.prob == 0 ? &tmSmall0 : &tmSmall1;
      const TileInfo ch = p.chunks[u.c];
      const int d0 = u.dt * C::BM;
      const int nk = (ch.row_end - ch.row0 + C::BK - 1) / C::BK;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      for (int ks = 0; ks < nk; ++ks) {
        const bool w = mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t sbig = s_base + stage * C::STAGE_BYTES;
          const int r0 = ch.row0 + ks * C::BK;
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          if constexpr (C::V) {
            tma_load_3d(tb, fb, sbig, 0, r0, d0 / 64);
          } else {
            tma_load_2d(tb, fb, sbig, d0, r0);
            tma_load_2d(tb, fb, sbig + C::BIG_BYTES / 2, d0 + 64, r0);
          }
          // Small [BK rows][RP]: groups of 8 columns, each BK rows x 16 bytes
          // (MN-major, no swizzle: core matrices of 8 rows x 8 columns)
          tma_load_3d(ts, fb, sbig + C::BIG_BYTES, 0, r0, 0);
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer (whole warp)
    // Big^T: MN-major, 128-byte swizzle, 64-column atoms BIG_BYTES/2 apart, 8-row
    // groups 1 KB apart (a 16-row K step advances 2 KB).  Small: MN-major, no swizzle,
    // 8-row groups 128 bytes apart, 8-column groups SMALL_NG apart (a K step: 256 B).
    const uint32_t idesc = idesc_bf16(128, RP, 1, 1);
    const uint64_t a_desc0 = smem_desc(s_base, C::BIG_BYTES / 2, 1024, kSw128);
    const uint64_t b_desc0 = smem_desc(s_base + C::BIG_BYTES, 128, C::SMALL_NG, kSwNone);
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true, issued_any = false;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
      const WgradUnit u = wgrad_unit(p, nch, t);
      const TileInfo ch = p.chunks[u.c];
      const int rows = ch.row_end - ch.row0;
      const int nk = (rows + C::BK - 1) / C::BK;
      const int b = it & 1;
      const bool aok = mbar_wait(smem_u32(&acc_empty[b]), ((it >> 1) & 1) ^ 1, p.err);
      if (!__all_sync(0xffffffffu, aok) || *abort_flag) { ok = false; break; }
      tc_fence_after();
      const uint32_t d = tmem + b * 32;
      for (int ks = 0; ks < nk; ++ks) {
        const bool fok = mbar_wait(smem_u32(&full[stage]), phase, p.err);
        if (!__all_sync(0xffffffffu, fok)) { ok = false; break; }
        const int kv = rows - ks * C::BK < C::BK ? rows - ks * C::BK : C::BK;   // rows of the chunk
        const int nsteps = (kv + 15) >> 4;
        const int z = nsteps * 16 - kv;                                          // rows past its end
        if (z > 0) {
          // zero Small rows kv .. 16 nsteps - 1 in every 8-column group
          uint8_t* zs = smem + stage * C::STAGE_BYTES + C::BIG_BYTES + kv * 16;
          for (int i = lane; i < z * (RP / 8); i += 32) {
            const int g = i / z, rr = i - g * z;
            *reinterpret_cast<uint4*>(zs + g * C::SMALL_NG + rr * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t so = (uint32_t)(stage * C::STAGE_BYTES) >> 4;
          for (int kk = 0; kk < nsteps; ++kk)
            umma_bf16(d, a_desc0 + so + kk * (2048 / 16), b_desc0 + so + kk * (256 / 16), idesc,
                      (ks | kk) ? 1u : 0u);
          umma_commit(smem_u32(&empty[stage]));
        }
        __syncwarp();
        issued_any = true;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(&acc_full[b]));
      __syncwarp();
    }
    if (!ok && lane == 0) *abort_flag = 1;
    if (issued_any) {
      if (lane == 0) umma_commit(smem_u32(drain));
      __syncwarp();
      mbar_wait(smem_u32(drain), 0, p.err);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue (warps 2..5)
    const int q4 = warp & 3;                       // TMEM lane quarter of this warp
    const int et = (warp - 2) * 32 + lane;         // 0..127
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const WgradUnit u = wgrad_unit(p, nch, t);
      const WgradProblem& q = p.pr[u.prob];
      const TileInfo ch = p.chunks[u.c];
      const int b = it & 1;
      const bool ok = mbar_wait(smem_u32(&acc_full[b]), (it >> 1) & 1, p.err);
      // every epilogue warp takes the same branch (named barriers follow)
      if (named_bar_or(1, C::EPI_THREADS, !ok || *abort_flag != 0)) { *abort_flag = 1; break; }
      tc_fence_after();
      float v[RP];
      if constexpr (RP == 16) {
        uint32_t rr[16];
        tmem_ld16(tmem + ((uint32_t)(q4 * 32) << 16) + b * 32, rr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(rr[i]);
      } else {
        uint32_t rr[32];
        tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + b * 32, rr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rr[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
      const int d = u.dt * C::BM + q4 * 32 + lane;
      const int c0 = p.chunk_start[ch.e], c1 = p.chunk_start[ch.e + 1];
      if (c1 - c0 == 1) {
        if (d < q.D) wgrad_store<RP>(q, p.r, p.scale, ch.e, d, v);
        continue;
      }
      // several chunks: fp32 partial, then the last arriving unit sums them in order
      if (d < q.D) {
        float4* dst = reinterpret_cast<float4*>(q.partial + ((size_t)u.c * q.D + d) * RP);
#pragma unroll
        for (int i = 0; i < RP / 4; ++i)
          dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
      __threadfence();
      named_bar(1, C::EPI_THREADS);
      if (et == 0) {
        int* cnt = q.counters + (size_t)ch.e * q.n_dtiles + u.dt;
        const int last = atomicAdd(cnt, 1) == c1 - c0 - 1;
        if (last) {
          *cnt = 0;                                // ready for the next launch
          __threadfence();
        }
        *last_flag = last;
      }
      named_bar(1, C::EPI_THREADS);
      if (*last_flag && d < q.D) {
        float acc[RP];
#pragma unroll
        for (int i = 0; i < RP; ++i) acc[i] = 0.f;
        for (int cc = c0; cc < c1; ++cc) {
          const float4* src = reinterpret_cast<const float4*>(q.partial + ((size_t)cc * q.D + d) * RP);
#pragma unroll
          for (int i = 0; i < RP / 4; ++i) {
            const float4 x = __ldcg(src + i);
            acc[4 * i] += x.x;
            acc[4 * i + 1] += x.y;
            acc[4 * i + 2] += x.z;
            acc[4 * i + 3] += x.w;
          }
        }
        wgrad_store<RP>(q, p.r, p.scale, ch.e, d, acc);
      }
    }
    // gradients of experts without rows are zero: after the units, so the scan never
    // holds up the accumulators; CTA b takes experts b, b + grid, ...
    for (int e = blockIdx.x; e < p.E; e += gridDim.x) {
      if (p.chunk_start[e + 1] != p.chunk_start[e]) continue;
      for (int prob = 0; prob < p.n_problems; ++prob) {
        const WgradProblem& q = p.pr[prob];
        float z[RP];
#pragma unroll
        for (int j = 0; j < RP; ++j) z[j] = 0.f;
        for (int d = et; d < q.D; d += C::EPI_THREADS) wgrad_store<RP>(q, p.r, p.scale, e, d, z);
      }
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
