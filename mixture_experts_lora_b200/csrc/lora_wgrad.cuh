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
// of one expert, 256-wide column tile of Big); a persistent CTA walks its units
// with one continuous TMA/MMA pipeline computing G^T for the tile:
//   M = 128 rank rows (Small^T, MN-major, no swizzle: 16 groups of 8 rank columns;
//       each stage copies the RP / 8 groups of Small's width (those past it read as
//       zero), the rest of the 16 stay zero from the kernel's start),
//   N = 256 columns of Big (MN-major, 128-byte swizzle, four 64-column atoms),
//   K = rows of the chunk, 64 per stage,
// one TMA copy per operand and stage.  A rank of 16 uses an eighth of M,
// but each MMA then moves 256 columns of Big: a thin N = r MMA costs the tensor
// pipe about as long as a full one and would bound the kernel instead of HBM.
// Every copy is full-size from the chunk's first row, so the stage that crosses the
// chunk's end also holds rows of the next chunk: the MMA warp issues only the
// 16-row K steps that reach into the chunk and zeroes Small's rows past its end in
// the last of them.
// The accumulator (128 lanes x 256 fp32 columns) is double buffered in TMEM.  The
// warps that own the TMEM lanes of the rank rows copy them to shared memory (in two
// column halves at ranks above 32); all four epilogue warps then write the gradient
// with 16-byte stores in its output orientation.  A unit of an expert whose rows fit in one chunk writes the final
// bf16 gradient (scaled).  Otherwise each unit writes an fp32 partial and counts
// itself in a per-(expert, column tile) arrival counter; the unit that arrives
// last sums the expert's partials in chunk order (deterministic, whatever the
// arrival order) and writes the gradient.  Gradients of experts without rows are
// written as zeros by the same launch.
#pragma once

#include "common.cuh"

namespace moe {

struct WgradProblem {
  const __nv_bfloat16* small;  // [P, ld_small]
  int ld_small;
  int r_small;                 // columns of `small` to read (rest zero)
  int D;
  int n_dtiles;                // 256-column tiles of Big
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
  static constexpr int THREADS = 192;
  static constexpr int BM = 128;            // rank rows on M (RP of them are used)
  static constexpr int BN = 256;            // Big columns per unit
  static constexpr int BK = 64;             // rows per stage
  static constexpr int SMALL_NG = BK * 16;  // bytes between 8-column groups of Small
  static constexpr int A_BYTES = (BM / 8) * SMALL_NG;     // 16 KB: 16 groups of 8 rank columns
  static constexpr int ATOM = BK * 128;                   // 8 KB: 64 Big columns x BK rows
  static constexpr int B_BYTES = (BN / 64) * ATOM;        // 32 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMALL_COPY = (RP / 8) * SMALL_NG;  // bytes of Small copied per stage
  static constexpr int STAGES = RP > 64 ? 3 : 4;
  // fp32 staging of the accumulator's rank rows, in column halves of SC columns when
  // the rank is wide (the staging of all 256 columns would not fit beside the ring)
  static constexpr int SC = RP > 32 ? BN / 2 : BN;
  static constexpr int ST_LD = SC + 4;                    // fp32 staging row (rank j), padded
  static constexpr int STG_BYTES = RP * ST_LD * 4;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STG_BYTES + 512 + 1024;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int EPI_THREADS = 128;                 // warps 2..5
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Unit t of the launch -> (problem, chunk, column tile).
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

// 8 consecutive output values as one 16-byte bf16 store (scaled).
__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* dst, float s, const float (&v)[8]) {
  uint4 o;
  o.x = pack_bf16x2(s * v[0], s * v[1]);
  o.y = pack_bf16x2(s * v[2], s * v[3]);
  o.z = pack_bf16x2(s * v[4], s * v[5]);
  o.w = pack_bf16x2(s * v[6], s * v[7]);
  *reinterpret_cast<uint4*>(dst) = o;
}

template <int RP, bool V>
__global__ void __launch_bounds__(WgradCfg<RP, V>::THREADS, 1)
    lora_wgrad_kernel(const __grid_constant__ CUtensorMap tmBig0,
                      const __grid_constant__ CUtensorMap tmBig1,
                      const __grid_constant__ CUtensorMap tmSmall0,
                      const __grid_constant__ CUtensorMap tmSmall1, const WgradParams p) {
  using C = WgradCfg<RP, V>;
  constexpr int OWNERS = RP <= 32 ? 1 : RP / 32;   // epilogue warps holding rank rows
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  float* stg = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);   // [RP][ST_LD]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::STG_BYTES);
  uint64_t* full = bars;                     // [STAGES]
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
      mbar_init(smem_u32(&acc_empty[b]), OWNERS);
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
  // the rank groups past RP of every stage's Small^T tile are zero for the whole launch
  for (int s = 0; s < C::STAGES; ++s)
    for (int i = threadIdx.x; i < (C::A_BYTES - C::SMALL_COPY) / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(smem + s * C::STAGE_BYTES + C::SMALL_COPY)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();          // predecessors' outputs visible from here
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
      const int d0 = u.dt * C::BN;
      const int nk = (ch.row_end - ch.row0 + C::BK - 1) / C::BK;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
      for (int ks = 0; ks < nk; ++ks) {
        const bool w = mbar_wait(smem_u32(&empty[stage]), phase ^ 1, p.err);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t sa = s_base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          const int r0 = ch.row0 + ks * C::BK;
          mbar_arrive_expect_tx(fb, C::SMALL_COPY + C::B_BYTES);
          // Small [BK rows][RP / 8 groups of 8 rank columns] (MN-major, no swizzle: core
          // matrices of 8 rows x 8 columns)
          tma_load_3d(ts, fb, sa, 0, r0, 0);
          if constexpr (C::V) {
            tma_load_3d(tb, fb, sb, 0, r0, d0 / 64);
          } else {
#pragma unroll
            for (int a = 0; a < C::BN / 64; ++a) tma_load_2d(tb, fb, sb + a * C::ATOM, d0 + a * 64, r0);
          }
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer (whole warp)
    // A = Small^T: MN-major, no swizzle, 8-row K groups 128 B apart, 8-column M groups
    // SMALL_NG apart (a 16-row K step advances 256 B).  B = Big: MN-major, 128-byte
    // swizzle, 64-column atoms ATOM apart, 8-row K groups 1 KB apart (a K step: 2 KB).
    const uint32_t idesc = idesc_bf16(C::BM, C::BN, 1, 1);
    const uint64_t a_desc0 = smem_desc(s_base, 128, C::SMALL_NG, kSwNone);
    const uint64_t b_desc0 = smem_desc(s_base + C::A_BYTES, C::ATOM, 1024, kSw128);
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
      const uint32_t d = tmem + b * C::BN;
      for (int ks = 0; ks < nk; ++ks) {
        const bool fok = mbar_wait(smem_u32(&full[stage]), phase, p.err);
        if (!__all_sync(0xffffffffu, fok)) { ok = false; break; }
        const int kv = rows - ks * C::BK < C::BK ? rows - ks * C::BK : C::BK;   // rows of the chunk
        const int nsteps = (kv + 15) >> 4;
        const int z = nsteps * 16 - kv;                                          // rows past its end
        if (z > 0) {
          // zero Small rows kv .. 16 nsteps - 1 in the groups that hold rank columns
          uint8_t* zs = smem + stage * C::STAGE_BYTES + kv * 16;
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
            umma_bf16(d, a_desc0 + so + kk * (256 / 16), b_desc0 + so + kk * (2048 / 16), idesc,
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
    const int et = (warp - 2) * 32 + lane;         // 0..127
    const int q4 = warp & 3;                       // TMEM lane quarter: rank rows 32 q4 ..
    const bool owner = q4 < OWNERS;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const WgradUnit u = wgrad_unit(p, nch, t);
      const WgradProblem& q = p.pr[u.prob];
      const TileInfo ch = p.chunks[u.c];
      const int b = it & 1;
      const int d0 = u.dt * C::BN;
      const int c0 = p.chunk_start[ch.e], c1 = p.chunk_start[ch.e + 1];
      bool ok = true;
      if (owner) {
        ok = mbar_wait(smem_u32(&acc_full[b]), (it >> 1) & 1, p.err);
        tc_fence_after();
      }
      if (named_bar_or(1, C::EPI_THREADS, !ok || *abort_flag != 0)) { *abort_flag = 1; break; }
#pragma unroll 1
      for (int hf = 0; hf < C::BN / C::SC; ++hf) {
        const int cb = d0 + hf * C::SC;            // first Big column of this half
        if (owner) {
          // rank row 32 q4 + lane of the accumulator -> staging row (fp32)
          const uint32_t acc = tmem + ((uint32_t)(q4 * 32) << 16) + b * C::BN + hf * C::SC;
          const int j = q4 * 32 + lane;
#pragma unroll 1
          for (int cc = 0; cc < C::SC; cc += 32) {
            uint32_t v[32];
            tmem_ld32(acc + cc, v);
            tmem_wait_ld();
            if (j < RP) {
              float4* dst = reinterpret_cast<float4*>(stg + j * C::ST_LD + cc);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
          }
          if (hf == C::BN / C::SC - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
          }
        }
        named_bar(1, C::EPI_THREADS);              // staging of this half complete
        if (c1 - c0 == 1) {
          if (q.transpose) {
            // out [E][r][D]: row j, 8 consecutive columns per store
            for (int i = et; i < p.r * (C::SC / 8); i += C::EPI_THREADS) {
              const int j = i / (C::SC / 8), cc = (i - j * (C::SC / 8)) * 8;
              if (cb + cc >= q.D) continue;
              float v[8];
#pragma unroll
              for (int x = 0; x < 8; ++x) v[x] = stg[j * C::ST_LD + cc + x];
              store_bf16x8(q.out + ((size_t)ch.e * p.r + j) * q.D + cb + cc, p.scale, v);
            }
          } else {
            // out [E][D][r]: column d, 8 consecutive rank entries per store
            for (int i = et; i < C::SC * (p.r / 8); i += C::EPI_THREADS) {
              const int dd = i / (p.r / 8), g = i - dd * (p.r / 8);
              if (cb + dd >= q.D) continue;
              float v[8];
#pragma unroll
              for (int x = 0; x < 8; ++x) v[x] = stg[(g * 8 + x) * C::ST_LD + dd];
              store_bf16x8(q.out + ((size_t)ch.e * q.D + cb + dd) * p.r + g * 8, p.scale, v);
            }
          }
        } else {
          // several chunks: fp32 partial [chunk][d][RP] of this half
          for (int dd = et; dd < C::SC; dd += C::EPI_THREADS) {
            if (cb + dd >= q.D) continue;
            float4* dst = reinterpret_cast<float4*>(q.partial + ((size_t)u.c * q.D + cb + dd) * RP);
#pragma unroll
            for (int i = 0; i < RP / 4; ++i)
              dst[i] = make_float4(stg[(4 * i) * C::ST_LD + dd], stg[(4 * i + 1) * C::ST_LD + dd],
                                   stg[(4 * i + 2) * C::ST_LD + dd], stg[(4 * i + 3) * C::ST_LD + dd]);
          }
        }
        named_bar(1, C::EPI_THREADS);              // staging is rewritten by the next half
      }
      if (c1 - c0 == 1) continue;
      // the last arriving unit of the expert's chunks sums their partials in chunk order
      // and writes the gradient
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
      if (*last_flag) {
        for (int i = et; i < C::BN * (RP / 8); i += C::EPI_THREADS) {
          const int dd = i / (RP / 8), g = i - dd * (RP / 8);
          const int dg = d0 + dd;
          if (dg >= q.D || g * 8 >= p.r) continue;
          float acc[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) acc[x] = 0.f;
          for (int cc = c0; cc < c1; ++cc) {
            const float4* src = reinterpret_cast<const float4*>(q.partial + ((size_t)cc * q.D + dg) * RP + g * 8);
            const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
            acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
            acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
          }
          if (q.transpose) {
#pragma unroll
            for (int x = 0; x < 8; ++x)
              q.out[((size_t)ch.e * p.r + g * 8 + x) * q.D + dg] = __float2bfloat16_rn(p.scale * acc[x]);
          } else {
            store_bf16x8(q.out + ((size_t)ch.e * q.D + dg) * p.r + 8 * g, p.scale, acc);
          }
        }
      }
      named_bar(1, C::EPI_THREADS);                 // the flag is rewritten next
    }
    // gradients of experts without rows are zero (D * r contiguous values in either
    // orientation): after the units, so the scan never holds up the accumulators;
    // CTA b takes experts b, b + grid, ...
    for (int e = blockIdx.x; e < p.E; e += gridDim.x) {
      if (p.chunk_start[e + 1] != p.chunk_start[e]) continue;
      const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int prob = 0; prob < p.n_problems; ++prob) {
        const WgradProblem& q = p.pr[prob];
        const int64_t n8 = (int64_t)q.D * p.r / 8;
        for (int64_t i = et; i < n8; i += C::EPI_THREADS)
          store_bf16x8(q.out + (size_t)e * q.D * p.r + i * 8, 0.f, z);
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
