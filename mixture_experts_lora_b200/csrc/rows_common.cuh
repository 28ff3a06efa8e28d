// Parameters and helpers shared by the row kernels (rows_gather.cuh: gathered X or
// w * dY rows; rows_swiglu.cuh: SwiGLU and its backward), each fused with a rank-r
// product of the Split-LoRA reordering ("Accelerating Mixture-of-Experts
// Fine-Tuning", Mathematical Formulation section 2, step 1: the compact [s, r]
// intermediate).
#pragma once

#include "common.cuh"

namespace moe {

enum RowsMode : int { ROWS_GATHER = 0, ROWS_SWIGLU = 1, ROWS_SWIGLU_BWD = 2 };

struct RowsParams {
  const TileInfo* tiles;   // 128-row tiles {e, row0, row_end}
  const int* n_tiles;
  int K;                   // columns of the rows (m, n or 2n)
  int nk;                  // K chunks of 64
  // ROWS_GATHER
  const __nv_bfloat16* src;   // [T, K]
  const int32_t* sorted_pairs;
  const float* w;             // [P] or nullptr
  int k;
  // ROWS_SWIGLU / ROWS_SWIGLU_BWD
  const __nv_bfloat16* gu;    // [P, 2n]
  const __nv_bfloat16* dh;    // [P, n]
  int n;
  // outputs
  __nv_bfloat16* rows_out;    // [P, K] (or nullptr)
  float scale;
  __nv_bfloat16* save;        // [P, ld_save]: first r_save columns of LR
  int ld_save;
  int r_save;
  __nv_bfloat16* outc;        // [P, RP]: bf16(scale * LR)
  // persistent kernels: fp32 rank-r partials of tiles split between CTAs and their
  // per-tile arrival counters (zero on entry, left zero)
  float* partial;             // [grid][2][128][RP]
  int* counters;              // [max tiles]
  int* err;
};

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint4 o;
  o.x = pack_bf16x2(x[0], x[1]);
  o.y = pack_bf16x2(x[2], x[3]);
  o.z = pack_bf16x2(x[4], x[5]);
  o.w = pack_bf16x2(x[6], x[7]);
  return o;
}
__device__ __forceinline__ void unpack8(uint4 v, float (&x)[8]) {
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x);
  x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z);
  x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}

// ---------------------------------------------------------------- persistent split
// The units of a launch (tile, 64-column stage), tile-major, are cut into G equal
// contiguous ranges, one per CTA: CTA b owns [U b / G, U (b + 1) / G).  A range
// covers whole tiles in its middle and may cut a tile at either end; the parts of
// one tile ("segments") are combined by the unit that arrives last.
__device__ __forceinline__ int64_t split_beg(int64_t U, int G, int b) { return U * b / G; }
__device__ __forceinline__ int split_owner(int64_t U, int G, int64_t u) {
  int b = (int)((u * G) / U);
  while (b + 1 < G && split_beg(U, G, b + 1) <= u) ++b;
  while (b > 0 && split_beg(U, G, b) > u) --b;
  return b;
}

// Epilogue of one segment of tile t, run by 128 threads (et = 0..127, each with
// TMEM lane quarter q4 and lane), v = the segment's fp32 rank-r row of tile row
// q4 * 32 + lane.  A segment that is the whole tile writes save = LR and
// outc = bf16(c LR); otherwise it stores an fp32 partial (slot 0: the CTA's first
// segment, 1: its last), and the last arriving segment of the tile sums the
// partials of CTAs bfirst..blast in order and writes the outputs.
template <int RP>
__device__ __forceinline__ void rows_store_lr(const RowsParams& p, int row, const float (&v)[RP]) {
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

template <int RP>
__device__ __forceinline__ void rows_segment_epilogue(const RowsParams& p, const float (&v)[RP], int et,
                                                      int rin, int t, bool whole, int cta, int slot,
                                                      int64_t U, int G, int n_it, int bar_id,
                                                      volatile int* flag) {
  const TileInfo ti = p.tiles[t];
  const int row = ti.row0 + rin;
  if (whole) {
    if (row < ti.row_end) rows_store_lr<RP>(p, row, v);
    return;
  }
  float4* dst = reinterpret_cast<float4*>(p.partial + (((size_t)cta * 2 + slot) * 128 + rin) * RP);
#pragma unroll
  for (int i = 0; i < RP / 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  __threadfence();
  named_bar(bar_id, 128);
  const int bfirst = split_owner(U, G, (int64_t)t * n_it);
  const int blast = split_owner(U, G, (int64_t)(t + 1) * n_it - 1);
  if (et == 0) {
    const int last = atomicAdd(&p.counters[t], 1) == blast - bfirst;
    if (last) {
      p.counters[t] = 0;          // ready for the next launch
      __threadfence();
    }
    *flag = last;
  }
  named_bar(bar_id, 128);
  if (*flag && row < ti.row_end) {
    float acc[RP];
#pragma unroll
    for (int i = 0; i < RP; ++i) acc[i] = 0.f;
    for (int cb = bfirst; cb <= blast; ++cb) {
      const int cs = split_beg(U, G, cb) / n_it == t ? 0 : 1;
      const float4* src = reinterpret_cast<const float4*>(p.partial + (((size_t)cb * 2 + cs) * 128 + rin) * RP);
#pragma unroll
      for (int i = 0; i < RP / 4; ++i) {
        const float4 x = __ldcg(src + i);
        acc[4 * i] += x.x;
        acc[4 * i + 1] += x.y;
        acc[4 * i + 2] += x.z;
        acc[4 * i + 3] += x.w;
      }
    }
    rows_store_lr<RP>(p, row, acc);
  }
  named_bar(bar_id, 128);         // the flag is rewritten by the next segment
}

}  // namespace moe
