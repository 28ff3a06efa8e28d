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

}  // namespace moe
