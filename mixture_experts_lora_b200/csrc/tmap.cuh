// Host helpers shared by the launchers: TMA tensor-map encoding (through the driver
// entry point, so the library needs no link-time libcuda) and kernel attributes.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace moe {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

inline CUtensorMapSwizzle swz_for_bytes(int inner_bytes) {
  switch (inner_bytes) {
    case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
    case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
    default: return CU_TENSOR_MAP_SWIZZLE_128B;
  }
}

// bf16 tensor of `rank` dims (dims[0] innermost, contiguous), box `box`.  Elements of
// a box outside the tensor read as zero.
inline bool encode(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base),
                  reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes),
                  reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [rows, cols] with row stride ld elements, box [box_rows, box_cols], swizzle by the
// box's row bytes (32, 64 or 128) unless `plain`.
inline bool encode2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                     uint32_t box_rows, uint32_t box_cols, bool plain = false) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t str[1] = {ld * 2};
  const uint32_t box[2] = {box_cols, box_rows};
  return encode(m, base, 2, dims, str, box,
                plain ? CU_TENSOR_MAP_SWIZZLE_NONE : swz_for_bytes((int)box_cols * 2));
}

// [E, rows, cols] row-major, box [1, box_rows, box_cols]
inline bool encode3d(CUtensorMap* m, const void* base, uint64_t E, uint64_t rows, uint64_t cols,
                     uint32_t box_rows, uint32_t box_cols) {
  const uint64_t dims[3] = {cols, rows, E};
  const uint64_t str[2] = {cols * 2, rows * cols * 2};
  const uint32_t box[3] = {box_cols, box_rows, 1};
  return encode(m, base, 3, dims, str, box, swz_for_bytes((int)box_cols * 2));
}

// [E, R, C] row-major (C % 64 == 0) seen as [E][C/64 atoms][R][64]: a box of
// `box_atoms` 64-wide atoms of `box_r` rows lands as atom-major 128-byte-swizzled
// tiles, so one copy fills a whole operand tile.  per_expert = false: a 2-D tensor
// [R, C] (3-D view, E ignored); true: always the 4-D view, even for E = 1, since the
// kernels address it with four coordinates.
inline bool encode_atoms(CUtensorMap* m, const void* base, bool per_expert, uint64_t E, uint64_t R,
                         uint64_t C, uint32_t box_r, uint32_t box_atoms) {
  const uint64_t dims[4] = {64, R, C / 64, E};
  const uint64_t str[3] = {C * 2, 128, R * C * 2};
  const uint32_t box[4] = {64, box_r, box_atoms, 1};
  return encode(m, base, per_expert ? 4 : 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <class Kern>
cudaError_t ensure_smem(Kern kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace moe
