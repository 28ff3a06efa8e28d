// moe_permute_noalloc: the counting-sort permute with its scratch memory built
// into the library, for callers that cannot allocate device memory themselves.
//
// The per-chunk histograms that moe_permute keeps in the caller's workspace live
// here in a file-scope device array of fixed size, present on every GPU that loads
// the library until the process exits.  Host code cannot pass the array's name to
// a kernel (on the host it names a stand-in, not device memory), so the device
// address is looked up with cudaGetSymbolAddress, once per device and context, and
// cached.
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// 2^19 int32 = 2 MiB: room for ceil(T*k / kPermuteChunk) * E histogram entries, then
// the expert totals (E <= 1024, one per kTotStride ints) and the arrival counter of
// the histogram launch.
constexpr size_t kPermuteScratchInts = size_t(1) << 19;
constexpr size_t kTotalsInts = size_t(1024) * kTotStride;
__device__ __align__(256) int32_t g_permute_scratch[kPermuteScratchInts + kTotalsInts + 64];

constexpr int kMaxDevices = 64;

// Device address of g_permute_scratch on the current device (nullptr on failure),
// looked up with that device current the first time a (device, context) is seen: a
// device reset or a new primary context gets a fresh lookup, never a stale address.
int32_t* permute_scratch() {
  static std::mutex mu;
  static int32_t* ptrs[kMaxDevices] = {nullptr};
  static void* ctxs[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* ctx = current_context();
  std::lock_guard<std::mutex> lk(mu);
  if (ptrs[dev] == nullptr || ctxs[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int32_t*>(p);
    ctxs[dev] = ctx;
  }
  return ptrs[dev];
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_permute_noalloc(const int32_t* topk_ids, int64_t T, int32_t k,
                                            int32_t E, int32_t* counts, int32_t* offsets,
                                            int32_t* sorted_pairs, int32_t* pair_pos,
                                            void* stream) {
  struct Range {
    Range() { nvtxRangePushA("moe_permute_noalloc"); }
    ~Range() { nvtxRangePop(); }
  } range;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > 32 || E < k || E > 1024) return MOE_ERR_UNSUPPORTED;
  const int64_t P = T * (int64_t)k;
  if (P >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
  if (P > 0 && (topk_ids == nullptr || sorted_pairs == nullptr || pair_pos == nullptr))
    return MOE_ERR_INVALID_ARG;
  // every histogram entry is written before it is read; the totals and the arrival
  // counter after them are zeroed by the call itself
  const int64_t n_hist = ((P + kPermuteChunk - 1) / kPermuteChunk) * (int64_t)E;
  if (n_hist > (int64_t)kPermuteScratchInts) return MOE_ERR_WORKSPACE;
  static_assert(kPermuteScratchInts + kTotalsInts + 1 <= sizeof(g_permute_scratch) / sizeof(int32_t),
                "histograms, totals and counter");
  int32_t* scratch = permute_scratch();
  int* err = moe_status_word();
  if (scratch == nullptr || err == nullptr) return MOE_ERR_CUDA;
  const cudaError_t st = launch_permute(topk_ids, P, E, counts, offsets, sorted_pairs, pair_pos,
                                        scratch, err, static_cast<cudaStream_t>(stream));
  return st == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
