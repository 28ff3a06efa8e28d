// C ABI of the layer (include/moelora.h): argument checks, workspace layout and
// the launch sequence of each call.  Every call is asynchronous on the caller's
// stream; the library allocates nothing.
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

#include <nvtx3/nvToolsExt.h>

namespace moe {

// Device status word (one per device); kernels set it with atomicCAS, the host
// reads and clears it in moe_get_device_error().
__device__ int g_moe_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kTileRows = 128;
constexpr int kGemmChunkRows = 256;

// Device address of g_moe_status in the current context, looked up once per
// (device, context): a device reset or a new primary context re-resolves it.
int* status_ptr() {
  static std::mutex mu;
  static int* ptrs[kMaxDevices] = {nullptr};
  static void* ctxs[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* ctx = current_context();
  std::lock_guard<std::mutex> lk(mu);
  if (ptrs[dev] == nullptr || ctxs[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
    ctxs[dev] = ctx;
  }
  return ptrs[dev];
}

int device_sms() {
  static int sms[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (sms[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    sms[dev] = v > 0 ? v : 148;
  }
  return sms[dev];
}

inline int rank_padded(int r) { return r <= 16 ? 16 : r <= 32 ? 32 : r <= 64 ? 64 : 128; }

// Row chunk of the adapter-gradient kernel.  An expert cut into several chunks
// needs fp32 partials and a last-arriver sum per 256-column unit, and the cut
// leaves remainder chunks of a few rows whose units are all epilogue; one chunk
// per expert avoids both.  Start at 1024 rows and double while an expert of 1.5x
// the average rows would still be cut, as long as the first launch keeps at least
// kMinWgradUnits units (expert chunks x 256-column tiles of both problems) to
// spread over the SMs.  At T = 32768, k = 8, E = 256 this gives 2048 rows.
constexpr int64_t kMinWgradUnits = 296;
inline int64_t chunk_rows_for(const moe_dims_t& d, int64_t P) {
  const int64_t avg = d.E > 0 ? (P + d.E - 1) / d.E : 0;
  const int64_t dtiles = (d.n + 255) / 256 + (d.m + 255) / 256;
  int64_t chunk = 1024;
  while (chunk < 8192 && avg + avg / 2 > chunk) {
    const int64_t nxt = 2 * chunk;
    const int64_t units = (int64_t)d.E * ((avg + nxt - 1) / nxt) * dtiles;
    if (units < kMinWgradUnits) break;
    chunk = nxt;
  }
  return chunk;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_dims(const moe_dims_t* d) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->T < 0) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(d->scale)) return MOE_ERR_INVALID_ARG;
  if (d->k < 1 || d->k > 32 || d->E < d->k || d->E > 1024) return MOE_ERR_UNSUPPORTED;
  if (d->m < 16 || d->n < 16 || d->m % 16 != 0 || d->n % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (d->r < 8 || d->r > 128 || d->r % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (d->T * (int64_t)d->k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  // largest row index times the widest row must stay within 32-bit tile coordinates
  if ((int64_t)d->m > (1 << 20) || (int64_t)d->n > (1 << 19)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Workspace regions (byte offsets), one layout for every call.
struct Layout {
  int64_t P;
  int rp;
  int max_row_tiles, max_gchunks, max_chunks, chunk_rows, perm_chunks;
  size_t hist, tiles, n_tiles, gchunks, n_gchunks, chunks, n_chunks, chunk_start;
  int max_dtiles;            // 128-column tiles of the widest adapter gradient
  size_t rows;               // expert-ordered w dY (the backward's token operand)
  size_t dh, dgu, t1, t2, lrc1, lrc2, partial, partial2;
  size_t counters;           // arrival counters of the four adapter gradients
  size_t total;
};

Layout make_layout(const moe_dims_t& d) {
  Layout L{};
  L.P = d.T * d.k;
  L.rp = rank_padded(d.r);
  L.max_row_tiles = (int)((L.P + kTileRows - 1) / kTileRows) + d.E;
  L.max_gchunks = (int)((L.P + kGemmChunkRows - 1) / kGemmChunkRows) + d.E;
  L.chunk_rows = (int)chunk_rows_for(d, L.P);
  L.max_chunks = (int)((L.P + L.chunk_rows - 1) / L.chunk_rows) + d.E;
  {
    // chunks of moe_permute (kPermuteChunk pairs) or of moe_route_permute (whole tokens)
    const int64_t tpb = route_tokens_per_chunk(d.k);
    const int64_t a = (L.P + kPermuteChunk - 1) / kPermuteChunk, b = (d.T + tpb - 1) / tpb;
    L.perm_chunks = (int)(a > b ? a : b);
  }
  const size_t E = d.E, m = d.m, n = d.n, rp = L.rp, P = (size_t)L.P;
  const size_t dmax = m > 2 * n ? m : 2 * n;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  L.hist = take(permute_scratch_ints(L.perm_chunks, d.E) * 4);
  L.tiles = take((size_t)L.max_row_tiles * sizeof(TileInfo));
  L.n_tiles = take(4);
  L.gchunks = take((size_t)L.max_gchunks * sizeof(TileInfo));
  L.n_gchunks = take(4);
  L.chunks = take((size_t)L.max_chunks * sizeof(TileInfo));
  L.n_chunks = take(4);
  L.chunk_start = take((E + 1) * 4);
  L.rows = take(P * m * 2);
  L.dh = take(P * n * 2);
  L.dgu = take(P * 2 * n * 2);
  L.t1 = take(P * rp * 2);
  L.t2 = take(P * rp * 2);
  L.lrc1 = take(P * rp * 2);
  L.lrc2 = take(P * rp * 2);
  L.partial = take((size_t)L.max_chunks * dmax * rp * 4);
  L.partial2 = take((size_t)L.max_chunks * dmax * rp * 4);
  L.max_dtiles = (int)((dmax + 127) / 128);
  L.counters = take((size_t)4 * E * L.max_dtiles * 4);
  L.total = off;
  return L;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                                  \
  do {                                                 \
    cudaError_t e_ = (expr);                           \
    if (e_ != cudaSuccess) return MOE_ERR_CUDA;        \
  } while (0)

// Common set-up of the grouped GEMMs: operand pointers, and the description of the
// tables that the first kernel of the call builds from the offsets (tb).  Adapters are
// used as given: ranks r .. rp - 1 read as zero through the tensor maps.
moe_status_t prepare(const moe_dims_t& d, const Layout& L, void* ws, const int32_t* offsets,
                     const uint16_t* W_gu, const uint16_t* W_d, const uint16_t* A_gu,
                     const uint16_t* B_gu, const uint16_t* A_d, const uint16_t* B_d,
                     bool with_chunks, GemmShape* g, LayerPtrs* w, TableBuild* tb) {
  int* err = status_ptr();
  if (err == nullptr) return MOE_ERR_CUDA;
  *tb = TableBuild{};
  tb->offsets = offsets;
  tb->E = d.E;
  tb->tile_rows = kTileRows;
  tb->tiles = at<TileInfo>(ws, L.tiles);
  tb->n_tiles = at<int>(ws, L.n_tiles);
  tb->gchunk_rows = kGemmChunkRows;
  tb->gchunks = at<TileInfo>(ws, L.gchunks);
  tb->n_gchunks = at<int>(ws, L.n_gchunks);
  tb->chunk_rows = L.chunk_rows;
  tb->chunks = with_chunks ? at<TileInfo>(ws, L.chunks) : nullptr;
  tb->n_chunks = at<int>(ws, L.n_chunks);
  tb->chunk_start = at<int32_t>(ws, L.chunk_start);
  tb->zero = at<int>(ws, L.counters);
  tb->n_zero = with_chunks ? 4 * d.E * L.max_dtiles : 0;
  w->W_gu = W_gu;
  w->W_d = W_d;
  w->A_gu = A_gu; w->B_gu = B_gu; w->A_d = A_d; w->B_d = B_d;
  g->P = L.P;
  g->m = d.m;
  g->n = d.n;
  g->E = d.E;
  g->r = d.r;
  g->rp = L.rp;
  g->scale = d.scale;
  g->max_row_tiles = L.max_row_tiles;
  g->tiles = at<TileInfo>(ws, L.tiles);
  g->n_row_tiles = at<int>(ws, L.n_tiles);
  g->max_gchunks = L.max_gchunks;
  g->gchunks = at<TileInfo>(ws, L.gchunks);
  g->n_gchunks = at<int>(ws, L.n_gchunks);
  g->err = err;
  g->num_sms = device_sms();
  return MOE_OK;
}

// The backward pass.  Adapter gradients when dA_gu.. are given (all four or none),
// expert-weight gradients (full fine-tuning) when dW_gu, dW_d are given; each weight
// gradient runs while its sorted operands are at hand (w dY in the row buffer after
// the rank-r kernel; X sorted saved by the forward).
moe_status_t backward(
    const moe_dims_t* dims, const moe_bf16_t* dY, const float* topk_w,
    const int32_t* sorted_pairs, const int32_t* offsets, const moe_bf16_t* W_gu,
    const moe_bf16_t* W_d, const moe_bf16_t* A_gu, const moe_bf16_t* B_gu, const moe_bf16_t* A_d,
    const moe_bf16_t* B_d, const moe_bf16_t* save_Xs, const moe_bf16_t* save_GU,
    const moe_bf16_t* save_H, const moe_bf16_t* save_XA, const moe_bf16_t* save_HA,
    moe_bf16_t* dX_sorted, moe_bf16_t* dA_gu, moe_bf16_t* dB_gu, moe_bf16_t* dA_d,
    moe_bf16_t* dB_d, moe_bf16_t* dW_gu, moe_bf16_t* dW_d, void* ws, size_t ws_bytes,
    void* stream) {
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t d = *dims;
  const bool lora = dA_gu != nullptr, full = dW_gu != nullptr;
  const void* outs[] = {dA_gu, dB_gu, dA_d, dB_d, dW_gu, dW_d};
  for (const void* p : outs)
    if (p != nullptr && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t E = d.E, m = d.m, n = d.n, r = d.r;
  if (d.T == 0) {
    if (lora) {
      MOE_TRY(launch_zero(dA_gu, E * m * r * 2, s));
      MOE_TRY(launch_zero(dB_gu, E * r * 2 * n * 2, s));
      MOE_TRY(launch_zero(dA_d, E * n * r * 2, s));
      MOE_TRY(launch_zero(dB_d, E * r * m * 2, s));
    }
    if (full) {
      MOE_TRY(launch_zero(dW_gu, E * m * 2 * n * 2, s));
      MOE_TRY(launch_zero(dW_d, E * n * m * 2, s));
    }
    return MOE_OK;
  }
  const void* ins[] = {dY, W_gu, W_d, A_gu, B_gu, A_d, B_d, save_Xs, save_GU, save_H, save_XA,
                       save_HA, dX_sorted, ws};
  for (const void* p : ins)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (topk_w == nullptr || sorted_pairs == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(d);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  GemmShape g;
  LayerPtrs w;
  TableBuild tb;
  st = prepare(d, L, ws, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d, true, &g, &w, &tb);
  if (st != MOE_OK) return st;
  uint16_t* rows = at<uint16_t>(ws, L.rows);
  uint16_t* dh = at<uint16_t>(ws, L.dh);
  uint16_t* dgu = at<uint16_t>(ws, L.dgu);
  uint16_t* t1 = at<uint16_t>(ws, L.t1);
  uint16_t* t2 = at<uint16_t>(ws, L.t2);
  uint16_t* lrc1 = at<uint16_t>(ws, L.lrc1);
  uint16_t* lrc2 = at<uint16_t>(ws, L.lrc2);
  float* partial = at<float>(ws, L.partial);
  float* partial2 = at<float>(ws, L.partial2);
  const TileInfo* chunks = at<TileInfo>(ws, L.chunks);
  const int* n_chunks = at<int>(ws, L.n_chunks);
  const int32_t* chunk_start = at<int32_t>(ws, L.chunk_start);
  int* counters = at<int>(ws, L.counters);
  const size_t cstride = (size_t)d.E * L.max_dtiles;
  const int rp = L.rp;
  // dy = w dY[t] in expert order (the row buffer), T1 = dy B_d^T (kept for dA_d) and
  // bf16(c T1); this first kernel also builds the call's tables
  MOE_TRY(launch_rank_gathered(K_RANK_T1, g, dY, d.m, sorted_pairs, d.k, topk_w, rows, w.B_d,
                               false, t1, rp, rp, lrc1, &tb, s));
  // dH = dy W_d^T + (c T1) A_d^T
  MOE_TRY(launch_gemm_down_bwd(g, w, rows, lrc1, dh, s));
  // dA_d = c H^T T1 and dB_d = c HA^T dy, one launch
  if (lora) {
    const WgradJob jobs[2] = {{save_H, d.n, t1, rp, false, dA_d, partial, counters},
                              {rows, d.m, save_HA, d.r, true, dB_d, partial2, counters + cstride}};
    MOE_TRY(launch_lora_wgrad(g, jobs, 2, chunks, n_chunks, L.max_chunks, chunk_start, s));
  }
  // dW_d = H^T dy per expert
  if (full) MOE_TRY(launch_expert_dw(K_GEMM_DW_D, g, offsets, save_H, d.n, rows, d.m, dW_d, s));
  // dGU = SwiGLU backward of dH, T2 = dGU B_gu^T and bf16(c T2)
  MOE_TRY(launch_rank_dswiglu(g, dh, save_GU, w.B_gu, dgu, t2, rp, rp, lrc2, s));
  // dX_sorted = dGU W_gu^T + (c T2) A_gu^T
  MOE_TRY(launch_gemm_gateup_bwd(g, w, dgu, lrc2, dX_sorted, s));
  // dB_gu = c XA^T dGU and dA_gu = c X^T T2 (X in expert order from the forward), one launch
  if (lora) {
    const WgradJob jobs[2] = {
        {dgu, 2 * d.n, save_XA, d.r, true, dB_gu, partial, counters + 2 * cstride},
        {save_Xs, d.m, t2, rp, false, dA_gu, partial2, counters + 3 * cstride}};
    MOE_TRY(launch_lora_wgrad(g, jobs, 2, chunks, n_chunks, L.max_chunks, chunk_start, s));
  }
  // dW_gu = X^T dGU per expert
  if (full) MOE_TRY(launch_expert_dw(K_GEMM_DW_GU, g, offsets, save_Xs, d.m, dgu, 2 * d.n, dW_gu, s));
  return MOE_OK;
}

}  // namespace

void* current_context() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

int* moe_status_word() { return status_ptr(); }

}  // namespace moe

using namespace moe;

namespace {
// An NVTX range named after the entry point around each call (visible to profilers
// that record NVTX; a no-op otherwise).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace

extern "C" {

size_t moe_workspace_bytes(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  return make_layout(*dims).total;
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_INDEX: return "expert id out of range (device)";
    case MOE_ERR_TIMEOUT: return "bounded wait expired (device)";
    case MOE_ERR_DEVICE_CHECK: return "permutation invariant broken (device check)";
  }
  return "unknown status";
}

moe_status_t moe_get_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int* p = status_ptr();
  if (p == nullptr) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status_t>(v);
}

moe_status_t moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k,
                            int32_t* topk_ids, float* topk_w, void* stream) {
  NvtxRange nr("moe_route_topk");
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > 32 || E < k || E > 1024) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (logits == nullptr || topk_ids == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_route_topk(logits, T, E, k, topk_ids, topk_w, status_ptr(),
                                       static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_permute(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E, int32_t* counts,
                         int32_t* offsets, int32_t* sorted_pairs, int32_t* pair_pos, void* ws,
                         size_t ws_bytes, void* stream) {
  NvtxRange nr("moe_permute");
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > 32 || E < k || E > 1024) return MOE_ERR_UNSUPPORTED;
  const int64_t P = T * (int64_t)k;
  if (P >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (counts == nullptr || offsets == nullptr || ws == nullptr) return MOE_ERR_INVALID_ARG;
  if (P > 0 && (topk_ids == nullptr || sorted_pairs == nullptr || pair_pos == nullptr))
    return MOE_ERR_INVALID_ARG;
  const size_t need = permute_scratch_ints((P + kPermuteChunk - 1) / kPermuteChunk, E) * 4;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE;
  int* err = status_ptr();
  if (err == nullptr) return MOE_ERR_CUDA;
  return cuda_status(launch_permute(topk_ids, P, E, counts, offsets, sorted_pairs, pair_pos,
                                    static_cast<int32_t*>(ws), err,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_route_permute(const float* logits, int64_t T, int32_t E, int32_t k,
                               int32_t* topk_ids, float* topk_w, int32_t* counts, int32_t* offsets,
                               int32_t* sorted_pairs, int32_t* pair_pos, void* ws, size_t ws_bytes,
                               void* stream) {
  NvtxRange nr("moe_route_permute");
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > 32 || E < k || E > 1024) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (counts == nullptr || offsets == nullptr || ws == nullptr) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (logits == nullptr || topk_ids == nullptr || topk_w == nullptr ||
                sorted_pairs == nullptr || pair_pos == nullptr))
    return MOE_ERR_INVALID_ARG;
  const int64_t tpb = route_tokens_per_chunk(k);
  if (ws_bytes < permute_scratch_ints((T + tpb - 1) / tpb, E) * 4) return MOE_ERR_WORKSPACE;
  if (status_ptr() == nullptr) return MOE_ERR_CUDA;
  return cuda_status(launch_route_permute(logits, T, E, k, topk_ids, topk_w, counts, offsets,
                                          sorted_pairs, pair_pos, static_cast<int32_t*>(ws),
                                          static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_check_permutation(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                                   const int32_t* counts, const int32_t* offsets,
                                   const int32_t* sorted_pairs, const int32_t* pair_pos,
                                   void* stream) {
  NvtxRange nr("moe_check_permutation");
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > 32 || E < k || E > 1024) return MOE_ERR_UNSUPPORTED;
  const int64_t P = T * (int64_t)k;
  if (P >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
  if (P > 0 && (topk_ids == nullptr || sorted_pairs == nullptr || pair_pos == nullptr))
    return MOE_ERR_INVALID_ARG;
  int* err = status_ptr();
  if (err == nullptr) return MOE_ERR_CUDA;
  return cuda_status(launch_check_permutation(topk_ids, P, E, counts, offsets, sorted_pairs, pair_pos,
                                              err, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_gemm_lora_fwd(const moe_dims_t* dims, const moe_bf16_t* X,
                                       const int32_t* sorted_pairs, const int32_t* offsets,
                                       const moe_bf16_t* W_gu, const moe_bf16_t* W_d,
                                       const moe_bf16_t* A_gu, const moe_bf16_t* B_gu,
                                       const moe_bf16_t* A_d, const moe_bf16_t* B_d,
                                       moe_bf16_t* Y_sorted, moe_bf16_t* save_Xs,
                                       moe_bf16_t* save_GU, moe_bf16_t* save_H,
                                       moe_bf16_t* save_XA, moe_bf16_t* save_HA, void* ws,
                                       size_t ws_bytes, void* stream) {
  NvtxRange nr("moe_grouped_gemm_lora_fwd");
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t d = *dims;
  if (d.T == 0) return MOE_OK;
  const void* ptrs[] = {X, W_gu, W_d, A_gu, B_gu, A_d, B_d, Y_sorted, save_Xs, save_GU, save_H,
                        save_XA, save_HA, ws};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (sorted_pairs == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(d);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GemmShape g;
  LayerPtrs w;
  TableBuild tb;
  st = prepare(d, L, ws, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d, false, &g, &w, &tb);
  if (st != MOE_OK) return st;
  uint16_t* xac = at<uint16_t>(ws, L.lrc1);
  uint16_t* hac = at<uint16_t>(ws, L.lrc2);
  // X rows in expert order (saved), XA = X A_gu (saved) and bf16(c XA); this first
  // kernel also builds the call's tables
  MOE_TRY(launch_rank_gathered(K_RANK_XA, g, X, d.m, sorted_pairs, d.k, nullptr, save_Xs, w.A_gu,
                               true, save_XA, d.r, d.r, xac, &tb, s));
  // GU = X W_gu + (c XA) B_gu and H = silu(g) u, fused
  MOE_TRY(launch_gemm_gateup_fwd(g, w, save_Xs, xac, save_GU, save_H, s));
  // HA = H A_d (saved) and bf16(c HA)
  MOE_TRY(launch_rank_sorted(K_RANK_HA, g, save_H, d.n, w.A_d, true, save_HA, d.r, d.r, hac, s));
  // Y = H W_d + (c HA) B_d
  MOE_TRY(launch_gemm_down_fwd(g, w, save_H, hac, Y_sorted, s));
  return MOE_OK;
}

moe_status_t moe_grouped_gemm_lora_bwd(
    const moe_dims_t* dims, const moe_bf16_t* dY, const float* topk_w,
    const int32_t* sorted_pairs, const int32_t* offsets, const moe_bf16_t* W_gu,
    const moe_bf16_t* W_d, const moe_bf16_t* A_gu, const moe_bf16_t* B_gu, const moe_bf16_t* A_d,
    const moe_bf16_t* B_d, const moe_bf16_t* save_Xs, const moe_bf16_t* save_GU,
    const moe_bf16_t* save_H, const moe_bf16_t* save_XA, const moe_bf16_t* save_HA,
    moe_bf16_t* dX_sorted, moe_bf16_t* dA_gu, moe_bf16_t* dB_gu, moe_bf16_t* dA_d,
    moe_bf16_t* dB_d, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nr("moe_grouped_gemm_lora_bwd");
  if (dA_gu == nullptr || dB_gu == nullptr || dA_d == nullptr || dB_d == nullptr)
    return MOE_ERR_INVALID_ARG;
  return backward(dims, dY, topk_w, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d,
                  save_Xs, save_GU, save_H, save_XA, save_HA, dX_sorted, dA_gu, dB_gu, dA_d, dB_d,
                  nullptr, nullptr, ws, ws_bytes, stream);
}

moe_status_t moe_grouped_gemm_full_bwd(
    const moe_dims_t* dims, const moe_bf16_t* dY, const float* topk_w,
    const int32_t* sorted_pairs, const int32_t* offsets, const moe_bf16_t* W_gu,
    const moe_bf16_t* W_d, const moe_bf16_t* A_gu, const moe_bf16_t* B_gu, const moe_bf16_t* A_d,
    const moe_bf16_t* B_d, const moe_bf16_t* save_Xs, const moe_bf16_t* save_GU,
    const moe_bf16_t* save_H, const moe_bf16_t* save_XA, const moe_bf16_t* save_HA,
    moe_bf16_t* dX_sorted, moe_bf16_t* dW_gu, moe_bf16_t* dW_d, moe_bf16_t* dA_gu,
    moe_bf16_t* dB_gu, moe_bf16_t* dA_d, moe_bf16_t* dB_d, void* ws, size_t ws_bytes,
    void* stream) {
  NvtxRange nr("moe_grouped_gemm_full_bwd");
  if (dW_gu == nullptr || dW_d == nullptr) return MOE_ERR_INVALID_ARG;
  const int given = (dA_gu != nullptr) + (dB_gu != nullptr) + (dA_d != nullptr) + (dB_d != nullptr);
  if (given != 0 && given != 4) return MOE_ERR_INVALID_ARG;
  return backward(dims, dY, topk_w, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d,
                  save_Xs, save_GU, save_H, save_XA, save_HA, dX_sorted, dA_gu, dB_gu, dA_d, dB_d,
                  dW_gu, dW_d, ws, ws_bytes, stream);
}

moe_status_t moe_router_backward(const moe_bf16_t* dY, const moe_bf16_t* Y_sorted,
                                 const int32_t* topk_ids, const float* topk_w,
                                 const int32_t* pair_pos, int64_t T, int32_t k, int32_t E,
                                 int32_t m, float* dlogits, void* stream) {
  NvtxRange nr("moe_router_backward");
  if (T < 0 || m < 8) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > 32 || E < k || E > 1024 || m % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!aligned16(dY) || !aligned16(Y_sorted) || topk_ids == nullptr || topk_w == nullptr ||
      pair_pos == nullptr || dlogits == nullptr)
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_router_backward(dY, Y_sorted, topk_ids, topk_w, pair_pos, T, k, E, m,
                                            dlogits, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_unpermute_combine(const moe_bf16_t* Y_sorted, const float* topk_w,
                                   const int32_t* pair_pos, int64_t T, int32_t k, int32_t m,
                                   moe_bf16_t* Y, void* stream) {
  NvtxRange nr("moe_unpermute_combine");
  if (T < 0 || k < 1 || m < 8) return MOE_ERR_INVALID_ARG;
  if (m % 8 != 0 || k > 1024) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!aligned16(Y_sorted) || !aligned16(Y) || pair_pos == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(
      launch_combine(Y_sorted, topk_w, pair_pos, T, k, m, Y, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
