// Kernel timing for the benchmark and for tracing: while enabled, every launch
// the library makes is bracketed by a pair of CUDA events recorded on the
// launch stream (as event-record nodes when the stream is being captured into a
// CUDA graph, so that a captured step is timed at each of its launches).  moe_profile_read() waits for the events and reports, per
// kernel kind, the number of launches and their summed device time.  Events
// come from a pool that grows on demand and is reused; no device memory is
// allocated.
#include <atomic>
#include <mutex>
#include <string.h>
#include <vector>

#include "internal.h"

namespace moe {

const char* const kKernelNames[K_NUM_KINDS] = {
    "route_topk",        "permute_hist",      "permute_scatter",
    "gemm_gateup_fwd",   "gemm_down_fwd",     "gemm_down_bwd",
    "gemm_gateup_bwd",   "lora_wgrad",        "unpermute_combine", "memset",
    "rank_xa",           "rank_ha",           "rank_t1",          "rank_t2",
    "router_backward",   "gemm_dw_gu",        "gemm_dw_d"};

namespace {
struct Rec {
  int kind;
  cudaEvent_t a, b;
  bool closed;
};
std::mutex g_mu;
std::atomic<bool> g_on{false};
std::atomic<uint32_t> g_kinds{~0u};     // bit k set: launches of kind k are traced
std::vector<Rec*> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

bool prof_enabled() { return g_on.load(); }

bool prof_traced(int kind) { return g_on.load() && ((g_kinds.load() >> kind) & 1u); }

// While `s` is being captured into a CUDA graph the records become event-record
// nodes of the graph (timed when the graph is launched).
cudaError_t record(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  return cudaEventRecord(e, s);
}

void* prof_begin(int kind, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  Rec* r = new Rec{kind, take_event(), take_event(), false};
  if (r->a == nullptr || r->b == nullptr) { delete r; return nullptr; }
  record(r->a, s);
  g_recs.push_back(r);
  return r;
}

void prof_end(void* token, cudaStream_t s) {
  Rec* r = static_cast<Rec*>(token);
  record(r->b, s);
  std::lock_guard<std::mutex> lk(g_mu);
  r->closed = true;
}

}  // namespace moe

using namespace moe;

extern "C" {

void moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = on != 0;
}

int moe_profile_select(const char* kinds) {
  uint32_t mask = 0;
  int n = 0;
  if (kinds == nullptr || kinds[0] == 0) {
    mask = ~0u;
  } else {
    const char* p = kinds;
    while (*p) {
      const char* q = p;
      while (*q && *q != ',') ++q;
      const size_t len = (size_t)(q - p);
      int found = -1;
      for (int k = 0; k < K_NUM_KINDS; ++k)
        if (strlen(kKernelNames[k]) == len && strncmp(kKernelNames[k], p, len) == 0) found = k;
      if (found < 0) return -1;
      mask |= 1u << found;
      ++n;
      p = *q ? q + 1 : q;
    }
  }
  g_kinds.store(mask);
  return kinds == nullptr || kinds[0] == 0 ? K_NUM_KINDS : n;
}

int moe_profile_read(int max_kinds, char* names, int name_len, int* launches, double* total_ms) {
  std::vector<int> cnt(K_NUM_KINDS, 0);
  std::vector<double> ms(K_NUM_KINDS, 0.0);
  std::vector<Rec*> recs;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    recs.swap(g_recs);
  }
  for (Rec* r : recs) {
    float t = 0.f;
    if (r->closed && cudaEventSynchronize(r->b) == cudaSuccess &&
        cudaEventElapsedTime(&t, r->a, r->b) == cudaSuccess) {
      cnt[r->kind] += 1;
      ms[r->kind] += t;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    g_pool.push_back(r->a);
    g_pool.push_back(r->b);
    delete r;
  }
  int w = 0;
  for (int k = 0; k < K_NUM_KINDS && w < max_kinds; ++k) {
    if (cnt[k] == 0) continue;
    if (names != nullptr && name_len > 0) {
      strncpy(names + (size_t)w * name_len, kKernelNames[k], name_len - 1);
      names[(size_t)w * name_len + name_len - 1] = 0;
    }
    if (launches) launches[w] = cnt[k];
    if (total_ms) total_ms[w] = ms[k];
    ++w;
  }
  return w;
}

}  // extern "C"
