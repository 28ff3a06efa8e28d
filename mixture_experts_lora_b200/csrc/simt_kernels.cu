// SIMT kernels of the layer: top-k routing, the stable counting-sort permute,
// tile tables, weighted un-permute combine and router backward.
// All are HBM- or latency-bound; they use coalesced 16-byte accesses and warp
// primitives, no floating-point atomics.
#include "common.cuh"
#include "internal.h"

namespace moe {

// ------------------------------------------------------------------ routing
// One warp per token.  The k rounds each pick the largest remaining logit, lower
// expert id on ties, and the weights are a softmax over the k picked logits.  Router
// equation: "Accelerating Mixture-of-Experts Fine-Tuning", section "The Dynamic
// Dispatch Bottleneck in Mixture-of-Experts Architectures".
//
// Values are compared through an order-preserving unsigned key.  Lane l holds the
// logits of experts l, l + 32, ...; up to 256 experts these PL <= 8 logits are sorted
// once in registers (largest first, lower id first on ties: a total order, so any
// sorting network gives the same list), and each round is two warp max-reductions
// (redux.sync) over the lanes' list heads, after which the winning lane drops its
// head.  Wider rows stage the logits in shared memory and every lane rescans its
// untaken candidates each round.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                       // -0 ties with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // larger float -> larger key
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Lane j < k receives the j-th pick: its expert id and logit.
template <int PL>
__device__ __forceinline__ void warp_topk_sorted(const float* __restrict__ src, int E, int k,
                                                 int lane, float& my_val, int& my_id) {
  uint32_t key[PL];
  int id[PL];
#pragma unroll
  for (int q = 0; q < PL; ++q) {
    id[q] = lane + 32 * q;
    key[q] = id[q] < E ? order_key(__ldg(src + id[q])) : 0u;
  }
  // odd-even transposition sort, best first; ids >= E (no expert) sort last
#pragma unroll
  for (int rnd = 0; rnd < PL; ++rnd) {
#pragma unroll
    for (int q = rnd & 1; q + 1 < PL; q += 2) {
      const bool vq = id[q] < E, vn = id[q + 1] < E;
      const bool swap =
          vn && (!vq || key[q + 1] > key[q] || (key[q + 1] == key[q] && id[q + 1] < id[q]));
      if (swap) {
        const uint32_t tk = key[q]; key[q] = key[q + 1]; key[q + 1] = tk;
        const int ti = id[q]; id[q] = id[q + 1]; id[q + 1] = ti;
      }
    }
  }
  for (int j = 0; j < k; ++j) {
    const bool has = id[0] < E;
    const uint32_t wkey = __reduce_max_sync(0xffffffffu, has ? key[0] : 0u);
    const uint32_t wlo = __reduce_max_sync(0xffffffffu, (has && key[0] == wkey) ? ~(uint32_t)id[0] : 0u);
    const int bi = (int)(~wlo);
    if (lane == j) { my_val = key_value(wkey); my_id = bi; }
    if (has && id[0] == bi) {
#pragma unroll
      for (int q = 0; q + 1 < PL; ++q) { key[q] = key[q + 1]; id[q] = id[q + 1]; }
      key[PL - 1] = 0u;
      id[PL - 1] = E;
    }
  }
}

// Rows of more than 256 experts: `row` is the token's logits in shared memory.
__device__ __forceinline__ void warp_topk_scan(const float* row, int E, int k, int lane,
                                               float& my_val, int& my_id) {
  const int per_lane = (E + 31) >> 5;
  uint32_t taken = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bkey = 0, blo = 0;          // blo = ~e of the lane's candidate (0: none)
    for (int i = 0; i < per_lane; ++i) {
      const int e = lane + 32 * i;
      if (e >= E || ((taken >> i) & 1u)) continue;
      const uint32_t key = order_key(row[e]);
      if (blo == 0 || key > bkey) { bkey = key; blo = ~(uint32_t)e; }
    }
    const uint32_t wkey = __reduce_max_sync(0xffffffffu, blo != 0 ? bkey : 0u);
    const uint32_t wlo = __reduce_max_sync(0xffffffffu, (blo != 0 && bkey == wkey) ? blo : 0u);
    const int bi = (int)(~wlo);
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) { my_val = key_value(wkey); my_id = bi; }
  }
}

// Token t's top k (lane j < k gets pick j) and its softmax weight.  s_row: this
// warp's E floats of shared memory, used for rows of more than 256 experts.
__device__ __forceinline__ void warp_route(const float* __restrict__ logits, int64_t t, int E,
                                           int k, int lane, float* s_row, int& my_id,
                                           float& my_w) {
  const float* src = logits + t * E;
  float my_val = 0.f;
  my_id = 0;
  if (E <= 32) warp_topk_sorted<1>(src, E, k, lane, my_val, my_id);
  else if (E <= 64) warp_topk_sorted<2>(src, E, k, lane, my_val, my_id);
  else if (E <= 128) warp_topk_sorted<4>(src, E, k, lane, my_val, my_id);
  else if (E <= 256) warp_topk_sorted<8>(src, E, k, lane, my_val, my_id);
  else {
    for (int e = lane; e < E; e += 32) s_row[e] = src[e];
    __syncwarp();
    warp_topk_scan(s_row, E, k, lane, my_val, my_id);
  }
  const float vmax = __shfl_sync(0xffffffffu, my_val, 0);
  const float z = lane < k ? expf(my_val - vmax) : 0.f;
  float sum = z;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  my_w = z / sum;
}

__global__ void route_topk_kernel(const float* __restrict__ logits, int64_t T, int E, int k,
                                  int32_t* __restrict__ ids, float* __restrict__ wout) {
  pdl_begin();
  extern __shared__ float s_logits[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  int my_id;
  float my_w;
  warp_route(logits, t, E, k, lane, s_logits + (E > 256 ? warp * E : 0), my_id, my_w);
  if (lane < k) {
    ids[t * k + lane] = my_id;
    wout[t * k + lane] = my_w;
  }
}

cudaError_t launch_route_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* w,
                              int* err, cudaStream_t s) {
  (void)err;
  if (T == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (T + warps - 1) / warps;
  const size_t smem = E > 256 ? (size_t)warps * E * sizeof(float) : 0;
  ProfScope ps(K_ROUTE, s);
  if (cudaError_t le_ = launch_pdl(route_topk_kernel, dim3((unsigned)blocks), dim3(warps * 32), smem, s, 1, logits, T, E, k, ids, w); le_ != cudaSuccess) return le_;
  return cudaGetLastError();
}

static int g_num_sms_cache = 0;
static int num_sms() {
  if (g_num_sms_cache == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms_cache, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms_cache <= 0) g_num_sms_cache = 148;
  }
  return g_num_sms_cache;
}

// ------------------------------------------------------------------ permute
// Counting sort in two launches.  Pairs are cut into chunks of consecutive pair
// indices, one block per chunk.  Scratch: hist [n_chunks][E], the expert totals tot
// (one per 128-byte line, so that the atomics of different experts do not queue on
// one line), arrive.
//   1. each block counts its chunk's pairs per expert into hist[c][e] and adds them
//      to tot[e] (integer atomics: the sums do not depend on their order); the
//      block that finishes last (an arrival counter decides which) scans tot into
//      counts and offsets;
//   2. block c starts expert e's run at offsets[e] + sum over c' < c of hist[c'][e],
//      then ranks its pairs: __match_any_sync groups the lanes of a warp by expert
//      (rank = earlier lanes of the group), a shared [warp][expert] table prefix-
//      summed over the warps orders the warps; positions are therefore stable
//      (ascending pair index inside every segment).
// moe_route_permute does routing and all of this in one cooperative launch
// (route_permute_kernel below): its routing warps fill the histogram, and one grid
// barrier separates that from the scan and the scatter.
// Replaces the per-expert mask lookup of the loop form ("What is
// torch._grouped_mm?", Unsloth faster-moe docs).
constexpr int kPermThreads = kPermuteChunk;
constexpr int kPermWarps = kPermThreads / 32;

// Run by every thread of the last block of a histogram launch (any block size that is
// a multiple of 32, at most 1024): counts and offsets from the expert totals.
// The expert totals tot[e * kTotStride] scanned into counts and offsets (written when
// write_out) by one block; on return s_tot[e] holds offsets[e] for every e < E.
__device__ void scan_totals(const int32_t* __restrict__ tot, int E, int64_t P,
                            int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                            int* s_tot, int* s_warp, bool write_out = true) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_tot[e] = __ldcg(tot + (int64_t)e * kTotStride);
  __syncthreads();
  // exclusive scan of the totals: each thread owns a run of `per` experts
  const int per = (E + (int)blockDim.x - 1) / (int)blockDim.x;
  const int e0 = threadIdx.x * per;
  int mine = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) mine += s_tot[e];
  int all;
  int run = block_exclusive_scan_1024(mine, s_warp, &all);
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int t = s_tot[e];
    s_tot[e] = run;                   // (each thread owns its run of entries)
    if (write_out) {
      counts[e] = t;
      offsets[e] = run;
    }
    run += t;
  }
  if (write_out && threadIdx.x == 0) offsets[E] = (int32_t)P;
  __syncthreads();
}

__global__ void __launch_bounds__(kPermThreads)
    permute_hist_kernel(const int32_t* __restrict__ ids, int64_t P, int E, int n_chunks,
                        int32_t* __restrict__ hist, int32_t* __restrict__ tot,
                        int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int* arrive,
                        int* err) {
  pdl_begin();
  __shared__ int s_hist[1024], s_warp[33], s_last;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int64_t p = (int64_t)blockIdx.x * kPermuteChunk + threadIdx.x;
  if (p < P) {
    const int e = ids[p];
    if (e >= 0 && e < E) atomicAdd(&s_hist[e], 1);
    else report_error(err, MOE_ERR_DEVICE_INDEX);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = s_hist[e];
    hist[(int64_t)blockIdx.x * E + e] = c;
    if (c != 0) atomicAdd(&tot[(int64_t)e * kTotStride], c);
  }
  // the block's writes are ordered before its arrival by the barrier and one fence
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(arrive, 1) == n_chunks - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  scan_totals(tot, E, P, counts, offsets, s_hist, s_warp);
  if (threadIdx.x == 0) *arrive = 0;                 // ready for the next call
}

// Chunk c of the counting sort's scatter (a block of kPermThreads threads): its base per
// expert from the offsets and the earlier chunks' counts, then the ranks of its pairs.
// The offsets come from global memory, or from shared memory when s_off is given.
// s_cnt holds (kPermWarps + 1) * E ints.
__device__ void scatter_chunk(const int32_t* __restrict__ ids, int64_t P, int E, int chunk_pairs,
                              int c, const int32_t* __restrict__ hist,
                              const int32_t* __restrict__ offsets, const int* s_off,
                              int32_t* __restrict__ sorted_pairs, int32_t* __restrict__ pair_pos,
                              int* s_cnt) {
  int* s_base = s_cnt + kPermWarps * E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();                    // the previous chunk's reads of s_cnt are done
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) s_cnt[i] = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    s_base[e] = s_off != nullptr ? s_off[e] : __ldcg(offsets + e);
  __syncthreads();
  // the chunk's base: G threads per expert each add every G-th earlier chunk's count,
  // eight independent loads at a time
  {
    const int G = E < kPermThreads ? kPermThreads / E : 1;
    for (int i = threadIdx.x; i < G * E; i += blockDim.x) {
      const int e = i % E, part = i / E;
      int sum = 0;
      for (int c0 = part; c0 < c; c0 += 8 * G) {
        int v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int cc = c0 + j * G;
          v[j] = cc < c ? __ldcg(hist + (int64_t)cc * E + e) : 0;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) sum += v[j];
      }
      if (sum != 0) atomicAdd(&s_base[e], sum);
    }
  }
  const int64_t p = (int64_t)c * chunk_pairs + threadIdx.x;
  const bool in = (int)threadIdx.x < chunk_pairs && p < P;
  int e = -1;
  if (in) e = __ldcg(ids + p);       // (written by other CTAs of the same launch)
  const bool ok = in && e >= 0 && e < E;
  const int key = ok ? e : -1 - lane;  // invalid lanes never group
  const unsigned grp = __match_any_sync(0xffffffffu, key);
  const int rank = __popc(grp & ((1u << lane) - 1u));
  if (ok && (31 - __clz(grp)) == lane) s_cnt[warp * E + e] = __popc(grp);
  __syncthreads();
  for (int ee = threadIdx.x; ee < E; ee += blockDim.x) {
    int run = s_base[ee];
    for (int w = 0; w < kPermWarps; ++w) {
      const int t = s_cnt[w * E + ee];
      s_cnt[w * E + ee] = run;
      run += t;
    }
  }
  __syncthreads();
  if (ok) {
    const int pos = s_cnt[warp * E + e] + rank;
    sorted_pairs[pos] = (int32_t)p;
    pair_pos[p] = pos;
  }
}

__global__ void __launch_bounds__(kPermThreads)
    permute_scatter_kernel(const int32_t* __restrict__ ids, int64_t P, int E, int chunk_pairs,
                           const int32_t* __restrict__ hist, const int32_t* __restrict__ offsets,
                           int32_t* __restrict__ sorted_pairs, int32_t* __restrict__ pair_pos) {
  pdl_begin();
  extern __shared__ int s_cnt[];   // [kPermWarps][E], then the chunk's base per expert [E]
  scatter_chunk(ids, P, E, chunk_pairs, blockIdx.x, hist, offsets, nullptr, sorted_pairs, pair_pos,
                s_cnt);
}

// Routing and the whole counting sort in one cooperative launch (all CTAs resident):
//   1. every warp routes tokens (warp_route) and adds its token's k pairs to the chunk
//      histogram hist[c][e] and the expert totals with integer atomics;
//   2. after a grid barrier, every CTA that has a chunk to scatter scans the totals into
//      its own copy of the offsets (CTA 0 also writes counts and offsets), then scatters
//      its chunks (scatter_chunk).
// hist, tot and the barrier counter after them are zero on entry.  The barrier's wait is
// bounded (MOE_ERR_TIMEOUT, then the CTA leaves).
__device__ __forceinline__ bool grid_barrier(int* ctr, int target, int* err, int* s_fail) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1);
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1; *reinterpret_cast<volatile int*>(ctr) < target; ++i) {
      if ((i & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
        report_error(err, MOE_ERR_TIMEOUT);
        *s_fail = 1;
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  return *s_fail == 0;
}

__global__ void __launch_bounds__(kPermThreads)
    route_permute_kernel(const float* __restrict__ logits, int64_t T, int E, int k, int tpc,
                         int n_chunks, int32_t* __restrict__ ids, float* __restrict__ wout,
                         int32_t* __restrict__ hist, int32_t* __restrict__ tot,
                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ sorted_pairs, int32_t* __restrict__ pair_pos,
                         int* bar, int* err) {
  pdl_begin();
  extern __shared__ int s_dyn[];    // routing: [kPermWarps][E] logits when E > 256;
                                    // scatter: (kPermWarps + 1) * E ints
  __shared__ int s_tot[1024], s_warp[33], s_fail;
  __shared__ int s_grp[2 * 1024];   // a group's pair counts in its (at most two) chunks
  if (threadIdx.x == 0) s_fail = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t P = T * k;
  // Groups of kPermWarps consecutive tokens, a warp per token.  A group spans at most two
  // chunks (tpc >= kPermWarps): its counts are summed in shared memory first, so a hot
  // expert costs one global atomic per group and chunk instead of one per pair, and the
  // expert totals one per CTA.
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_tot[e] = 0;
  const int64_t n_groups = (T + kPermWarps - 1) / kPermWarps;
  for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x) {
    for (int i = threadIdx.x; i < 2 * E; i += blockDim.x) s_grp[i] = 0;
    __syncthreads();
    const int64_t t0 = g * kPermWarps, t = t0 + warp, c0 = t0 / tpc;
    if (t < T) {
      int my_id;
      float my_w;
      warp_route(logits, t, E, k, lane, reinterpret_cast<float*>(s_dyn) + (E > 256 ? warp * E : 0),
                 my_id, my_w);
      if (lane < k) {
        ids[t * k + lane] = my_id;
        wout[t * k + lane] = my_w;
        atomicAdd(&s_grp[(int)(t / tpc - c0) * E + my_id], 1);
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 2 * E; i += blockDim.x) {
      const int cnt = s_grp[i];
      if (cnt != 0) {
        const int half = i >= E ? 1 : 0, e = i - half * E;
        atomicAdd(&hist[(c0 + half) * E + e], cnt);
        atomicAdd(&s_tot[e], cnt);
      }
    }
    __syncthreads();                // s_grp and the warps' logits rows are reused
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (s_tot[e] != 0) atomicAdd(&tot[(int64_t)e * kTotStride], s_tot[e]);
  if (!grid_barrier(bar, (int)gridDim.x, err, &s_fail)) return;
  if ((int)blockIdx.x >= n_chunks) return;
  scan_totals(tot, E, P, counts, offsets, s_tot, s_warp, blockIdx.x == 0);
  for (int c = blockIdx.x; c < n_chunks; c += gridDim.x)
    scatter_chunk(ids, P, E, tpc * k, c, hist, offsets, s_tot, sorted_pairs, pair_pos, s_dyn);
}

static cudaError_t launch_scatter(const int32_t* ids, int64_t P, int E, int n_chunks, int chunk_pairs,
                                  const int32_t* hist, const int32_t* offsets,
                                  int32_t* sorted_pairs, int32_t* pair_pos, cudaStream_t s) {
  const int smem = (kPermWarps + 1) * E * (int)sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t st = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (st != cudaSuccess) return st;
  }
  ProfScope ps(K_PERM_SCATTER, s);
  if (cudaError_t le_ = launch_pdl(permute_scatter_kernel, dim3(n_chunks), dim3(kPermThreads), smem, s, 1, ids,
                                   P, E, chunk_pairs, hist, offsets, sorted_pairs, pair_pos);
      le_ != cudaSuccess)
    return le_;
  return cudaGetLastError();
}

cudaError_t launch_permute(const int32_t* ids, int64_t P, int E, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_pairs, int32_t* pair_pos, int32_t* scratch, int* err,
                           cudaStream_t s) {
  const int n_chunks = (int)((P + kPermuteChunk - 1) / kPermuteChunk);
  if (n_chunks == 0) {
    // no pairs: zero counts, offsets all zero
    cudaError_t st = cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), s);
    if (st != cudaSuccess) return st;
    return cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s);
  }
  int32_t* hist = scratch;
  int32_t* tot = hist + (size_t)n_chunks * E;
  int* arrive = tot + (size_t)E * kTotStride;
  // every hist entry is written by its block; the totals and the counter start at zero
  cudaError_t st = cudaMemsetAsync(tot, 0, ((size_t)E * kTotStride + 1) * sizeof(int32_t), s);
  if (st != cudaSuccess) return st;
  {
    ProfScope ps(K_PERM_HIST, s);
    if (cudaError_t le_ = launch_pdl(permute_hist_kernel, dim3(n_chunks), dim3(kPermThreads), 0, s, 1,
                                     ids, P, E, n_chunks, hist, tot, counts, offsets, arrive, err);
        le_ != cudaSuccess)
      return le_;
    st = cudaGetLastError();
    if (st != cudaSuccess) return st;
  }
  return launch_scatter(ids, P, E, n_chunks, kPermuteChunk, hist, offsets, sorted_pairs, pair_pos, s);
}

int route_tokens_per_chunk(int k) { return kPermuteChunk / k; }

cudaError_t launch_route_permute(const float* logits, int64_t T, int E, int k, int32_t* ids,
                                 float* w, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                                 int32_t* pair_pos, int32_t* scratch, cudaStream_t s) {
  const int tpc = route_tokens_per_chunk(k);
  if (tpc < kPermWarps || E > 1024) return cudaErrorInvalidValue;   // (k <= 32 by the API)
  const int n_chunks = (int)((T + tpc - 1) / tpc);
  if (n_chunks == 0) {
    cudaError_t st = cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), s);
    if (st != cudaSuccess) return st;
    return cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s);
  }
  // the histograms, the totals and the barrier counter after them start at zero
  int32_t* hist = scratch;
  int32_t* tot = hist + (size_t)n_chunks * E;
  int* bar = tot + (size_t)E * kTotStride;
  int* err = moe_status_word();
  if (err == nullptr) return cudaErrorInvalidValue;
  cudaError_t st = cudaMemsetAsync(hist, 0, permute_scratch_ints(n_chunks, E) * sizeof(int32_t), s);
  if (st != cudaSuccess) return st;
  const int lsm = E > 256 ? kPermWarps * E * (int)sizeof(float) : 0;
  const int ssm = (kPermWarps + 1) * E * (int)sizeof(int);
  const int smem = lsm > ssm ? lsm : ssm;
  if (smem > 48 * 1024) {
    st = cudaFuncSetAttribute(route_permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (st != cudaSuccess) return st;
  }
  // every CTA must be resident at once (the grid barriers): at most the occupancy bound
  int per_sm = 0;
  st = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_permute_kernel, kPermThreads, smem);
  if (st != cudaSuccess) return st;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t want_route = (T + kPermWarps - 1) / kPermWarps;
  const int64_t want = want_route > n_chunks ? want_route : n_chunks;
  const int64_t cap = (int64_t)per_sm * num_sms();
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPermThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfScope ps(K_ROUTE, s);
  st = cudaLaunchKernelEx(&cfg, route_permute_kernel, logits, T, E, k, tpc, n_chunks, ids, w, hist, tot,
                          counts, offsets, sorted_pairs, pair_pos, bar, err);
  if (st != cudaSuccess) return st;
  return cudaGetLastError();
}

static unsigned grid_for(int64_t work, int threads) {
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms() * 16;
  return (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
}

// ------------------------------------------------------------------ permutation check
// Every invariant of the counting sort (debug mode): one thread per sorted position,
// plus the expert table checked by the first E + 1 threads.
__global__ void check_permutation_kernel(const int32_t* __restrict__ ids, int64_t P, int E,
                                         const int32_t* __restrict__ counts,
                                         const int32_t* __restrict__ offsets,
                                         const int32_t* __restrict__ sp,
                                         const int32_t* __restrict__ pos, int* err) {
  pdl_begin();
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  bool bad = false;
  if (i0 <= E) {
    const int e = (int)i0;
    if (e == 0 && offsets[0] != 0) bad = true;
    if (e == E && offsets[E] != (int32_t)P) bad = true;
    if (e < E && (offsets[e + 1] < offsets[e] || counts[e] != offsets[e + 1] - offsets[e])) bad = true;
  }
  for (int64_t q = i0; q < P; q += (int64_t)gridDim.x * blockDim.x) {
    const int32_t p = sp[q];
    if (p < 0 || p >= P) { bad = true; continue; }
    if (pos[p] != (int32_t)q) bad = true;
    const int e = ids[p];
    if (e < 0 || e >= E || q < offsets[e] || q >= offsets[e + 1]) { bad = true; continue; }
    if (q > offsets[e] && sp[q - 1] >= p) bad = true;      // stable: ascending pair index
  }
  if (bad) report_error(err, MOE_ERR_DEVICE_CHECK);
}

cudaError_t launch_check_permutation(const int32_t* ids, int64_t P, int E, const int32_t* counts,
                                     const int32_t* offsets, const int32_t* sorted_pairs,
                                     const int32_t* pair_pos, int* err, cudaStream_t s) {
  const int64_t work = P > E + 1 ? P : E + 1;
  if (cudaError_t le_ = launch_pdl(check_permutation_kernel, dim3(grid_for(work, 256)), dim3(256), 0, s,
                                   1, ids, P, E, counts, offsets, sorted_pairs, pair_pos, err);
      le_ != cudaSuccess)
    return le_;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ combine
// y[t, :] = sum_j w[t, j] ysorted[pair_pos[t k + j], :], fp32 over ascending j,
// one bf16 rounding; w == nullptr means every weight is 1.
__global__ void combine_kernel(const uint4* __restrict__ ys, const float* __restrict__ w,
                               const int32_t* __restrict__ pos, int64_t T, int k, int vpr,
                               uint4* __restrict__ y) {
  pdl_begin();
  const int64_t total = T * vpr;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / vpr;
    const int v = (int)(i - t * vpr);
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int64_t p = t * k + j;
      const float s = w != nullptr ? w[p] : 1.0f;
      const uint4 x = ys[(int64_t)pos[p] * vpr + v];
      acc[0] += s * bf16_lo(x.x); acc[1] += s * bf16_hi(x.x);
      acc[2] += s * bf16_lo(x.y); acc[3] += s * bf16_hi(x.y);
      acc[4] += s * bf16_lo(x.z); acc[5] += s * bf16_hi(x.z);
      acc[6] += s * bf16_lo(x.w); acc[7] += s * bf16_hi(x.w);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    y[i] = o;
  }
}

cudaError_t launch_combine(const uint16_t* ysorted, const float* w, const int32_t* pair_pos,
                           int64_t T, int k, int m, uint16_t* y, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int vpr = m / 8;
  ProfScope ps(K_COMBINE, s);
  if (cudaError_t le_ = launch_pdl(combine_kernel, dim3(grid_for(T * vpr, 256)), dim3(256), 0, s, 1, reinterpret_cast<const uint4*>(ysorted), w,
                                                        pair_pos, T, k, vpr,
                                                        reinterpret_cast<uint4*>(y)); le_ != cudaSuccess) return le_;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ router backward
// Beyond the path: the gradient into the router logits (for logits computed as
// x W_r inside a model; router equation of "Accelerating Mixture-of-Experts
// Fine-Tuning", section "The Dynamic Dispatch Bottleneck in Mixture-of-Experts
// Architectures").  A block of 8 warps owns TPB = max(1, 8 / k) whole tokens;
// each warp takes pairs (t, j) of the block in turn:
//   dw[t,j] = <dY[t], y_(t,j)>   (fp32 over 16-byte column pieces, y in sorted order;
//                                  the block's warps share dY[t] through L1)
// and one warp per token then writes the row
//   dlogits[t, ids[t,j]] = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i]),  0 for the others.
__device__ __forceinline__ float warp_allsum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__global__ void __launch_bounds__(256)
    router_backward_kernel(const uint4* __restrict__ dY, const uint4* __restrict__ ys,
                           const int32_t* __restrict__ ids, const float* __restrict__ w,
                           const int32_t* __restrict__ pos, int64_t T, int k, int E, int vpr,
                           float* __restrict__ dlogits) {
  pdl_begin();
  __shared__ float s_dw[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tpb = k >= 8 ? 1 : 8 / k;                 // tokens per block
  const int64_t t0 = (int64_t)blockIdx.x * tpb;
  const int npairs = (int)((t0 + tpb <= T ? tpb : T - t0) * k);
  for (int i = warp; i < npairs; i += 8) {
    const int64_t t = t0 + i / k;
    const int64_t q = pos[t0 * k + i];
    const uint4* a = dY + t * vpr;
    const uint4* b = ys + q * vpr;
    float acc = 0.f;
    for (int v = lane; v < vpr; v += 32) {
      const uint4 x = a[v], y = b[v];
      acc += bf16_lo(x.x) * bf16_lo(y.x) + bf16_hi(x.x) * bf16_hi(y.x) +
             bf16_lo(x.y) * bf16_lo(y.y) + bf16_hi(x.y) * bf16_hi(y.y) +
             bf16_lo(x.z) * bf16_lo(y.z) + bf16_hi(x.z) * bf16_hi(y.z) +
             bf16_lo(x.w) * bf16_lo(y.w) + bf16_hi(x.w) * bf16_hi(y.w);
    }
    acc = warp_allsum(acc);
    if (lane == 0) s_dw[i] = acc;
  }
  __syncthreads();
  const int ntok = npairs / k;
  if (warp < ntok) {
    const int64_t t = t0 + warp;
    const float my_dw = lane < k ? s_dw[warp * k + lane] : 0.f;
    const float my_w = lane < k ? w[t * k + lane] : 0.f;
    const float mean = warp_allsum(my_w * my_dw);
    for (int e = lane; e < E; e += 32) dlogits[t * E + e] = 0.f;
    __syncwarp();
    if (lane < k) dlogits[t * E + ids[t * k + lane]] = my_w * (my_dw - mean);
  }
}

cudaError_t launch_router_backward(const uint16_t* dY, const uint16_t* ys, const int32_t* ids,
                                   const float* w, const int32_t* pos, int64_t T, int k, int E,
                                   int m, float* dlogits, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int tpb = k >= 8 ? 1 : 8 / k;
  ProfScope ps(K_ROUTER_BWD, s);
  if (cudaError_t le_ = launch_pdl(router_backward_kernel, dim3((unsigned)((T + tpb - 1) / tpb)), dim3(256), 0, s, 1, 
      reinterpret_cast<const uint4*>(dY), reinterpret_cast<const uint4*>(ys), ids, w, pos, T, k, E,
      m / 8, dlogits); le_ != cudaSuccess) return le_;
  return cudaGetLastError();
}

cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t s) {
  if (bytes == 0) return cudaSuccess;
  ProfScope ps(K_MEMSET, s);
  return cudaMemsetAsync(p, 0, bytes, s);
}

}  // namespace moe
