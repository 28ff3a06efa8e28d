// Device-side helpers shared by the kernels: status word, bf16 packing, and thin
// inline-PTX wrappers for mbarriers, TMA bulk-tensor copies and tcgen05
// (tensor-memory allocation, UMMA issue/commit, TMEM loads) on sm_100a.
//
// Every wait on an mbarrier is bounded by a wall-clock limit read from
// %globaltimer; a wait that expires reports MOE_ERR_TIMEOUT through the status
// word and returns false so that the caller can leave its loop.  No kernel here
// traps or spins without a limit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moelora.h"

namespace moe {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait

__device__ __forceinline__ void report_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- bf16 packing
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// tanh by the hardware approximation (PTX tanh.approx.f32, one special-function
// op, relative error about 2^-11).  The SwiGLU kernels take the logistic sigmoid
// through s(x) = (1 + tanh(x / 2)) / 2: one such op per element instead of an
// exponential and a reciprocal, whose special-function work was part of what bound
// their worker warps.  The error stays well below the bf16 rounding of the outputs.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) {
  return __uint_as_float(v << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t v) {
  return __uint_as_float(v & 0xffff0000u);
}
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

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete, giving up after
// limit_ns nanoseconds of %globaltimer (MOE_ERR_TIMEOUT in the status word).
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, int* err,
                                              uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 0 && globaltimer_ns() - t0 > limit_ns) {
      report_error(err, MOE_ERR_TIMEOUT);
      return false;
    }
  }
}
// The kernels' wait: the same with the library's 1 s limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* err) {
  return mbar_wait_for(bar, parity, err, kWaitLimitNs);
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* m, uint32_t bar, uint32_t dst,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(const CUtensorMap* m, uint32_t bar, uint32_t dst,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ---------------------------------------------------------------- cp.async
// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N committed groups of this thread are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- tcgen05
// Shared-memory matrix descriptor (sm_100 format): start address, leading and
// stride byte offsets (all >> 4), version 1 at bit 46, layout type at bits 61-63
// (0 none, 2 = 128B swizzle, 4 = 64B swizzle, 6 = 32B swizzle).
enum : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 inputs and fp32 accumulation.
// a_mn / b_mn: operand stored MN-major (1) or K-major (0).
__host__ __device__ __forceinline__ uint32_t idesc_bf16(uint32_t M, uint32_t N, uint32_t a_mn,
                                                        uint32_t b_mn) {
  return (1u << 4)            // D format fp32
         | (1u << 7)          // A bf16
         | (1u << 10)         // B bf16
         | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]; one thread issues.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 lanes x 32 consecutive fp32 columns; thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

// ---------------------------------------------------------------- clusters / 2-SM MMA
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_smem(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA load into this CTA's shared memory that completes on an mbarrier of either
// CTA of the pair (here: the pair's leader).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* m, uint32_t bar_cluster,
                                                 uint32_t dst, int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(const CUtensorMap* m, uint32_t bar_cluster,
                                                 uint32_t dst, int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(const CUtensorMap* m, uint32_t bar_cluster,
                                                 uint32_t dst, int32_t c0, int32_t c1, int32_t c2,
                                                 int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d_pair(const CUtensorMap* m, uint32_t bar_cluster,
                                                 uint32_t dst, int32_t c0, int32_t c1, int32_t c2,
                                                 int32_t c3, int32_t c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (256 rows over the pair) (+)= A (128 rows per CTA) * B (N/2 rows per CTA); leader issues.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the mbarrier at this offset in every CTA of `cta_mask` once the pair's
// previously issued tcgen05 ops complete.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}

// ---------------------------------------------------------------- TMA stores
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int32_t c0,
                                             int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, uint32_t src, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- dependent launch
// Every kernel of the library is launched with programmatic stream serialization: it
// may be scheduled while its predecessor in the stream drains (its prologue - barrier
// set-up, TMEM allocation, descriptor prefetch - overlaps that tail).  pdl_wait()
// blocks until the predecessors have completed and their writes are visible; each
// kernel calls it before its first global-memory access, read or write, and then
// lets its own dependents be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_begin() {
  pdl_wait();
  pdl_launch_dependents();
}

// ---------------------------------------------------------------- misc
// ---------------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void named_bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
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

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// One entry per row tile of a grouped GEMM: rows [row0, row_end) of expert e.
struct TileInfo {
  int e;
  int row0;
  int row_end;
  int pad;
};

// ---------------------------------------------------------------- block scan
// Exclusive scan of one value per thread (int or 64-bit) over a block of up to 1024
// threads; *total_out receives the block total.  s_warp holds 33 values.
template <class T>
__device__ __forceinline__ T block_exclusive_scan_1024(T v, T* s_warp, T* total_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const T u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  __syncthreads();
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const T w = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : T(0);
    T inc2 = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const T u = __shfl_up_sync(0xffffffffu, inc2, off);
      if (lane >= off) inc2 += u;
    }
    s_warp[lane] = inc2 - w;
    if (lane == 31) s_warp[32] = inc2;
  }
  __syncthreads();
  *total_out = s_warp[32];
  return incl - v + s_warp[warp];
}

// ---------------------------------------------------------------- layer tables
// The tables of one layer call, derived from the permutation's offsets:
//   tiles    128-row tiles that never straddle two experts (rank-r kernels): every
//            expert's full tiles in expert order, then the short last tiles in four
//            size classes from the largest to the smallest (expert order inside a
//            class), so that a launch of one CTA per tile, dispatched in tile order,
//            gives the smallest tiles to the CTAs that share an SM with two others;
//   gchunks  token chunks of the grouped GEMMs: ceil(cnt / gchunk_rows) chunks per
//            expert of equal size rounded up to 16 rows;
//   chunks   row chunks of chunk_rows rows for the adapter gradients, with
//            chunk_start[e] the first chunk of expert e (optional);
//   zero     arrival counters set to zero (optional).
struct TableBuild {
  const int32_t* offsets;   // [E + 1]; nullptr: the tables are built already
  int E;
  int tile_rows;
  TileInfo* tiles;
  int* n_tiles;
  int gchunk_rows;
  TileInfo* gchunks;
  int* n_gchunks;
  int chunk_rows;
  TileInfo* chunks;         // nullptr: no gradient chunks
  int* n_chunks;
  int32_t* chunk_start;     // [E + 1]
  int* zero;
  int n_zero;
};

// Run by every thread of every CTA of the first kernel of a call (a grid of at least
// E CTAs): each CTA finds its own tile b among the tiles and writes it, CTA e writes
// expert e's token and gradient chunks, CTA 0 the counts, and each CTA a slice of the
// zeroed counters.  Returns the number of tiles; *my receives tile b (unchanged when
// b is past the last tile).
static __device__ int build_tables_cta(const TableBuild& tb, int b, int nb, TileInfo* my, int* s_warp,
                                unsigned long long* s_warp64, TileInfo* s_tile) {
  const int E = tb.E, R = tb.tile_rows;
  const int per = (E + (int)blockDim.x - 1) / (int)blockDim.x;
  const int e0 = threadIdx.x * per, e1 = min(E, e0 + per);
  int my_full = 0, my_ng = 0, my_nc = 0;
  unsigned long long my_cls = 0;
  for (int e = e0; e < e1; ++e) {
    const int cnt = tb.offsets[e + 1] - tb.offsets[e];
    const int rag = cnt % R;
    my_full += cnt / R;
    if (rag > 0) my_cls += 1ull << (16 * (3 - (rag * 4) / R));
    my_ng += (cnt + tb.gchunk_rows - 1) / tb.gchunk_rows;
    if (tb.chunks != nullptr) my_nc += (cnt + tb.chunk_rows - 1) / tb.chunk_rows;
  }
  int total_full, gtotal, ctotal = 0;
  unsigned long long ctot;
  int f = block_exclusive_scan_1024(my_full, s_warp, &total_full);
  unsigned long long cr = block_exclusive_scan_1024(my_cls, s_warp64, &ctot);
  int g = block_exclusive_scan_1024(my_ng, s_warp, &gtotal);
  int cc = tb.chunks != nullptr ? block_exclusive_scan_1024(my_nc, s_warp, &ctotal) : 0;
  int cbase[4];
  int n_tiles = total_full;
  for (int c = 0; c < 4; ++c) {
    cbase[c] = n_tiles;
    n_tiles += (int)((ctot >> (16 * c)) & 0xffffu);
  }
  if (threadIdx.x == 0) s_tile->e = -1;
  __syncthreads();
  for (int e = e0; e < e1; ++e) {
    const int lo = tb.offsets[e], hi = tb.offsets[e + 1], cnt = hi - lo;
    const int nf = cnt / R, rag = cnt - nf * R;
    if (b >= f && b < f + nf) *s_tile = TileInfo{e, lo + (b - f) * R, lo + (b - f + 1) * R, 0};
    f += nf;
    if (rag > 0) {
      const int c = 3 - (rag * 4) / R;
      if (cbase[c] + (int)((cr >> (16 * c)) & 0xffffu) == b) *s_tile = TileInfo{e, lo + nf * R, hi, 0};
      cr += 1ull << (16 * c);
    }
    const int ng = (cnt + tb.gchunk_rows - 1) / tb.gchunk_rows;
    if (e == b) {
      const int sz = ng > 0 ? (((cnt + ng - 1) / ng + 15) & ~15) : 0;
      for (int i = 0; i < ng; ++i)
        tb.gchunks[g + i] = TileInfo{e, lo + i * sz, min(hi, lo + (i + 1) * sz), 0};
    }
    g += ng;
    if (tb.chunks != nullptr) {
      const int nc = (cnt + tb.chunk_rows - 1) / tb.chunk_rows;
      if (e == b) {
        for (int i = 0; i < nc; ++i)
          tb.chunks[cc + i] = TileInfo{e, lo + i * tb.chunk_rows, min(hi, lo + (i + 1) * tb.chunk_rows), 0};
        tb.chunk_start[e] = cc;
      }
      cc += nc;
    }
  }
  if (b == 0 && threadIdx.x == 0) {
    *tb.n_tiles = n_tiles;
    *tb.n_gchunks = gtotal;
    if (tb.chunks != nullptr) {
      *tb.n_chunks = ctotal;
      tb.chunk_start[E] = ctotal;
    }
  }
  if (tb.n_zero > 0) {
    const int zper = (tb.n_zero + nb - 1) / nb;
    for (int i = b * zper + (int)threadIdx.x; i < min(tb.n_zero, (b + 1) * zper); i += blockDim.x)
      tb.zero[i] = 0;
  }
  __syncthreads();
  if (s_tile->e >= 0) {
    *my = *s_tile;
    if (threadIdx.x == 0) tb.tiles[b] = *s_tile;
  }
  return n_tiles;
}

}  // namespace moe
