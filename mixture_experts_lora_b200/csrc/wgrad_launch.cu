// Host launchers of the adapter-gradient kernel (lora_wgrad.cuh) and of the
// expert-weight-gradient kernel of full fine-tuning (expert_dw.cuh).
#include "expert_dw.cuh"
#include "lora_wgrad.cuh"
#include "tmap.cuh"

namespace moe {

namespace {

template <int RP, bool V>
cudaError_t wgrad_rp(const GemmShape& g, const CUtensorMap* tm, const WgradParams& wp,
                     int max_chunks, cudaStream_t s) {
  using C = WgradCfg<RP, V>;
  auto kern = lora_wgrad_kernel<RP, V>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  int dtiles = wp.pr[0].n_dtiles + (wp.n_problems > 1 ? wp.pr[1].n_dtiles : 0);
  const int64_t units = (int64_t)max_chunks * dtiles;
  // at least one CTA per SM: the zero fill of experts without rows runs in every CTA
  const int grid = (int)(units > 0 && units < g.num_sms ? units : g.num_sms);
  ProfScope ps(K_WGRAD, s);
  st = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, 1, tm[0], tm[1], tm[2], tm[3], wp);
  if (st != cudaSuccess) return st;
  return cudaGetLastError();
}

template <bool V>
cudaError_t wgrad_dispatch(const GemmShape& g, const CUtensorMap* tm, const WgradParams& wp,
                           int max_chunks, cudaStream_t s) {
  switch (g.rp) {
    case 16: return wgrad_rp<16, V>(g, tm, wp, max_chunks, s);
    case 32: return wgrad_rp<32, V>(g, tm, wp, max_chunks, s);
    case 64: return wgrad_rp<64, V>(g, tm, wp, max_chunks, s);
    case 128: return wgrad_rp<128, V>(g, tm, wp, max_chunks, s);
  }
  return cudaErrorInvalidValue;
}

template <class C>
cudaError_t expert_dw_launch(int kind, const CUtensorMap* tm, const DwParams& p, int num_sms,
                             cudaStream_t s) {
  auto kern = moe_dw_kernel<C>;
  cudaError_t st = ensure_smem(kern, C::SMEM_BYTES);
  if (st != cudaSuccess) return st;
  const int64_t total = (int64_t)p.E * p.n_mt * p.n_nt;
  const int grid = (int)(total < num_sms ? total : num_sms);
  ProfScope ps(kind, s);
  st = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, 1, tm[0], tm[1], tm[2], p);
  if (st != cudaSuccess) return st;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_lora_wgrad(const GemmShape& g, const WgradJob* jobs, int n_jobs,
                              const TileInfo* chunks, const int* n_chunks, int max_chunks,
                              const int32_t* chunk_start, cudaStream_t s) {
  if (n_jobs < 1 || n_jobs > 2) return cudaErrorInvalidValue;
  using C0 = WgradCfg<16>;
  CUtensorMap tm[4];      // Big of each problem, then Small of each problem
  WgradParams wp{};
  const uint64_t P = (uint64_t)(g.P > 0 ? g.P : 1);
  bool v = true;
  for (int j = 0; j < n_jobs; ++j) v = v && jobs[j].D % 64 == 0;
  for (int j = 0; j < n_jobs; ++j) {
    const WgradJob& jb = jobs[j];
    const uint64_t ls = (uint64_t)jb.ld_small;
    // Small [P, ld_small] seen as [ld_small / 8 groups][P rows][8 columns]: a box of
    // BK rows x rp / 8 groups lands group-major, groups past ld_small reading as zero
    const uint64_t sd[3] = {8, P, ls / 8};
    const uint64_t ss[2] = {ls * 2, 16};
    const uint32_t sb[3] = {8, (uint32_t)C0::BK, (uint32_t)g.rp / 8};
    if (!encode(&tm[2 + j], jb.small, 3, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    // Big [P, D] sorted: BK rows x 256 columns per stage (four 64-column atoms)
    const bool okb = v ? encode_atoms(&tm[j], jb.big, false, 1, P, (uint64_t)jb.D, C0::BK, C0::BN / 64)
                       : encode2d(&tm[j], jb.big, P, (uint64_t)jb.D, (uint64_t)jb.D, C0::BK, 64);
    if (!okb) return cudaErrorInvalidValue;
    WgradProblem& q = wp.pr[j];
    q.small = reinterpret_cast<const __nv_bfloat16*>(jb.small);
    q.ld_small = jb.ld_small;
    q.r_small = jb.ld_small;
    q.D = jb.D;
    q.n_dtiles = (jb.D + C0::BN - 1) / C0::BN;
    q.transpose = jb.transpose;
    q.out = reinterpret_cast<__nv_bfloat16*>(jb.out);
    q.partial = jb.partial;
    q.counters = jb.counters;
  }
  if (n_jobs == 1) {
    tm[1] = tm[0];
    tm[3] = tm[2];
  }
  wp.n_problems = n_jobs;
  wp.chunks = chunks;
  wp.n_chunks = n_chunks;
  wp.chunk_start = chunk_start;
  wp.E = g.E;
  wp.r = g.r;
  wp.scale = g.scale;
  wp.err = g.err;
  return v ? wgrad_dispatch<true>(g, tm, wp, max_chunks, s) : wgrad_dispatch<false>(g, tm, wp, max_chunks, s);
}

cudaError_t launch_expert_dw(int kind, const GemmShape& g, const int32_t* offsets, const uint16_t* Lm,
                             int Mdim, const uint16_t* Rm, int Ndim, uint16_t* out, cudaStream_t s) {
  using C = DwCfg<true>;
  CUtensorMap tm[3];
  const uint64_t P = (uint64_t)g.P;
  const bool v = Mdim % 64 == 0 && Ndim % 64 == 0;
  const bool ok = v ? encode_atoms(&tm[0], Lm, false, 1, P, (uint64_t)Mdim, C::BK, 2) &&
                          encode_atoms(&tm[1], Rm, false, 1, P, (uint64_t)Ndim, C::BK, 4)
                    : encode2d(&tm[0], Lm, P, (uint64_t)Mdim, (uint64_t)Mdim, C::BK, 64) &&
                          encode2d(&tm[1], Rm, P, (uint64_t)Ndim, (uint64_t)Ndim, C::BK, 64);
  // output [E, Mdim, Ndim] in 32 x 32 blocks, 64-byte swizzle (the staging layout)
  const uint64_t odims[3] = {(uint64_t)Ndim, (uint64_t)Mdim, (uint64_t)g.E};
  const uint64_t ostr[2] = {(uint64_t)Ndim * 2, (uint64_t)Mdim * Ndim * 2};
  const uint32_t obox[3] = {32, 32, 1};
  if (!ok || !encode(&tm[2], out, 3, odims, ostr, obox, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  DwParams p{};
  p.offsets = offsets;
  p.E = g.E;
  p.Mdim = Mdim;
  p.Ndim = Ndim;
  p.n_mt = (Mdim + C::BM - 1) / C::BM;
  p.n_nt = (Ndim + C::BN - 1) / C::BN;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.err = g.err;
  return v ? expert_dw_launch<DwCfg<true>>(kind, tm, p, g.num_sms, s)
           : expert_dw_launch<DwCfg<false>>(kind, tm, p, g.num_sms, s);
}

}  // namespace moe
