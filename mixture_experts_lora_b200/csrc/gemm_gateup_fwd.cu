// gate_up projection, forward: GU = Xs W_gu + (c XA) B_gu over each expert's token
// chunks (Xs the expert-ordered X rows), with the SwiGLU in the epilogue
// (H = silu(g) u); writes GU and H.
#include "gemm_host.cuh"

namespace moe {

cudaError_t launch_gemm_gateup_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* Xs,
                                   const uint16_t* XAc, uint16_t* GU, uint16_t* H, cudaStream_t s) {
  GemmMaps mp;
  const uint64_t E = g.E, m = g.m, n = g.n, P = g.P;
  // W_gu [E, m, 2n] as [E][gate | up][n / 64 atoms][m rows][64]: one copy brings the
  // CTA's 64 gate columns and the 64 up columns of the same indices (MN-major A)
  const bool v = g.n % 64 == 0 && g.m % 64 == 0;
  bool ok;
  if (v) {
    const uint64_t dims[5] = {64, m, n / 64, 2, E};
    const uint64_t str[4] = {2 * n * 2, 128, n * 2, m * 2 * n * 2};
    const uint32_t box[5] = {64, 128, 1, 2, 1};
    ok = encode(&mp.m[0], w.W_gu, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_atoms(&mp.m[1], Xs, false, 1, P, m, 128, 2);
  } else {
    ok = encode3d(&mp.m[0], w.W_gu, E, m, 2 * n, 128, 64) && encode2d(&mp.m[1], Xs, P, m, m, 128, 64);
  }
  ok = ok && encode_lora(mp, g, true, w.B_gu, 2 * g.n, XAc) &&
       encode_out(&mp.m[4], GU, g, n, 2 * n) && encode_out(&mp.m[5], GU + n, g, n, 2 * n) &&
       encode_out(&mp.m[6], H, g, n, n);
  ok = ok && encode_act_boxes(mp, Xs, P, m, v);
  if (!ok) return cudaErrorInvalidValue;
  GemmParams p{};
  p.chunks = g.gchunks;
  p.n_chunks = g.n_gchunks;
  p.F = g.n;
  p.n_ftiles = (g.n + 127) / 128;
  p.nk = (g.m + 127) / 128;
  p.n = g.n;
  p.out = reinterpret_cast<__nv_bfloat16*>(GU);
  p.out_h = reinterpret_cast<__nv_bfloat16*>(H);
  p.err = g.err;
  return dispatch_gemm<true, EPI_SWIGLU>(K_GEMM_GATEUP_FWD, g, v, mp, p, s);
}

}  // namespace moe
