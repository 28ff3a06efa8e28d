// down projection, backward, with the SwiGLU backward fused:
//   dH  = w (dY W_d^T + (c T1') A_d^T),  T1' = dY B_d^T   (dY rows gathered, no
//         expert-ordered copy of w dY; the routing weight w applied in the epilogue)
//   dGU = [dH u s (1 + g (1 - s)), dH g s],  s = sigmoid(g), [g | u] = GU
// writes dGU; dH never reaches memory.
#include "gemm_host.cuh"

namespace moe {

cudaError_t launch_gemm_down_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dY,
                                 const int32_t* sorted_pairs, int k, const float* topk_w,
                                 const uint16_t* GU, const uint16_t* T1c, uint16_t* dGU,
                                 cudaStream_t s) {
  GemmMaps mp;
  const uint64_t E = g.E, m = g.m, n = g.n;
  const bool v = g.m % 64 == 0;
  bool ok = v ? encode_atoms(&mp.m[0], w.W_d, true, E, n, m, 128, 2)
              : encode3d(&mp.m[0], w.W_d, E, n, m, 128, 64);
  ok = ok && encode_lora(mp, g, false, w.A_d, g.n, T1c) &&
       encode_out(&mp.m[4], dGU, g, n, 2 * n) && encode_out(&mp.m[5], dGU + n, g, n, 2 * n);
  if (!ok) return cudaErrorInvalidValue;
  mp.m[1] = mp.m[0];   // token operand gathered, no map
  mp.m[6] = mp.m[4];
  GemmParams p{};
  p.chunks = g.gchunks;
  p.n_chunks = g.n_gchunks;
  p.F = g.n;
  p.n_ftiles = (g.n + 255) / 256;
  p.nk = (g.m + 127) / 128;
  p.K = g.m;
  p.gsrc = reinterpret_cast<const __nv_bfloat16*>(dY);
  p.sorted_pairs = sorted_pairs;
  p.k = k;
  p.w = topk_w;
  p.gu = reinterpret_cast<const __nv_bfloat16*>(GU);
  p.n = g.n;
  p.out = reinterpret_cast<__nv_bfloat16*>(dGU);
  p.err = g.err;
  return dispatch_gemm<false, true, EPI_DSWIGLU>(K_GEMM_DOWN_BWD, g, v, mp, p, s);
}

}  // namespace moe
