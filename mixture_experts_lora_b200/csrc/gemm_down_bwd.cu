// down projection, backward: dH = dy W_d^T + (c T1) A_d^T over each expert's token
// chunks (dy the expert-ordered w dY rows, T1 = dy B_d^T).
#include "gemm_host.cuh"

namespace moe {

cudaError_t launch_gemm_down_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dys,
                                 const uint16_t* T1c, uint16_t* dH, cudaStream_t s) {
  GemmMaps mp;
  const uint64_t E = g.E, m = g.m, n = g.n, P = g.P;
  const bool v = g.m % 64 == 0;
  bool ok = v ? encode_atoms(&mp.m[0], w.W_d, true, E, n, m, 128, 2) &&
                    encode_atoms(&mp.m[1], dys, false, 1, P, m, 128, 2)
              : encode3d(&mp.m[0], w.W_d, E, n, m, 128, 64) && encode2d(&mp.m[1], dys, P, m, m, 128, 64);
  ok = ok && encode_lora(mp, g, false, w.A_d, g.n, T1c) && encode_out(&mp.m[4], dH, g, n, n);
  ok = ok && encode_act_boxes(mp, dys, P, m, v);
  if (!ok) return cudaErrorInvalidValue;
  mp.m[5] = mp.m[4];
  mp.m[6] = mp.m[4];
  GemmParams p{};
  p.chunks = g.gchunks;
  p.n_chunks = g.n_gchunks;
  p.F = g.n;
  p.n_ftiles = (g.n + 255) / 256;
  p.nk = (g.m + 127) / 128;
  p.n = g.n;
  p.out = reinterpret_cast<__nv_bfloat16*>(dH);
  p.err = g.err;
  return dispatch_gemm<false, EPI_PLAIN>(K_GEMM_DOWN_BWD, g, v, mp, p, s);
}

}  // namespace moe
