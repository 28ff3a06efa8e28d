// down projection, forward: Y_sorted = H W_d + (c HA) B_d over each expert's token
// chunks (H sorted rows through TMA).
#include "gemm_host.cuh"

namespace moe {

cudaError_t launch_gemm_down_fwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* H,
                                 const uint16_t* HAc, uint16_t* Yp, cudaStream_t s) {
  GemmMaps mp;
  const uint64_t E = g.E, m = g.m, n = g.n, P = g.P;
  const bool v = g.n % 64 == 0 && g.m % 64 == 0;
  bool ok = v ? encode_atoms(&mp.m[0], w.W_d, true, E, n, m, 128, 2) &&
                    encode_atoms(&mp.m[1], H, false, 1, P, n, 128, 2)
              : encode3d(&mp.m[0], w.W_d, E, n, m, 128, 64) && encode2d(&mp.m[1], H, P, n, n, 128, 64);
  ok = ok && encode_lora(mp, g, true, w.B_d, g.m, HAc) && encode_out(&mp.m[4], Yp, g, m, m);
  ok = ok && encode_act_boxes(mp, H, P, n, v);
  if (!ok) return cudaErrorInvalidValue;
  mp.m[5] = mp.m[4];
  mp.m[6] = mp.m[4];
  GemmParams p{};
  p.chunks = g.gchunks;
  p.n_chunks = g.n_gchunks;
  p.F = g.m;
  p.n_ftiles = (g.m + 255) / 256;
  p.nk = (g.n + 127) / 128;
  p.n = g.n;
  p.out = reinterpret_cast<__nv_bfloat16*>(Yp);
  p.err = g.err;
  return dispatch_gemm<true, EPI_PLAIN>(K_GEMM_DOWN_FWD, g, v, mp, p, s);
}

}  // namespace moe
