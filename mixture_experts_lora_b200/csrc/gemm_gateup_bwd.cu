// gate_up projection, backward: dX_sorted = dGU W_gu^T + (c T2) A_gu^T over each
// expert's token chunks (dGU sorted rows through TMA).
#include "gemm_host.cuh"

namespace moe {

cudaError_t launch_gemm_gateup_bwd(const GemmShape& g, const LayerPtrs& w, const uint16_t* dGU,
                                   const uint16_t* T2c, uint16_t* dXp, cudaStream_t s) {
  GemmMaps mp;
  const uint64_t E = g.E, m = g.m, n = g.n, P = g.P;
  const bool v = (2 * g.n) % 64 == 0;
  bool ok = v ? encode_atoms(&mp.m[0], w.W_gu, true, E, m, 2 * n, 128, 2) &&
                    encode_atoms(&mp.m[1], dGU, false, 1, P, 2 * n, 128, 2)
              : encode3d(&mp.m[0], w.W_gu, E, m, 2 * n, 128, 64) &&
                    encode2d(&mp.m[1], dGU, P, 2 * n, 2 * n, 128, 64);
  ok = ok && encode_lora(mp, g, false, w.A_gu, g.m, T2c) && encode_out(&mp.m[4], dXp, g, m, m);
  ok = ok && encode_act_boxes(mp, dGU, P, 2 * n, v);
  if (!ok) return cudaErrorInvalidValue;
  mp.m[5] = mp.m[4];
  mp.m[6] = mp.m[4];
  GemmParams p{};
  p.chunks = g.gchunks;
  p.n_chunks = g.n_gchunks;
  p.F = g.m;
  p.n_ftiles = (g.m + 255) / 256;
  p.nk = (2 * g.n + 127) / 128;
  p.n = g.n;
  p.out = reinterpret_cast<__nv_bfloat16*>(dXp);
  p.err = g.err;
  return dispatch_gemm<false, EPI_PLAIN>(K_GEMM_GATEUP_BWD, g, v, mp, p, s);
}

}  // namespace moe
