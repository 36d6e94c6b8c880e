// decode_e4m3.cu -- the 8-bit (E4M3) pool decode kernel instances (see launch.cuh).
#include "launch.cuh"

namespace pkv_host {

template <>
pa_status run_decode_mode<pkv::kPlain, true>(bool bf16, int d, int bs, const pkv::DecodeArgs& a,
                                       const CUtensorMap& mk, const CUtensorMap& mv, int grid,
                                       cudaStream_t s) {
  if (a.k_bscale) return run_e4m3_bs(bf16, d, bs, a, mk, mv, grid, s);
  if (bf16) return dispatch_e4m3<__nv_bfloat16>(d, bs, a, mk, mv, grid, s);
  return dispatch_e4m3<__half>(d, bs, a, mk, mv, grid, s);
}

}  // namespace pkv_host
