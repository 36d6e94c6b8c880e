// decode_suffix.cu -- the cascade suffix-pass decode kernel instances (see launch.cuh).
#include "launch.cuh"

namespace pkv_host {

template <>
pa_status run_decode_mode<pkv::kSuffix, false>(bool bf16, int d, int bs, const pkv::DecodeArgs& a,
                                       const CUtensorMap& mk, const CUtensorMap& mv, int grid,
                                       cudaStream_t s) {
  if (bf16) return dispatch_d<__nv_bfloat16, pkv::kSuffix>(d, bs, a, mk, mv, grid, s);
  return dispatch_d<__half, pkv::kSuffix>(d, bs, a, mk, mv, grid, s);
}

}  // namespace pkv_host
