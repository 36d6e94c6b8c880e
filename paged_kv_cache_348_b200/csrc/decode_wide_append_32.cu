// decode_wide_append_32.cu -- the tcgen05 decode kernel instances of mode kAppend with 32 query
// columns (see launch.cuh).
#include "launch.cuh"

namespace pkv_host {

template <>
pa_status run_wide_mode<pkv::kAppend, 32>(bool bf16, int d, int bs, const pkv::DecodeArgs& a,
                                  const CUtensorMap& mk, const CUtensorMap& mv, int grid,
                                  cudaStream_t s) {
  if (bf16) return dispatch_wide<__nv_bfloat16, pkv::kAppend, 32>(d, bs, a, mk, mv, grid, s);
  return dispatch_wide<__half, pkv::kAppend, 32>(d, bs, a, mk, mv, grid, s);
}

}  // namespace pkv_host
