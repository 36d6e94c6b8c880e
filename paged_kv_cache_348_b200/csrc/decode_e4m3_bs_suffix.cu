// decode_e4m3_bs_suffix.cu -- the suffix mode's 8-bit (E4M3) pool instances, per-(block, kv
// head) scales (see launch.cuh).
#include "launch.cuh"

namespace pkv_host {

template <>
pa_status run_decode_mode<pkv::kSuffix, true>(bool bf16, int d, int bs, const pkv::DecodeArgs& a,
                                          const CUtensorMap& mk, const CUtensorMap& mv,
                                          int grid, cudaStream_t s) {
  if (!a.k_bscale || !a.v_bscale) return PA_ERR_UNSUPPORTED;
  if (bf16) return dispatch_e4m3<__nv_bfloat16, true, pkv::kSuffix>(d, bs, a, mk, mv, grid, s);
  return dispatch_e4m3<__half, true, pkv::kSuffix>(d, bs, a, mk, mv, grid, s);
}

}  // namespace pkv_host
