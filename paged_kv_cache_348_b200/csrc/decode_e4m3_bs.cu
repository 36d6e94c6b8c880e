// decode_e4m3_bs.cu -- the 8-bit (E4M3) pool decode kernel instances with per-(block, kv
// head) scales (see launch.cuh).
#include "launch.cuh"

namespace pkv_host {

pa_status run_e4m3_bs(bool bf16, int d, int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                      const CUtensorMap& mv, int grid, cudaStream_t s) {
  if (bf16) return dispatch_e4m3<__nv_bfloat16, true>(d, bs, a, mk, mv, grid, s);
  return dispatch_e4m3<__half, true>(d, bs, a, mk, mv, grid, s);
}

}  // namespace pkv_host
