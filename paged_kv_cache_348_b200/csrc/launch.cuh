// launch.cuh -- host-side launch helpers and the template dispatch from runtime shape
// arguments (dtype, head_dim, block_size, query columns) to a decode kernel instance.
// The instances are spread over several translation units (decode_*.cu), one per kernel
// mode, so that they compile in parallel; api.cu reaches them through run_decode_mode.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>

#include "decode.cuh"
#include "decode_wide.cuh"
#include "pagedkv.h"

namespace pkv_host {

// Programmatic dependent launch lets a kernel's launch and prologue overlap the tail of
// the kernel before it in the stream (PAGEDKV_NO_PDL=1 turns it off).
inline bool use_pdl() {
  static const bool on = [] {
    const char* v = std::getenv("PAGEDKV_NO_PDL");
    return !(v && v[0] && v[0] != '0');
  }();
  return on;
}

template <typename Kernel, typename... Args>
cudaError_t launch(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                   Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = use_pdl() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename T, int D, int BS, int NT, int MODE, bool KV8 = false, bool KSC = false>
pa_status launch_decode(const pkv::DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv,
                        int grid, cudaStream_t stream) {
  using L = pkv::Layout<D, KV8, pkv::ctas_per_sm(KV8, NT, BS), MODE == pkv::kAppend, KSC, BS == 1>;
  auto split = pkv::pa_decode_split_kernel<T, D, BS, NT, MODE, KV8, KSC>;
  if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynSmem) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  if (launch(split, dim3(grid), dim3(pkv::kThreads), L::kDynSmem, stream, a, mk, mv) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D, int BS, int MODE>
pa_status dispatch_nt(const pkv::DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv,
                      int grid, cudaStream_t s) {
  return a.ncol <= 8 ? launch_decode<T, D, BS, 1, MODE>(a, mk, mv, grid, s)
                     : launch_decode<T, D, BS, 2, MODE>(a, mk, mv, grid, s);
}

template <typename T, int D, int MODE>
pa_status dispatch_bs(int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                      const CUtensorMap& mv, int grid, cudaStream_t s) {
  switch (bs) {
    case 1: return dispatch_nt<T, D, 1, MODE>(a, mk, mv, grid, s);
    case 8: return dispatch_nt<T, D, 8, MODE>(a, mk, mv, grid, s);
    case 16: return dispatch_nt<T, D, 16, MODE>(a, mk, mv, grid, s);
    case 32: return dispatch_nt<T, D, 32, MODE>(a, mk, mv, grid, s);
  }
  return PA_ERR_UNSUPPORTED;
}

template <typename T, int MODE>
pa_status dispatch_d(int d, int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                     const CUtensorMap& mv, int grid, cudaStream_t s) {
  return d == 64 ? dispatch_bs<T, 64, MODE>(bs, a, mk, mv, grid, s)
                 : dispatch_bs<T, 128, MODE>(bs, a, mk, mv, grid, s);
}

// 8-bit (E4M3) caches, head_dim 128 or 64: plain decode (one or several new tokens) with
// one scale per pool or, KSC, per-(block, kv head) scales; the cascade passes and the fused
// append with per-(block, kv head) scales.
template <typename T, int D, bool KSC, int MODE>
pa_status dispatch_e4m3_d(int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                          const CUtensorMap& mv, int grid, cudaStream_t s) {
  const bool nt1 = a.ncol <= 8;
  switch (bs) {
    case 1: return nt1 ? launch_decode<T, D, 1, 1, MODE, true, KSC>(a, mk, mv, grid, s)
                       : launch_decode<T, D, 1, 2, MODE, true, KSC>(a, mk, mv, grid, s);
    case 8: return nt1 ? launch_decode<T, D, 8, 1, MODE, true, KSC>(a, mk, mv, grid, s)
                       : launch_decode<T, D, 8, 2, MODE, true, KSC>(a, mk, mv, grid, s);
    case 16: return nt1 ? launch_decode<T, D, 16, 1, MODE, true, KSC>(a, mk, mv, grid, s)
                        : launch_decode<T, D, 16, 2, MODE, true, KSC>(a, mk, mv, grid, s);
    case 32: return nt1 ? launch_decode<T, D, 32, 1, MODE, true, KSC>(a, mk, mv, grid, s)
                        : launch_decode<T, D, 32, 2, MODE, true, KSC>(a, mk, mv, grid, s);
  }
  return PA_ERR_UNSUPPORTED;
}
template <typename T, bool KSC = false, int MODE = pkv::kPlain>
pa_status dispatch_e4m3(int d, int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                        const CUtensorMap& mv, int grid, cudaStream_t s) {
  return d == 64 ? dispatch_e4m3_d<T, 64, KSC, MODE>(bs, a, mk, mv, grid, s)
                 : dispatch_e4m3_d<T, 128, KSC, MODE>(bs, a, mk, mv, grid, s);
}

// The block-scaled 8-bit plain-decode instances; defined in decode_e4m3_bs.cu.
pa_status run_e4m3_bs(bool bf16, int d, int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                      const CUtensorMap& mv, int grid, cudaStream_t s);

// One kernel mode's instances, dispatched on the other parameters; defined in
// decode_<mode>.cu.  kv8: 8-bit E4M3 pools (decode_e4m3*.cu; every mode but kPlain needs
// per-(block, kv head) scales).
template <int MODE, bool KV8>
pa_status run_decode_mode(bool bf16, int d, int bs, const pkv::DecodeArgs& a,
                          const CUtensorMap& mk, const CUtensorMap& mv, int grid, cudaStream_t s);
#define PKV_DECL_RUN(MODE, KV8)                                                              \
  template <>                                                                                \
  pa_status run_decode_mode<MODE, KV8>(bool bf16, int d, int bs, const pkv::DecodeArgs& a,   \
                                       const CUtensorMap& mk, const CUtensorMap& mv, int grid, \
                                       cudaStream_t s);
PKV_DECL_RUN(pkv::kPlain, false)
PKV_DECL_RUN(pkv::kPrefix, false)
PKV_DECL_RUN(pkv::kSuffix, false)
PKV_DECL_RUN(pkv::kAppend, false)
PKV_DECL_RUN(pkv::kPlain, true)
PKV_DECL_RUN(pkv::kPrefix, true)
PKV_DECL_RUN(pkv::kSuffix, true)
PKV_DECL_RUN(pkv::kAppend, true)
#undef PKV_DECL_RUN

// ---- the tcgen05 kernel for 9..64 query rows per kv head (decode_wide.cuh); NC = the
// query rows rounded up to 16, 32 or 64
template <typename T, int D, int BS, int MODE, int NC>
pa_status launch_wide(const pkv::DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv,
                      int grid, cudaStream_t stream) {
  using L = pkv::WideLayout<D>;
  auto k = pkv::pa_decode_wide_kernel<T, D, BS, MODE, NC>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynSmem) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  if (launch(k, dim3(grid), dim3(pkv::wide_threads(NC)), L::kDynSmem, stream, a, mk, mv) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int MODE, int NC>
pa_status dispatch_wide(int d, int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                        const CUtensorMap& mv, int grid, cudaStream_t s) {
  if (d == 64) {
    switch (bs) {
      case 1: return launch_wide<T, 64, 1, MODE, NC>(a, mk, mv, grid, s);
      case 8: return launch_wide<T, 64, 8, MODE, NC>(a, mk, mv, grid, s);
      case 16: return launch_wide<T, 64, 16, MODE, NC>(a, mk, mv, grid, s);
      case 32: return launch_wide<T, 64, 32, MODE, NC>(a, mk, mv, grid, s);
    }
  } else {
    switch (bs) {
      case 1: return launch_wide<T, 128, 1, MODE, NC>(a, mk, mv, grid, s);
      case 8: return launch_wide<T, 128, 8, MODE, NC>(a, mk, mv, grid, s);
      case 16: return launch_wide<T, 128, 16, MODE, NC>(a, mk, mv, grid, s);
      case 32: return launch_wide<T, 128, 32, MODE, NC>(a, mk, mv, grid, s);
    }
  }
  return PA_ERR_UNSUPPORTED;
}

// One (mode, NC)'s wide instances; defined in decode_wide_<mode>_<NC>.cu.
template <int MODE, int NC>
pa_status run_wide_mode(bool bf16, int d, int bs, const pkv::DecodeArgs& a, const CUtensorMap& mk,
                        const CUtensorMap& mv, int grid, cudaStream_t s);
#define PKV_DECL_WIDE(MODE, NC)                                                               \
  template <>                                                                                 \
  pa_status run_wide_mode<MODE, NC>(bool bf16, int d, int bs, const pkv::DecodeArgs& a,       \
                                    const CUtensorMap& mk, const CUtensorMap& mv, int grid,   \
                                    cudaStream_t s);
PKV_DECL_WIDE(pkv::kPlain, 16)
PKV_DECL_WIDE(pkv::kPlain, 32)
PKV_DECL_WIDE(pkv::kPlain, 64)
PKV_DECL_WIDE(pkv::kPrefix, 16)
PKV_DECL_WIDE(pkv::kPrefix, 32)
PKV_DECL_WIDE(pkv::kPrefix, 64)
PKV_DECL_WIDE(pkv::kAppend, 16)
PKV_DECL_WIDE(pkv::kAppend, 32)
PKV_DECL_WIDE(pkv::kAppend, 64)
#undef PKV_DECL_WIDE

}  // namespace pkv_host
