// kv_ops.cuh -- cache append (slot scatter) and copy-on-write block copy for sm_100a.
// Both are pure byte movement: 16-byte vector loads/stores, consecutive threads on
// consecutive 16-byte chunks of a row so every warp access is coalesced.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "ptx.cuh"

namespace pkv {

constexpr int DEV_BAD_SLOT = 0x2;
constexpr int DEV_BAD_PAIR = 0x4;
constexpr int kMaxLayersPerLaunch = 128;

// "Paged Attention and Memory Efficiency in Production LLM Serving", section "How
// PagedAttention borrows OS paging": blocks are filled on demand as decoding proceeds.
// Token i with slot s >= 0 lands at block s / block_size, offset s % block_size.
__global__ void __launch_bounds__(256)
    pa_cache_append_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                           const uint4* __restrict__ k, const uint4* __restrict__ v,
                           const int64_t* __restrict__ slot_mapping, int num_tokens, int Hkv,
                           int chunks_per_row, int block_size, int num_blocks,
                           int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const long long total = (long long)num_tokens * Hkv * chunks_per_row;
  const long long limit = (long long)num_blocks * block_size;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(i % chunks_per_row);
    const long long rh = i / chunks_per_row;     // (token, kv head)
    const int h = (int)(rh % Hkv);
    const long long tok = rh / Hkv;
    const long long slot = slot_mapping[tok];
    if (slot < 0) continue;                      // padding token
    if (slot >= limit) {
      if (status && ch == 0) atomicOr(status, DEV_BAD_SLOT);
      continue;
    }
    const long long b = slot / block_size, off = slot % block_size;
    const long long dst = ((b * Hkv + h) * block_size + off) * chunks_per_row + ch;
    k_cache[dst] = k[i];
    v_cache[dst] = v[i];
  }
}

// First step of the block-scaled 8-bit append: every token whose slot is offset 0 of its
// block fixes that block's (K and V) scales for each kv head from its own rows.  One warp
// per (token, kv head); 16-bit input rows of D values.
template <typename T>
__global__ void __launch_bounds__(256)
    pa_e4m3_block_scale_kernel(float* __restrict__ k_bscale, float* __restrict__ v_bscale,
                               const T* __restrict__ k, const T* __restrict__ v,
                               const int64_t* __restrict__ slot_mapping, int num_tokens, int Hkv,
                               int D, int block_size, int num_blocks) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  if (w >= (long long)num_tokens * Hkv) return;
  const int h = (int)(w % Hkv);
  const long long tok = w / Hkv;
  const long long slot = slot_mapping[tok];
  if (slot < 0 || slot >= (long long)num_blocks * block_size || slot % block_size) return;
  const long long b = slot / block_size;
  float ak = 0.f, av = 0.f;
  for (int d = lane; d < D; d += 32) {
    const long long i = (tok * Hkv + h) * D + d;
    ak = fmaxf(ak, fabsf((float)k[i]));
    av = fmaxf(av, fabsf((float)v[i]));
  }
  ak = warp_max_f32(ak);
  av = warp_max_f32(av);
  if (lane == 0) {
    k_bscale[b * Hkv + h] = e4m3_block_scale(ak);
    v_bscale[b * Hkv + h] = e4m3_block_scale(av);
  }
}

// The append into 8-bit E4M3 caches: as pa_cache_append_kernel, each value quantised as
// x / scale (binary32, IEEE division) rounded to E4M3, with one scale per pool (k_scale,
// v_scale) or, when k_bscale is not null, the scale of the destination (block, kv head)
// (set beforehand for blocks whose offset 0 is written in the same call).  One thread per
// 16 values: two 16-byte loads of 16-bit input, one 16-byte store of codes.
template <typename T>
__global__ void __launch_bounds__(256)
    pa_cache_append_e4m3_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                const uint4* __restrict__ k, const uint4* __restrict__ v,
                                const int64_t* __restrict__ slot_mapping, int num_tokens,
                                int Hkv, int chunks_per_row, int block_size, int num_blocks,
                                float k_scale, float v_scale, const float* __restrict__ k_bscale,
                                const float* __restrict__ v_bscale, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const long long total = (long long)num_tokens * Hkv * chunks_per_row;
  const long long limit = (long long)num_blocks * block_size;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(i % chunks_per_row);    // 16 values
    const long long rh = i / chunks_per_row;
    const int h = (int)(rh % Hkv);
    const long long tok = rh / Hkv;
    const long long slot = slot_mapping[tok];
    if (slot < 0) continue;
    if (slot >= limit) {
      if (status && ch == 0) atomicOr(status, DEV_BAD_SLOT);
      continue;
    }
    const long long b = slot / block_size, off = slot % block_size;
    const long long dst = ((b * Hkv + h) * block_size + off) * chunks_per_row + ch;
    for (int kv = 0; kv < 2; ++kv) {
      const uint4* src = (kv ? v : k) + 2 * i;
      const float sc = k_bscale ? (kv ? v_bscale : k_bscale)[b * Hkv + h] : (kv ? v_scale : k_scale);
      const uint4 in[2] = {src[0], src[1]};
      const uint32_t* w = reinterpret_cast<const uint32_t*>(in);
      uint32_t q[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float f[4];
        for (int u = 0; u < 2; ++u) {
          uint32_t x = w[2 * e + u];
          float lo, hi;
          if constexpr (std::is_same_v<T, __nv_bfloat16>) {
            lo = __uint_as_float(x << 16);
            hi = __uint_as_float(x & 0xffff0000u);
          } else {
            const __half2 hx = *reinterpret_cast<const __half2*>(&x);
            const float2 fx = __half22float2(hx);
            lo = fx.x, hi = fx.y;
          }
          f[2 * u] = __fdiv_rn(lo, sc);
          f[2 * u + 1] = __fdiv_rn(hi, sc);
        }
        q[e] = f32x2_to_e4m3x2(f[0], f[1]) | (f32x2_to_e4m3x2(f[2], f[3]) << 16);
      }
      (kv ? v_cache : k_cache)[dst] = make_uint4(q[0], q[1], q[2], q[3]);
    }
  }
}

struct LayerPtrs {
  uint4* k[kMaxLayersPerLaunch];
  uint4* v[kMaxLayersPerLaunch];
};

// "Paged Attention and Memory Efficiency in Production LLM Serving", section "How
// PagedAttention borrows OS paging": a sequence that diverges from a shared prefix gets
// a new block (copy-on-write).  grid = (pairs, layers * 2 pools).
__global__ void __launch_bounds__(256)
    pa_copy_blocks_kernel(const __grid_constant__ LayerPtrs P, const int32_t* __restrict__ pairs,
                          int num_blocks, long long chunks_per_block, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  const int layer = blockIdx.y >> 1, pool = blockIdx.y & 1;
  const int src = pairs[2 * p], dst = pairs[2 * p + 1];
  if ((unsigned)src >= (unsigned)num_blocks || (unsigned)dst >= (unsigned)num_blocks) {
    if (status && threadIdx.x == 0) atomicOr(status, DEV_BAD_PAIR);
    return;
  }
  uint4* base = pool ? P.v[layer] : P.k[layer];
  const uint4* s = base + (long long)src * chunks_per_block;
  uint4* d = base + (long long)dst * chunks_per_block;
  for (long long i = threadIdx.x; i < chunks_per_block; i += blockDim.x) d[i] = s[i];
}

// Preemption ("Paged Attention and Memory Efficiency in Production LLM Serving", section
// "Why KV cache memory was the bottleneck": requests are preempted when the cache runs
// out): the blocks of a preempted sequence are saved to a buffer the device can reach
// (page-locked host memory) and later restored into fresh blocks.  Buffer layout:
// [layer][pool: K, V][i][block], blocks[i] naming the pool block of entry i.
// grid = (n, layers * 2 pools); layer0 = the first layer of this launch's pointers.
template <bool kOut>
__global__ void __launch_bounds__(256)
    pa_swap_blocks_kernel(const __grid_constant__ LayerPtrs P, const int32_t* __restrict__ blocks,
                          int n, int num_blocks, long long chunks_per_block, int layer0,
                          uint4* buf, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  const int layer = blockIdx.y >> 1, pool = blockIdx.y & 1;
  const int b = blocks[i];
  if ((unsigned)b >= (unsigned)num_blocks) {
    if (status && threadIdx.x == 0) atomicOr(status, DEV_BAD_PAIR);
    return;
  }
  uint4* dev = (pool ? P.v[layer] : P.k[layer]) + (long long)b * chunks_per_block;
  uint4* h = buf + (((long long)(layer0 + layer) * 2 + pool) * n + i) * chunks_per_block;
  for (long long j = threadIdx.x; j < chunks_per_block; j += blockDim.x) {
    if constexpr (kOut) h[j] = dev[j];
    else dev[j] = h[j];
  }
}

}  // namespace pkv
