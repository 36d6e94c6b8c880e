// api.cu -- the extern "C" entry points of libpagedkv (declared in include/pagedkv.h):
// argument validation, workspace layout, TMA descriptor encoding, template dispatch
// and kernel launches.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "decode.cuh"
#include "kv_ops.cuh"
#include "launch.cuh"
#include "pagedkv.h"
#include "wait_check.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

struct WsLayout {
  size_t counters_off, acc_off, ml_off, total;
};

// arrival counters: uint64[G]; partial accumulators: float[G*2][rows][D]; partial (max,
// sum): float[G*2][rows][2], rows = query columns a kernel's partial holds (16 for the
// mma.sync kernel, 64 for the tcgen05 one).  The batch size does not change the size.
constexpr WsLayout ws_layout(int head_dim, int grid, int rows) {
  WsLayout w{};
  size_t off = align256(sizeof(unsigned long long) * (size_t)grid);
  w.acc_off = off;
  off = align256(off + sizeof(float) * (size_t)grid * 2 * rows * head_dim);
  w.ml_off = off;
  off = align256(off + sizeof(float) * (size_t)grid * 2 * rows * 2);
  w.total = off;
  return w;
}

// The workspace pa_decode and its variants take covers either kernel: the mma.sync one at
// up to 3 CTAs per SM with 16 query columns, the tcgen05 one at one CTA per SM with 64.
size_t split_workspace_bytes(int head_dim, int sms) {
  const size_t a = ws_layout(head_dim, sms * pkv::kMaxCtasPerSm, pkv::kMaxGroup).total;
  const size_t b = ws_layout(head_dim, sms, pkv::kWideCols).total;
  return a > b ? a : b;
}

// Query columns per kv head from which the tcgen05 kernel takes a launch (plain and prefix
// modes): 9, since at 16 columns it was measured faster than the mma.sync kernel's two
// n-tiles (70B shape with 2 new tokens 0.105 vs 0.107 ms, 8B shape with 4: 0.078 vs
// 0.084 ms).  PAGEDKV_WIDE_MIN_COLS=n overrides it, for comparing the two kernels.
int wide_min_cols() {
  static const int v = [] {
    const char* e = std::getenv("PAGEDKV_WIDE_MIN_COLS");
    const int x = e ? std::atoi(e) : 0;
    return (x >= 1 && x <= pkv::kWideCols + 1) ? x : 9;
  }();
  return v;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D view of one pool: rows = num_blocks*kv_heads*block_size, each head_dim elements;
// box = 64 dims x box_rows rows, 128-byte swizzle, out-of-range rows read as zero.
// kv8: an 8-bit (E4M3) pool, rows of head_dim bytes, box = head_dim x box_rows, with the
// 128-byte swizzle at head_dim 128 and the 64-byte one at head_dim 64 (one row a line).
bool encode_pool(CUtensorMap* map, const void* base, pa_dtype dtype, int head_dim,
                 uint64_t rows, int box_rows, bool kv8 = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim * (kv8 ? 1 : 2)};
  cuuint32_t box[2] = {kv8 ? (cuuint32_t)head_dim : 64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, kv8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                            : dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   (kv8 && head_dim == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The tcgen05 kernel's 4-D view of a 16-bit pool: (64 dims, 8 rows, column halves, 8-row
// groups) with byte strides (row D*2, half 128, group 8*D*2); a box of box_groups groups
// lands in shared memory as [group][half][8 rows][128 bytes], 128-byte swizzle.  rows must
// be a multiple of 8 (block_size >= 8).
bool encode_pool_wide(CUtensorMap* map, const void* base, pa_dtype dtype, int head_dim,
                      uint64_t rows, int box_groups) {
  auto enc = tensor_map_encoder();
  if (!enc || rows % 8) return false;
  const int halves = head_dim / 64;
  cuuint64_t dims[4] = {64u, 8u, (cuuint64_t)halves, (cuuint64_t)(rows / 8)};
  cuuint64_t strides[3] = {(cuuint64_t)head_dim * 2, 128u, (cuuint64_t)head_dim * 2 * 8};
  cuuint32_t box[4] = {64u, 8u, (cuuint32_t)halves, (cuuint32_t)box_groups};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Every call gets its own epoch so arrival counters left by earlier calls (or by an
// aborted one) read as zero; 0 is skipped so a zeroed workspace also reads as zero.
uint32_t next_epoch() {
  static std::atomic<uint32_t> epoch{0};
  uint32_t e = ++epoch;
  if (e == 0) e = ++epoch;
  return e;
}

// Kernel mode -> its translation unit's dispatcher.
pa_status dispatch_mode(bool kv8, bool wide, int mode, bool bf16, int d, int bs,
                        const pkv::DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv,
                        int grid, cudaStream_t s) {
  using namespace pkv_host;
  if (wide) {
    const int nc = a.ncol <= 16 ? 16 : (a.ncol <= 32 ? 32 : 64);
    if (mode == pkv::kPrefix)
      return nc == 16 ? run_wide_mode<pkv::kPrefix, 16>(bf16, d, bs, a, mk, mv, grid, s)
             : nc == 32 ? run_wide_mode<pkv::kPrefix, 32>(bf16, d, bs, a, mk, mv, grid, s)
                        : run_wide_mode<pkv::kPrefix, 64>(bf16, d, bs, a, mk, mv, grid, s);
    if (mode == pkv::kAppend)
      return nc == 16 ? run_wide_mode<pkv::kAppend, 16>(bf16, d, bs, a, mk, mv, grid, s)
             : nc == 32 ? run_wide_mode<pkv::kAppend, 32>(bf16, d, bs, a, mk, mv, grid, s)
                        : run_wide_mode<pkv::kAppend, 64>(bf16, d, bs, a, mk, mv, grid, s);
    return nc == 16 ? run_wide_mode<pkv::kPlain, 16>(bf16, d, bs, a, mk, mv, grid, s)
           : nc == 32 ? run_wide_mode<pkv::kPlain, 32>(bf16, d, bs, a, mk, mv, grid, s)
                      : run_wide_mode<pkv::kPlain, 64>(bf16, d, bs, a, mk, mv, grid, s);
  }
  if (kv8) {
    switch (mode) {
      case pkv::kPlain: return run_decode_mode<pkv::kPlain, true>(bf16, d, bs, a, mk, mv, grid, s);
      case pkv::kPrefix: return run_decode_mode<pkv::kPrefix, true>(bf16, d, bs, a, mk, mv, grid, s);
      case pkv::kSuffix: return run_decode_mode<pkv::kSuffix, true>(bf16, d, bs, a, mk, mv, grid, s);
      case pkv::kAppend: return run_decode_mode<pkv::kAppend, true>(bf16, d, bs, a, mk, mv, grid, s);
    }
    return PA_ERR_INVALID;
  }
  switch (mode) {
    case pkv::kPlain: return run_decode_mode<pkv::kPlain, false>(bf16, d, bs, a, mk, mv, grid, s);
    case pkv::kPrefix: return run_decode_mode<pkv::kPrefix, false>(bf16, d, bs, a, mk, mv, grid, s);
    case pkv::kSuffix: return run_decode_mode<pkv::kSuffix, false>(bf16, d, bs, a, mk, mv, grid, s);
    case pkv::kAppend: return run_decode_mode<pkv::kAppend, false>(bf16, d, bs, a, mk, mv, grid, s);
  }
  return PA_ERR_INVALID;
}

// Cascade extras of one launch (kPlain: all null).
struct CascadeArgs {
  int mode = pkv::kPlain;
  const int32_t* seq_start = nullptr;
  const int32_t* chunk_members = nullptr;
  int q_rows = 0;
  float2* ext_ml = nullptr;
  float* ext_acc = nullptr;
  const void* k_new = nullptr;   // kAppend
  const void* v_new = nullptr;
  int late_wait = 0;             // kSuffix: wait for the prefix pass only where it is needed
  bool kv8 = false;              // 8-bit E4M3 caches with these scales
  float k_scale = 1.f, v_scale = 1.f;
  const float* k_bscale = nullptr;   // 8-bit caches: per-(block, kv head) scales instead
  const float* v_bscale = nullptr;
  int max_grid = 0;              // > 0: at most this many CTAs (one per segment)
};

// Validation, workspace layout, tensor maps and launch shared by the decode entry points.
// grid_cap > 0 caps the number of split CTAs (the fixed scratch of pa_decode_noalloc).
pa_status decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                      int q_len, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                      pa_dtype dtype, void* workspace, size_t workspace_bytes, int grid_cap,
                      int32_t* dev_status, void* stream, const CascadeArgs& cx = CascadeArgs()) {
  if (num_seqs < 0 || q_len < 1 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      max_blocks_per_seq <= 0 || num_blocks <= 0 || !std::isfinite(scale))
    return PA_ERR_INVALID;
  if (num_q_heads % num_kv_heads) return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 1 && block_size != 8 && block_size != 16 && block_size != 32)
    return PA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  const long long ncol = (long long)group * q_len;
  // query columns per kv head: up to 16 on the mma.sync kernel (every mode), up to 64 on
  // the tcgen05 kernel (16-bit pools: plain, prefix and fused-append modes)
  const bool wide_mode = !cx.kv8 && (cx.mode == pkv::kPlain || cx.mode == pkv::kPrefix ||
                                     cx.mode == pkv::kAppend);
  if (ncol > (wide_mode ? pkv::kWideCols : pkv::kMaxGroup)) return PA_ERR_UNSUPPORTED;
  const bool wide = wide_mode && ncol >= wide_min_cols();
  if ((long long)num_blocks * num_kv_heads * block_size >= (1ll << 31) ||
      (long long)max_blocks_per_seq * block_size >= (1ll << 31) ||
      (long long)num_seqs * num_kv_heads >= (1ll << 31))
    return PA_ERR_INVALID;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(workspace))
    return PA_ERR_INVALID;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  int grid = wide ? sms : sms * pkv::ctas_per_sm(cx.kv8, ncol <= 8 ? 1 : 2, block_size);
  // a cap counts mma.sync CTAs (up to kMaxCtasPerSm a SM); the tcgen05 kernel runs one a SM
  const int cap = grid_cap > 0 ? (wide ? grid_cap / pkv::kMaxCtasPerSm : grid_cap) : 0;
  if (cap > 0 && grid > cap) grid = cap;
  if (cx.max_grid > 0 && grid > cx.max_grid) grid = cx.max_grid;
  const WsLayout w = ws_layout(head_dim, grid, wide ? pkv::kWideCols : pkv::kMaxGroup);
  if (workspace_bytes < w.total) return PA_ERR_INVALID;

  CUtensorMap mk, mv;
  std::memset(&mk, 0, sizeof(mk));
  std::memset(&mv, 0, sizeof(mv));
  // 8-bit pools: the cascade and fused-append modes need per-block scales
  if (cx.kv8 && cx.mode != pkv::kPlain && !cx.k_bscale) return PA_ERR_UNSUPPORTED;
  if (block_size == 1) {
    // both kernels gather block_size-1 rows four at a time: one-row boxes
    const uint64_t rows = (uint64_t)num_blocks * num_kv_heads;
    if (!encode_pool(&mk, k_cache, dtype, head_dim, rows, 1, cx.kv8) ||
        !encode_pool(&mv, v_cache, dtype, head_dim, rows, 1, cx.kv8))
      return PA_ERR_CUDA;
  }
  if (block_size != 1) {
    const uint64_t rows = (uint64_t)num_blocks * num_kv_heads * block_size;
    const int box_rows = block_size < 16 ? block_size : 16;
    if (wide) {
      if (!encode_pool_wide(&mk, k_cache, dtype, head_dim, rows, box_rows / 8) ||
          !encode_pool_wide(&mv, v_cache, dtype, head_dim, rows, box_rows / 8))
        return PA_ERR_CUDA;
    } else if (!encode_pool(&mk, k_cache, dtype, head_dim, rows, box_rows, cx.kv8) ||
               !encode_pool(&mv, v_cache, dtype, head_dim, rows, box_rows, cx.kv8)) {
      return PA_ERR_CUDA;
    }
  }
  pkv::DecodeArgs a{};
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.counters = reinterpret_cast<unsigned long long*>(ws + w.counters_off);
  a.part_acc = reinterpret_cast<float*>(ws + w.acc_off);
  a.part_ml = reinterpret_cast<float*>(ws + w.ml_off);
  a.status = dev_status;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.ctx_cap = max_blocks_per_seq * block_size;
  a.q_len = q_len;
  a.ncol = group * q_len;
  a.scale_log2 = scale * cx.k_scale * 1.4426950408889634f;
  a.v_scale = cx.v_scale;
  a.epoch = next_epoch();
  a.seq_start = cx.seq_start;
  a.chunk_members = cx.chunk_members;
  a.q_rows = cx.q_rows;
  a.ext_ml = cx.ext_ml;
  a.ext_acc = cx.ext_acc;
  a.k_new = cx.k_new;
  a.v_new = cx.v_new;
  a.late_wait = cx.late_wait;
  a.k_bscale = cx.k_bscale;
  a.v_bscale = cx.v_bscale;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dispatch_mode(cx.kv8, wide, cx.mode, dtype == PA_BF16, head_dim, block_size, a, mk, mv,
                       grid, st);
}

// Cascade workspace: two split scratches (the two passes may run at the same time), then
// the external partials (max, sum)[B][Hq] and acc[B][Hq][D] that carry the prefix pass's
// result to the suffix pass.
struct CascadeLayout {
  size_t split, split2_off, ml_off, acc_off, total;
};
CascadeLayout cascade_layout(int num_seqs, int num_q_heads, int head_dim, int sms) {
  CascadeLayout c{};
  c.split = split_workspace_bytes(head_dim, sms);
  c.split2_off = align256(c.split);
  c.ml_off = align256(c.split2_off + c.split);
  c.acc_off = align256(c.ml_off + sizeof(float2) * (size_t)num_seqs * num_q_heads);
  c.total = align256(c.acc_off + sizeof(float) * (size_t)num_seqs * num_q_heads * head_dim);
  return c;
}

// The two cascade passes over one pool pair; cx carries the pool's element format (8-bit
// scales), the rest is filled in here.
pa_status cascade_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, const int32_t* context_lens,
                       const int32_t* prefix_lens, int num_seqs, const int32_t* chunk_members,
                       int chunk_width, const int32_t* chunk_prefix_lens, int num_chunks,
                       int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int num_blocks, float scale, pa_dtype dtype,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status,
                       void* stream, CascadeArgs cx) {
  if (num_seqs < 0 || num_chunks < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      num_q_heads % num_kv_heads || (num_chunks && chunk_width < 1))
    return PA_ERR_INVALID;
  if (num_seqs == 0) return PA_OK;
  if (!prefix_lens || (num_chunks && (!chunk_members || !chunk_prefix_lens)) || !workspace ||
      !aligned16(workspace))
    return PA_ERR_INVALID;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  const CascadeLayout cl = cascade_layout(num_seqs, num_q_heads, head_dim, sms);
  if (workspace_bytes < cl.total) return PA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int group = num_q_heads / num_kv_heads;
  // the prefix pass puts a chunk's members' query rows side by side (up to 64 columns on
  // 16-bit pools, 16 on 8-bit ones); the suffix pass decodes one new token per sequence
  // (up to 16)
  const int prefix_cols = cx.kv8 ? pkv::kMaxGroup : pkv::kWideCols;
  if (group > pkv::kMaxGroup || (num_chunks && (long long)group * chunk_width > prefix_cols))
    return PA_ERR_UNSUPPORTED;
  // pass 1 writes each chunk's prefix partial for its members (the external partials);
  // pass 2 decodes every sequence's own tokens and merges that partial.  Pass 2 uses a
  // split scratch of its own and reads the partials only when it merges, so it waits for
  // pass 1 there (and at its end) rather than at its start, and overlaps pass 1's end.
  cx.ext_ml = reinterpret_cast<float2*>(ws + cl.ml_off);
  cx.ext_acc = reinterpret_cast<float*>(ws + cl.acc_off);
  if (num_chunks > 0) {
    // pass 1: each chunk's shared prefix once, its members' query rows as MMA columns
    cx.mode = pkv::kPrefix;
    cx.chunk_members = chunk_members;
    cx.q_rows = num_seqs;
    // no more CTAs than (chunk, kv head) segments: the weighted split still balances the
    // CTAs, but segments of equal length are no longer split (no partials, arrivals or
    // merges), and the SMs left over start the suffix pass at once
    cx.max_grid = (int)std::min<long long>((long long)num_chunks * num_kv_heads, 1 << 30);
    const pa_status r = decode_impl(out, q, k_cache, v_cache, block_tables, chunk_prefix_lens,
                                    num_chunks, chunk_width, num_q_heads, num_kv_heads,
                                    head_dim, block_size, max_blocks_per_seq, num_blocks, scale,
                                    dtype, workspace, cl.split, 0, dev_status, stream, cx);
    if (r != PA_OK) return r;
  }
  // pass 2: every sequence's own tokens, merged with its prefix partial
  cx.mode = pkv::kSuffix;
  cx.max_grid = 0;
  cx.chunk_members = nullptr;
  cx.seq_start = prefix_lens;
  cx.late_wait = num_chunks > 0 ? 1 : 0;      // its previous grid is then pass 1
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, ws + cl.split2_off, cl.split, 0, dev_status,
                     stream, cx);
}


}  // namespace

extern "C" {

int pa_version(void) { return 100; }

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_NO_BLOCKS: return "not enough free blocks";
    case PA_ERR_NO_MEMORY: return "out of host memory";
  }
  return "unknown status";
}

size_t pa_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0) return 0;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  return split_workspace_bytes(head_dim, sms);
}

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int max_blocks_per_seq, int num_blocks, float scale, pa_dtype dtype,
                    void* workspace, size_t workspace_bytes, int32_t* dev_status,
                    void* stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, workspace, workspace_bytes, 0, dev_status,
                     stream);
}

pa_status pa_decode_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                          int q_len, int num_q_heads, int num_kv_heads, int head_dim,
                          int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                          pa_dtype dtype, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, void* stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, q_len,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, workspace, workspace_bytes, 0, dev_status,
                     stream);
}

pa_status pa_decode_append(void* out, const void* q, void* k_cache, void* v_cache,
                           const void* k_new, const void* v_new, const int32_t* block_tables,
                           const int32_t* context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                           int num_blocks, float scale, pa_dtype dtype, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (num_seqs > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)))
    return PA_ERR_INVALID;
  CascadeArgs cx;
  cx.mode = pkv::kAppend;
  cx.k_new = k_new;
  cx.v_new = v_new;
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, workspace, workspace_bytes, 0, dev_status, stream,
                     cx);
}

pa_status pa_decode_e4m3(void* out, const void* q, const void* k_cache, const void* v_cache,
                         float k_scale, float v_scale, const int32_t* block_tables,
                         const int32_t* context_lens, int num_seqs, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                         int num_blocks, float scale, pa_dtype dtype, void* workspace,
                         size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) ||
      !(v_scale > 0.f))
    return PA_ERR_INVALID;
  CascadeArgs cx;
  cx.kv8 = true;
  cx.k_scale = k_scale;
  cx.v_scale = v_scale;
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, workspace, workspace_bytes, 0, dev_status, stream,
                     cx);
}

pa_status pa_cache_append_e4m3(void* k_cache, void* v_cache, const void* k, const void* v,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               float k_scale, float v_scale, int32_t* dev_status, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID;
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) || !(v_scale > 0.f))
    return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim % 16) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k_cache || !v_cache || !k || !v || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
    return PA_ERR_INVALID;
  const int cpr = head_dim / 16;
  const long long total = (long long)num_tokens * num_kv_heads * cpr;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  long long blocks = (total + 255) / 256;
  if (blocks > (long long)sms * 16) blocks = (long long)sms * 16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == PA_BF16)
    e = pkv_host::launch(pkv::pa_cache_append_e4m3_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3(256),
               0, st, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
               static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
               num_tokens, num_kv_heads, cpr, block_size, num_blocks, k_scale, v_scale,
               (const float*)nullptr, (const float*)nullptr, dev_status);
  else
    e = pkv_host::launch(pkv::pa_cache_append_e4m3_kernel<__half>, dim3((unsigned)blocks), dim3(256), 0, st,
               static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
               static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
               num_tokens, num_kv_heads, cpr, block_size, num_blocks, k_scale, v_scale,
               (const float*)nullptr, (const float*)nullptr, dev_status);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_cache_append_e4m3_bs(void* k_cache, void* v_cache, float* k_scales,
                                  float* v_scales, const void* k, const void* v,
                                  const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                                  int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                                  int32_t* dev_status, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim % 16) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k_cache || !v_cache || !k || !v || !slot_mapping || !k_scales || !v_scales)
    return PA_ERR_INVALID;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
    return PA_ERR_INVALID;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // 1. the blocks whose offset 0 is written here take their scales from that token
  const long long warps = (long long)num_tokens * num_kv_heads;
  const unsigned sblocks = (unsigned)((warps * 32 + 255) / 256);
  cudaError_t e =
      dtype == PA_BF16
          ? pkv_host::launch(pkv::pa_e4m3_block_scale_kernel<__nv_bfloat16>, dim3(sblocks), dim3(256),
                             0, st, k_scales, v_scales, static_cast<const __nv_bfloat16*>(k),
                             static_cast<const __nv_bfloat16*>(v), slot_mapping, num_tokens,
                             num_kv_heads, head_dim, block_size, num_blocks)
          : pkv_host::launch(pkv::pa_e4m3_block_scale_kernel<__half>, dim3(sblocks), dim3(256), 0, st,
                             k_scales, v_scales, static_cast<const __half*>(k),
                             static_cast<const __half*>(v), slot_mapping, num_tokens, num_kv_heads,
                             head_dim, block_size, num_blocks);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  // 2. every token quantised with its block's scales
  const int cpr = head_dim / 16;
  const long long total = (long long)num_tokens * num_kv_heads * cpr;
  long long blocks = (total + 255) / 256;
  if (blocks > (long long)sms * 16) blocks = (long long)sms * 16;
  if (dtype == PA_BF16)
    e = pkv_host::launch(pkv::pa_cache_append_e4m3_kernel<__nv_bfloat16>, dim3((unsigned)blocks),
                         dim3(256), 0, st, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                         static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
                         num_tokens, num_kv_heads, cpr, block_size, num_blocks, 1.f, 1.f,
                         (const float*)k_scales, (const float*)v_scales, dev_status);
  else
    e = pkv_host::launch(pkv::pa_cache_append_e4m3_kernel<__half>, dim3((unsigned)blocks), dim3(256),
                         0, st, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                         static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
                         num_tokens, num_kv_heads, cpr, block_size, num_blocks, 1.f, 1.f,
                         (const float*)k_scales, (const float*)v_scales, dev_status);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode_e4m3_bs(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const float* k_scales, const float* v_scales,
                            const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                            int q_len, int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                            pa_dtype dtype, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream) {
  if (num_seqs > 0 && (!k_scales || !v_scales)) return PA_ERR_INVALID;
  CascadeArgs cx;
  cx.kv8 = true;
  cx.k_bscale = k_scales;
  cx.v_bscale = v_scales;
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, q_len,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, workspace, workspace_bytes, 0, dev_status, stream,
                     cx);
}

size_t pa_decode_cascade_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads,
                                         int head_dim) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0) return 0;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  return cascade_layout(num_seqs, num_q_heads, head_dim, sms).total;
}

pa_status pa_decode_cascade(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            const int32_t* prefix_lens, int num_seqs,
                            const int32_t* chunk_members, int chunk_width,
                            const int32_t* chunk_prefix_lens, int num_chunks, int num_q_heads,
                            int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int num_blocks, float scale, pa_dtype dtype,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream) {
  return cascade_impl(out, q, k_cache, v_cache, block_tables, context_lens, prefix_lens,
                      num_seqs, chunk_members, chunk_width, chunk_prefix_lens, num_chunks,
                      num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                      num_blocks, scale, dtype, workspace, workspace_bytes, dev_status, stream,
                      CascadeArgs());
}

pa_status pa_decode_cascade_e4m3_bs(void* out, const void* q, const void* k_cache,
                                    const void* v_cache, const float* k_scales,
                                    const float* v_scales, const int32_t* block_tables,
                                    const int32_t* context_lens, const int32_t* prefix_lens,
                                    int num_seqs, const int32_t* chunk_members, int chunk_width,
                                    const int32_t* chunk_prefix_lens, int num_chunks,
                                    int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int num_blocks,
                                    float scale, pa_dtype dtype, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (num_seqs > 0 && (!k_scales || !v_scales)) return PA_ERR_INVALID;
  CascadeArgs cx;
  cx.kv8 = true;
  cx.k_bscale = k_scales;
  cx.v_bscale = v_scales;
  return cascade_impl(out, q, k_cache, v_cache, block_tables, context_lens, prefix_lens,
                      num_seqs, chunk_members, chunk_width, chunk_prefix_lens, num_chunks,
                      num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                      num_blocks, scale, dtype, workspace, workspace_bytes, dev_status, stream,
                      cx);
}

pa_status pa_decode_append_e4m3_bs(void* out, const void* q, void* k_cache, void* v_cache,
                                   float* k_scales, float* v_scales, const void* k_new,
                                   const void* v_new, const int32_t* block_tables,
                                   const int32_t* context_lens, int num_seqs, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int max_blocks_per_seq, int num_blocks, float scale,
                                   pa_dtype dtype, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_status, void* stream) {
  if (num_seqs > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new) ||
                       !k_scales || !v_scales))
    return PA_ERR_INVALID;
  CascadeArgs cx;
  cx.mode = pkv::kAppend;
  cx.k_new = k_new;
  cx.v_new = v_new;
  cx.kv8 = true;
  cx.k_bscale = k_scales;
  cx.v_bscale = v_scales;
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, workspace, workspace_bytes, 0, dev_status, stream,
                     cx);
}

pa_status pa_cache_append(void* k_cache, void* v_cache, const void* k, const void* v,
                          const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                          int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                          int32_t* dev_status, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if ((head_dim * 2) % 16) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k_cache || !v_cache || !k || !v || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
    return PA_ERR_INVALID;
  const int cpr = head_dim * 2 / 16;
  const long long total = (long long)num_tokens * num_kv_heads * cpr;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  long long blocks = (total + 255) / 256;
  if (blocks > (long long)sms * 16) blocks = (long long)sms * 16;
  if (pkv_host::launch(pkv::pa_cache_append_kernel, dim3((unsigned)blocks), dim3(256), 0,
             static_cast<cudaStream_t>(stream), static_cast<uint4*>(k_cache),
             static_cast<uint4*>(v_cache), static_cast<const uint4*>(k),
             static_cast<const uint4*>(v), slot_mapping, num_tokens, num_kv_heads, cpr,
             block_size, num_blocks, dev_status) != cudaSuccess)
    return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void* const* k_caches, void* const* v_caches, int num_layers,
                         const int32_t* pairs, int num_pairs, int num_blocks, size_t block_bytes,
                         int32_t* dev_status, void* stream) {
  if (num_layers < 0 || num_pairs < 0 || num_blocks <= 0 || block_bytes == 0 ||
      block_bytes % 16)
    return PA_ERR_INVALID;
  if (num_layers == 0 || num_pairs == 0) return PA_OK;
  if (!k_caches || !v_caches || !pairs) return PA_ERR_INVALID;
  for (int l = 0; l < num_layers; ++l)
    if (!k_caches[l] || !v_caches[l] || !aligned16(k_caches[l]) || !aligned16(v_caches[l]))
      return PA_ERR_INVALID;
  for (int l0 = 0; l0 < num_layers; l0 += pkv::kMaxLayersPerLaunch) {
    const int n = (num_layers - l0) < pkv::kMaxLayersPerLaunch ? (num_layers - l0)
                                                               : pkv::kMaxLayersPerLaunch;
    pkv::LayerPtrs P;
    std::memset(&P, 0, sizeof(P));
    for (int i = 0; i < n; ++i) {
      P.k[i] = static_cast<uint4*>(k_caches[l0 + i]);
      P.v[i] = static_cast<uint4*>(v_caches[l0 + i]);
    }
    dim3 grid((unsigned)num_pairs, (unsigned)(2 * n));
    if (pkv_host::launch(pkv::pa_copy_blocks_kernel, grid, dim3(256), 0, static_cast<cudaStream_t>(stream),
               P, pairs, num_blocks, (long long)(block_bytes / 16), dev_status) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  return PA_OK;
}

pa_status pa_check_bounded_waits(int32_t* result, int limit_us, void* stream) {
  if (!result || (reinterpret_cast<uintptr_t>(result) & 3) || limit_us < 1 || limit_us > 2000000)
    return PA_ERR_INVALID;
  pkv::pa_wait_check_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      result, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"

namespace {

// The device-side address of a swap buffer: page-locked host memory (cudaHostAlloc,
// cudaMallocHost or cudaHostRegister) or device memory; nullptr for memory a kernel
// cannot reach (pageable host memory), which is refused rather than faulted on.
void* device_view(void* p) {
  cudaPointerAttributes at;
  if (!p || cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost && at.type != cudaMemoryTypeDevice &&
      at.type != cudaMemoryTypeManaged)
    return nullptr;
  return at.devicePointer;
}

pa_status swap_blocks(bool out, void* buf, void* const* k_caches, void* const* v_caches,
                      int num_layers, const int32_t* blocks, int n, int num_blocks,
                      size_t block_bytes, int32_t* dev_status, void* stream) {
  if (num_layers < 0 || n < 0 || num_blocks <= 0 || block_bytes == 0 || block_bytes % 16)
    return PA_ERR_INVALID;
  if (num_layers == 0 || n == 0) return PA_OK;
  if (!k_caches || !v_caches || !blocks || !buf) return PA_ERR_INVALID;
  for (int l = 0; l < num_layers; ++l)
    if (!k_caches[l] || !v_caches[l] || !aligned16(k_caches[l]) || !aligned16(v_caches[l]))
      return PA_ERR_INVALID;
  void* dbuf = device_view(buf);
  if (!dbuf || !aligned16(dbuf)) return PA_ERR_INVALID;
  for (int l0 = 0; l0 < num_layers; l0 += pkv::kMaxLayersPerLaunch) {
    const int m = (num_layers - l0) < pkv::kMaxLayersPerLaunch ? (num_layers - l0)
                                                               : pkv::kMaxLayersPerLaunch;
    pkv::LayerPtrs P;
    std::memset(&P, 0, sizeof(P));
    for (int i = 0; i < m; ++i) {
      P.k[i] = static_cast<uint4*>(k_caches[l0 + i]);
      P.v[i] = static_cast<uint4*>(v_caches[l0 + i]);
    }
    dim3 grid((unsigned)n, (unsigned)(2 * m));
    const cudaError_t e =
        out ? pkv_host::launch(pkv::pa_swap_blocks_kernel<true>, grid, dim3(256), 0,
                               static_cast<cudaStream_t>(stream), P, blocks, n, num_blocks,
                               (long long)(block_bytes / 16), l0, static_cast<uint4*>(dbuf),
                               dev_status)
            : pkv_host::launch(pkv::pa_swap_blocks_kernel<false>, grid, dim3(256), 0,
                               static_cast<cudaStream_t>(stream), P, blocks, n, num_blocks,
                               (long long)(block_bytes / 16), l0, static_cast<uint4*>(dbuf),
                               dev_status);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

extern "C" {

pa_status pa_swap_out_blocks(void* host_dst, void* const* k_caches, void* const* v_caches,
                             int num_layers, const int32_t* blocks, int n, int num_blocks,
                             size_t block_bytes, int32_t* dev_status, void* stream) {
  return swap_blocks(true, host_dst, k_caches, v_caches, num_layers, blocks, n, num_blocks,
                     block_bytes, dev_status, stream);
}

pa_status pa_swap_in_blocks(void* const* k_caches, void* const* v_caches, int num_layers,
                            const int32_t* blocks, int n, int num_blocks, const void* host_src,
                            size_t block_bytes, int32_t* dev_status, void* stream) {
  return swap_blocks(false, const_cast<void*>(host_src), k_caches, v_caches, num_layers, blocks,
                     n, num_blocks, block_bytes, dev_status, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// pa_decode_noalloc: pa_decode with its scratch in a fixed device array of this file, for
// callers that cannot allocate device memory (see include/pagedkv.h).
// ---------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoallocScratchBytes = PA_NOALLOC_SCRATCH_BYTES;
// split CTAs the scratch is sized for: 3 mma.sync CTAs per SM on a 148-SM B200, the most
// pa_decode runs there (block_size <= 8), or one tcgen05 CTA per SM; a GPU with more SMs
// runs at most this many
constexpr int kNoallocMaxGrid = 444;
constexpr int kNoallocMaxDevices = 64;
static_assert(ws_layout(128, kNoallocMaxGrid, pkv::kMaxGroup).total <= kNoallocScratchBytes,
              "the scratch must hold the split partials of kNoallocMaxGrid CTAs at head_dim 128");
static_assert(ws_layout(128, kNoallocMaxGrid / pkv::kMaxCtasPerSm, pkv::kWideCols).total <=
                  kNoallocScratchBytes,
              "and those of the tcgen05 kernel's CTAs (one a SM, 64 query columns)");

// Lives in the module's global memory: every device that loads the library holds it
// until the process exits.  Host code must not pass its name to a kernel (on the host
// it is only a stand-in); the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch on the current device; looked up once per device
// (the first call on a device does it) and cached.  nullptr on failure.
void* noalloc_scratch(int dev) {
  static std::mutex mu;
  static void* addr[kNoallocMaxDevices] = {};
  if (dev < 0 || dev >= kNoallocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       const int32_t* context_lens, int num_seqs,
                                       int num_q_heads, int num_kv_heads, int head_dim,
                                       int block_size, int max_blocks_per_seq, int num_blocks,
                                       float scale, pa_dtype dtype, int32_t* dev_status,
                                       void* stream) {
  if (num_seqs > PA_NOALLOC_MAX_SEQS) return PA_ERR_INVALID;   // the call's stated limit
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1,
                       num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                       num_blocks, scale, dtype, nullptr, 0, kNoallocMaxGrid, dev_status, stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (head_dim > 128) return PA_ERR_UNSUPPORTED;   // the scratch holds head_dim <= 128
  void* ws = noalloc_scratch(dev);
  if (!ws) return PA_ERR_CUDA;
  return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, scale, dtype, ws, kNoallocScratchBytes, kNoallocMaxGrid,
                     dev_status, stream);
}
