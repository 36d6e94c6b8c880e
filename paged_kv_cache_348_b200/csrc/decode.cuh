// decode.cuh -- paged decode attention for sm_100a.
//
// What it computes is defined in "Paged Attention and Memory Efficiency in Production
// LLM Serving", section "How PagedAttention borrows OS paging": the attention kernel
// resolves each request's block table at run time and the arithmetic is the plain
// softmax(scale q K^T) V; "PagedAttention -- The KV Cache Problem", section "How It
// Works": the kernel reads the block table to gather K/V from non-contiguous blocks.
//
// Design (B200):
//  * Work is the set of (sequence, kv head) segments, cut into 16-token units.  The
//    units of all segments are laid end to end and split into gridDim.x equal
//    ranges, one per persistent CTA (2 per SM; 3 with one query-column tile for 8-bit
//    caches or block_size <= 8), so a batch with a heavy-tailed
//    length mix still gives every SM the same number of KV bytes.  A segment that
//    straddles CTA ranges leaves one (max, sum, acc) partial per CTA in the
//    workspace; the last of those CTAs to finish (an epoch-tagged arrival counter,
//    released and acquired at GPU scope) merges them with a log-sum-exp reduction in
//    CTA order, so the result does not depend on which CTA came last and no second
//    kernel is needed.  The merge folds the partials in with a running maximum, several
//    contributors per L2 round trip: it sits at the end of most CTAs' ranges, on the
//    kernel's critical path.
//  * The producer keeps a window of block-table entries in registers, loaded 64 blocks
//    ahead of use (at block_size 1, three windows ahead), so the only table read a stage
//    waits for is a portion's first.
//  * Per CTA: one producer warp walks the CTA's range and streams K/V tiles of 64
//    tokens into a shared-memory ring (2-5 stages by configuration): for block_size >= 8
//    with 2-D TMA tensor copies (128-byte swizzle, box = min(block_size,16) rows x 64
//    dims) whose row coordinate is the physical block id read from the block table; for
//    block_size 1 with TMA gather4 loads of four 128-byte rows from four table entries.
//    Stages complete on mbarriers with transaction counts.
//  * Four consumer warps each take one 16-token unit of a stage.  All query rows of a
//    kv head -- the GQA group's heads times the new tokens of the sequence -- share
//    every K/V byte: S^T = K q^T and O^T += V^T P^T run as m16n8k16 tensor-core MMAs
//    with the tokens (resp. head dims) on M and those query rows on N (a group of 8
//    heads fills one n-tile exactly; up to 16 rows here, 9 to 64 also on the tcgen05
//    kernel of decode_wide.cuh).  With several new tokens, token j is masked from the
//    cached positions after its own.  Softmax is an fp32 online softmax in base 2; P is
//    split into a 16-bit high part and a 16-bit residual so the PV product keeps ~16
//    mantissa bits.  8-bit (E4M3) tiles are converted to fp16 fragments after ldmatrix.
//  * Every wait is bounded (2 s); on give-up the CTA sets PA_DEV_TIMEOUT and leaves.
//  * Launched with programmatic dependent launch: the prologue -- and the producer's
//    schedule, which reads only lengths, starts and block tables -- overlaps the previous
//    kernel's tail; nothing else global is touched before griddepcontrol.wait.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "ptx.cuh"

namespace pkv {

constexpr int kUnit = 16;                           // tokens per schedule unit
// Schedule weight of a segment beyond its units: a portion's fixed cost (first stage,
// end-of-portion merge) is worth about this many units of streaming, so a CTA whose range
// holds many short segments gets fewer units.  The weight is a tail of virtual units after
// each segment's real ones; ranges that fall on it do no work.  With block_size 1 a unit
// costs more (the producer issues a gather per 4 rows), so the tail is shorter.
__host__ __device__ constexpr int seg_weight(int bs) { return bs == 1 ? 2 : 8; }
constexpr int kConsumerWarps = 4;
constexpr int kUnitsPerStage = kConsumerWarps;      // one unit per consumer warp
constexpr int kTileTokens = kUnit * kUnitsPerStage; // 64 tokens per stage
constexpr int kStages = 3;
constexpr int kThreads = 32 * (1 + kConsumerWarps); // warp 0 produces, 1..4 consume
// Resident CTAs per SM: 2, or 3 with one query-column tile (128 registers a thread) when
// the rate is set per CTA rather than by HBM: 8-bit caches, whose consumers also convert
// codes (half-size stages keep a 3-deep ring), and block_size <= 8, whose producer issues
// a copy per 16 bytes (block_size 1) or per 1 KB box (block_size 8); 16-bit stages then
// form a 2-deep ring.
// 8-bit tile rows: D bytes at D = 128 or 64, 16-byte chunk c of row r stored at chunk
// c ^ kv8_swz(r): the 128-byte swizzle (the row's low 3 bits) or the 64-byte one (bits 1-2:
// two 64-byte rows share a 128-byte line), the patterns TMA writes
template <int D>
__host__ __device__ constexpr int kv8_swz(int r) {
  return D == 128 ? (r & 7) : ((r >> 1) & 3);
}

__host__ __device__ constexpr int ctas_per_sm(bool kv8, int nt, int bs) {
  return (kv8 || bs <= 8) && nt == 1 ? 3 : 2;
}
constexpr int kMaxCtasPerSm = 3;        // the split workspace covers this many per SM
constexpr int kMaxGroup = 16;                       // q heads per kv head handled
constexpr uint64_t kWaitLimitNs = 2000000000ull;

constexpr int DEV_BAD_BLOCK_ID = 0x1;
constexpr int DEV_BAD_CONTEXT_LEN = 0x8;
constexpr int DEV_TIMEOUT = 0x10;

enum : int { F_FIRST = 1, F_LAST = 2, F_END = 4, F_COMPLETE = 8, F_PREFIX = 16 };

// What a launch decodes (a template parameter, so the plain path carries none of the rest):
//  kPlain   -- every sequence over its cached tokens 0..ctx-1; q_len new tokens, causal.
//  kPrefix  -- cascade pass 1: "sequences" are chunks of sibling sequences sharing a prefix
//              of ctx tokens (read through the first member's block table); the query
//              columns are the members' rows, no causal mask, and the result is each
//              member's unnormalised (max, sum, acc) written to the external partials.
//  kSuffix  -- cascade pass 2: sequence s over its tokens seq_start[s]..ctx-1, merged with
//              the external partial of its prefix when seq_start[s] > 0.
//  kAppend  -- kPlain with one new token per sequence whose K/V (k_new, v_new) are patched
//              into the tiles and written to the cache in the same launch.
enum : int { kPlain = 0, kPrefix = 1, kSuffix = 2, kAppend = 3 };

struct StageMeta {
  int seq, kvh, tok0, nunits, ctx, flags, pidx, qslot;
  int newrow;                           // fused append: cache row of the new token, or -1
};

struct SeqSpan {
  int ctx, first;                       // tokens first..ctx-1 are decoded
};

// A segment portion this CTA shares with other CTAs, handed to the merger warp.
struct SplitDesc {
  int seq, kvh, cf, cl, ncontrib;       // first/last CTA of the segment, CTAs with units
  int has_prefix;                       // kSuffix: the sequence has a prefix partial
  long long seg0;                       // first unit of the segment
};

struct DecodeArgs {
  void* out;
  const void* q;
  const void* k_cache;          // used directly by the block_size-1 path
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* part_acc;              // [gridDim*2][kMaxGroup][D]
  float* part_ml;               // [gridDim*2][kMaxGroup][2]  (max, sum) in base 2
  unsigned long long* counters; // [gridDim] arrival counters: (epoch << 32) | arrivals
  int32_t* status;              // nullable
  int num_seqs, num_q_heads, num_kv_heads, group, max_blocks, num_blocks, ctx_cap;
  int q_len;                    // new tokens per sequence (query rows [seq][q_len][Hq][D])
  int ncol;                     // query rows per kv head: group * q_len (MMA columns)
  float scale_log2;             // scale * log2(e)
  uint32_t epoch;               // distinct per call: counters of older calls read as zero
  // cascade (kPrefix / kSuffix launches only)
  const int32_t* seq_start;     // kSuffix: first token of each sequence's own part
  const int32_t* chunk_members; // kPrefix: [num_seqs][q_len] member sequences, -1 pad
  int q_rows;                   // kPrefix: sequences in q / block_tables (valid member ids)
  int late_wait;                // kSuffix: wait for the previous grid (the cascade's prefix
                                // pass, whose only output this launch reads is the external
                                // partials) before reading those, and at the end, not at
                                // the start
  float2* ext_ml;               // [members][Hq] (max, sum) of the prefix part, base 2
  float* ext_acc;               // [members][Hq][D] its unnormalised accumulator
  // kAppend: K/V of each sequence's newest token, [seqs][Hkv][D]
  const void* k_new;
  const void* v_new;
  float v_scale;                // 8-bit caches: value = v_scale * code (1 otherwise); the
                                // K scale is folded into scale_log2
  // 8-bit caches with per-(block, kv head) scales [num_blocks][Hkv] (null: per-tensor)
  const float* k_bscale;
  const float* v_bscale;
};


// Shared-memory layout of a CTA.  16-bit caches: K and V tiles of 64 tokens in D/64
// column halves of 128-byte lines; 8-bit (E4M3) caches: one row of D bytes per token
// (D = 128: a 128-byte line, 128-byte swizzle; D = 64: a 64-byte row, 64-byte swizzle),
// and, since a stage is half the size, a deeper ring.  CPS = CTAs per SM;
// NEW: the fused append's staged rows, SC: the 8-bit per-row scales (regions left out
// when the launch has no use for them: every byte of shared memory a CTA takes is L1 the
// spilled registers of the 3-CTA configurations no longer have).
template <int D, bool KV8 = false, int CPS = 2, bool NEW = true, bool SC = KV8, bool G1 = false>
struct Layout {
  // 8-bit pools with per-row scales at 3 CTAs per SM: a 2-deep ring leaves the spilling
  // consumers more L1 (the fused append over them: 6.11 -> 5.61 ms per 70B-shape step);
  // with per-pool scales the 3-deep ring is faster (4.84 vs 5.04 ms)
  static constexpr int kStages = KV8 ? (CPS == 2 ? 5 : (SC ? 2 : 3)) : (CPS == 2 ? 3 : 2);
  static_assert(CPS == 2 || CPS == 3, "2 or 3 CTAs per SM");
  static constexpr int kHalves = D / 64;                   // 128-byte swizzled column halves
  static constexpr int kKvBytes = KV8 ? kTileTokens * D : kHalves * kTileTokens * 128;
  // the 16-bit query rows of the stage's columns: at 3 CTAs per SM (one n-tile) at most 8
  static constexpr int kQBytes = (CPS == 3 ? 8 : kMaxGroup) * D * 2;
  static constexpr int kStageBytes = 2 * kKvBytes + kQBytes;
  static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
  static constexpr int kMetaOff = kStages * kStageBytes;
  static constexpr int kBarOff = (kMetaOff + kStages * (int)sizeof(StageMeta) + 15) / 16 * 16;
  // full[kStages], empty[kStages]
  static constexpr int kMiscOff = kBarOff + (2 * kStages + 1) * 8;
  // abort flag, last-arrival flag, total units
  static constexpr int kDescOff = kMiscOff + 16;
  static constexpr int kMlOff = kDescOff + 2 * (int)sizeof(SplitDesc);
  // fused append: per stage the new token's K and V rows, staged by the producer
  static constexpr int kNewOff = (kMlOff + kConsumerWarps * kMaxGroup * 8 + 15) / 16 * 16;
  static constexpr int kNewBytes = NEW ? 2 * D * 2 : 0;   // the new token's 16-bit K, V rows
  // 8-bit caches with per-(block, kv head) scales: per stage the K and V scale of every
  // token row, staged by the producer
  static constexpr int kScOff = kNewOff + kStages * kNewBytes;
  static constexpr int kScBytes = SC ? 2 * kTileTokens * 4 : 0;
  // block size 1 (G1), for the consumer warp that issues the V gathers: per stage the row
  // coordinates of the fill, a barrier the producer arrives on once they are written and
  // the fill's count of 4-row groups (0: the producer is done); then that warp's count of
  // the arrivals it has taken
  static constexpr int kYOff = (kScOff + kStages * kScBytes + 15) / 16 * 16;
  static constexpr int kYBytes = G1 ? kTileTokens * 4 : 0;
  static constexpr int kYBarOff = kYOff + kStages * kYBytes;
  static constexpr int kYMarkOff = kYBarOff + (G1 ? kStages * 8 : 0);
  static constexpr int kBytes = kYMarkOff + (G1 ? (kStages + 1) * 4 : 0);
  static constexpr int kDynSmem = kBytes + 1024;           // slack for 1024-byte alignment
  static_assert(kBarOff % 8 == 0 && kMiscOff % 8 == 0 && kDescOff % 8 == 0 && kMlOff % 8 == 0 &&
                    kNewOff % 16 == 0 && kNewBytes % 16 == 0 && kYBarOff % 8 == 0,
                "mbarriers and 64-bit fields need 8-byte, bulk-copy targets 16-byte alignment");
  static_assert(CPS * (kDynSmem + 1024) <= 233472, "CPS CTAs per SM must fit");
};

__device__ __forceinline__ void st_relaxed_gpu(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long cas_acq_rel_gpu(unsigned long long* p,
                                                              unsigned long long cmp,
                                                              unsigned long long val) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.cas.b64 %0, [%1], %2, %3;"
               : "=l"(old)
               : "l"(p), "l"(cmp), "l"(val)
               : "memory");
  return old;
}

__device__ __forceinline__ int clamp_ctx(int c, int cap, int32_t* status) {
  if (c < 0 || c > cap) {
    if (status) atomicOr(status, DEV_BAD_CONTEXT_LEN);
    c = c < 0 ? 0 : cap;
  }
  return c;
}

// Member slot j of chunk s in a prefix launch, or -1 (padding or out of range).
__device__ __forceinline__ int chunk_member(const DecodeArgs& a, int s, int j) {
  const int mem = a.chunk_members[(long long)s * a.q_len + j];
  return (mem >= 0 && mem < a.q_rows) ? mem : -1;
}

template <int MODE>
__device__ __forceinline__ SeqSpan span_of(const DecodeArgs& a, int s, int32_t* status) {
  SeqSpan r;
  r.ctx = clamp_ctx(a.context_lens[s], a.ctx_cap, status);
  r.first = 0;
  if constexpr (MODE == kPrefix) {
    if (chunk_member(a, s, 0) < 0) r.ctx = 0;     // a chunk needs a valid first member
  }
  if constexpr (MODE == kSuffix) {
    const int f = a.seq_start[s];
    r.first = f < 0 ? 0 : (f > r.ctx ? r.ctx : f);
  }
  return r;
}

// Output row (sequence, head) of query column h of sequence/chunk `seq`, kv head kvh:
// -1 when the column is a padding member slot of a chunk.
template <int MODE>
__device__ __forceinline__ long long out_row(const DecodeArgs& a, int seq, int kvh, int h) {
  const int j = h / a.group, g = h % a.group;
  if constexpr (MODE == kPrefix) {
    const int mem = chunk_member(a, seq, j);
    return mem < 0 ? -1ll : (long long)mem * a.num_q_heads + (long long)kvh * a.group + g;
  } else {
    return ((long long)seq * a.q_len + j) * a.num_q_heads + (long long)kvh * a.group + g;
  }
}

// Index of the CTA whose unit range [start(c), start(c+1)) holds unit x, where
// start(c) = floor(c * total / G).
__device__ __forceinline__ int cta_of(long long x, long long total, int G) {
  return (int)(((x + 1) * (long long)G + total - 1) / total) - 1;
}
__device__ __forceinline__ long long cta_start(int c, long long total, int G) {
  return (long long)c * total / G;
}

template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (std::is_same_v<T, __nv_bfloat16>) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}
template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t x) {
  if constexpr (std::is_same_v<T, __nv_bfloat16>) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&x));
  } else {
    return __half22float2(*reinterpret_cast<__half2*>(&x));
  }
}
template <typename T>
__device__ __forceinline__ T from_float(float x) {
  if constexpr (std::is_same_v<T, __nv_bfloat16>) return __float2bfloat16_rn(x);
  else return __float2half_rn(x);
}

// Finish one output value from this launch's (M, L, acc) of a column: kPlain writes
// acc / L; kPrefix stores the unnormalised triple; kSuffix first folds in the prefix
// partial (xm, xa), which the caller loaded beforehand (xm.x = -inf: none).  `d0` is the
// first of `n` consecutive dims held in acc[] (n = 1 or 4).
template <typename T, int MODE, int D>
__device__ __forceinline__ void finish_row(const DecodeArgs& a, long long row, float M, float L,
                                           float* acc, int d0, int n, float2 xm,
                                           const float* xa) {
  if constexpr (MODE == kPrefix) {
    if (d0 == 0) a.ext_ml[row] = make_float2(M, L);
    for (int i = 0; i < n; ++i) a.ext_acc[row * D + d0 + i] = acc[i];
    return;
  } else {
    if constexpr (MODE == kSuffix) {
      if (xm.x != -INFINITY) {
        const float mn = fmaxf(M, xm.x);
        const float sa = M == -INFINITY ? 0.f : ex2(M - mn);
        const float sb = ex2(xm.x - mn);
        L = L * sa + xm.y * sb;
        for (int i = 0; i < n; ++i) acc[i] = acc[i] * sa + xa[i] * sb;
        M = mn;
      }
    }
    T* o = static_cast<T*>(a.out) + row * D + d0;
    const float inv = L > 0.f ? a.v_scale / L : 0.f;
    if (n == 4) {
      *reinterpret_cast<uint2*>(o) = make_uint2(pack2<T>(acc[0] * inv, acc[1] * inv),
                                                pack2<T>(acc[2] * inv, acc[3] * inv));
    } else {
      for (int i = 0; i < n; ++i) o[i] = from_float<T>(acc[i] * inv);
    }
  }
}

// Rows of a sequence (or chunk) that owns no unit, written by one warp: kPlain zeroes its
// output rows; kPrefix marks its members' prefix partials empty; kSuffix normalises the
// prefix partial (zero if there is none).
template <typename T, int MODE, int D>
__device__ __forceinline__ void empty_rows(const DecodeArgs& a, int s, int first, int lane) {
  const int Hq = a.num_q_heads;
  if constexpr (MODE == kPrefix) {
    for (int j = 0; j < a.q_len; ++j) {
      const int mem = chunk_member(a, s, j);
      if (mem < 0) continue;
      for (int h = lane; h < Hq; h += 32)
        a.ext_ml[(long long)mem * Hq + h] = make_float2(-INFINITY, 0.f);
    }
  } else if constexpr (MODE == kSuffix) {
    for (int i = lane; i < Hq * (D / 4); i += 32) {
      const long long row = (long long)s * Hq + i / (D / 4);
      const int d = (i % (D / 4)) * 4;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (first > 0) {
        const float2 x = __ldcg(a.ext_ml + row);
        const float4 y = __ldcg(reinterpret_cast<const float4*>(a.ext_acc + row * D + d));
        if (x.x != -INFINITY && x.y > 0.f) {
          const float inv = 1.f / x.y;
          v[0] = y.x * inv, v[1] = y.y * inv, v[2] = y.z * inv, v[3] = y.w * inv;
        }
      }
      *reinterpret_cast<uint2*>(static_cast<T*>(a.out) + row * D + d) =
          make_uint2(pack2<T>(v[0], v[1]), pack2<T>(v[2], v[3]));
    }
  } else {
    uint4* row = reinterpret_cast<uint4*>(static_cast<T*>(a.out) + (long long)s * a.q_len * Hq * D);
    for (int i = lane; i < a.q_len * Hq * D * 2 / 16; i += 32) row[i] = make_uint4(0, 0, 0, 0);
  }
}

// Four E4M3 codes (bytes 0..3 of x) to fp16 pairs (bytes 0, 1) and (bytes 2, 3), exactly.
// Splitting the word with mov.b32 hands each conversion a register half directly (no
// shift or mask to extract the upper pair).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

// Entry i (0 <= i < 96) of a block-table window held across the warp: lane l holds
// entries l, 32+l and 64+l in x0, x1, x2.  Every lane must call it.
__device__ __forceinline__ int win_lookup(int x0, int x1, int x2, int i) {
  const int a = __shfl_sync(0xffffffffu, x0, i & 31);
  const int b = __shfl_sync(0xffffffffu, x1, i & 31);
  const int c = __shfl_sync(0xffffffffu, x2, i & 31);
  return i < 32 ? a : (i < 64 ? b : c);
}

// ------------------------------------------------------------------------------------
// The decode kernel: every CTA processes its unit range; rows of segments it covers
// whole go straight to `out`, segments shared with other CTAs go through partials
// and the last contributing CTA merges them.
// ------------------------------------------------------------------------------------
// Partial slot of CTA cc for the segment starting at unit seg0 (-1: CTA without units).
__device__ __forceinline__ int partial_slot(int cc, long long seg0, long long total, int G) {
  const long long s0 = cta_start(cc, total, G);
  return s0 < cta_start(cc + 1, total, G) ? cc * 2 + (s0 < seg0 ? 1 : 0) : -1;
}

// Last arrival of a split segment: out = (sum_k acc_k 2^(m_k - M)) / (sum_k l_k 2^(m_k - M)),
// M = max_k m_k, over the contributing CTAs k.  Run by the 128 consumer threads; thread
// tid owns output elements (head, 4 dims) e = tid + 128 i.  The partials are folded in
// CTA order with a running maximum (so the result does not depend on which CTA arrived
// last), kMC contributors at a time with every load of a group issued before any use:
// one L2 round trip per group.
template <typename T, int D, int NT, int MODE>
__device__ __forceinline__ void merge_split(const DecodeArgs& a, const SplitDesc& dsc,
                                            long long total, int G, int group, int tid) {
  constexpr int kThr = 32 * kConsumerWarps;
  constexpr int kF4 = D / 4;
  constexpr int kPer = (8 * NT * kF4 + kThr - 1) / kThr;  // float4 elements per thread (max)
  constexpr int kMC = kPer >= 4 ? 2 : 4;                    // contributors per round trip
  const int nel = a.ncol * kF4;
  const int nr = dsc.cl - dsc.cf + 1;
  float M[kPer], Lsum[kPer];
  float4 acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    M[e] = -INFINITY;
    Lsum[e] = 0.f;
    acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int k0 = 0; k0 < nr; k0 += kMC) {
    int pk[kMC];
    float2 ml[kMC][kPer];
    float4 v[kMC][kPer];
#pragma unroll
    for (int k = 0; k < kMC; ++k) {
      pk[k] = k0 + k < nr ? partial_slot(dsc.cf + k0 + k, dsc.seg0, total, G) : -1;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int i = tid + kThr * e;
        const int h = i / kF4, d4 = i % kF4;
        ml[k][e] = make_float2(-INFINITY, 0.f);
        v[k][e] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (pk[k] >= 0 && i < nel) {
          const long long row = (long long)pk[k] * kMaxGroup + h;
          ml[k][e] = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + row);
          v[k][e] = __ldcg(reinterpret_cast<const float4*>(a.part_acc + row * D) + d4);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kMC; ++k)
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        if (ml[k][e].x == -INFINITY) continue;          // no unit, or an empty partial
        const float mn = fmaxf(M[e], ml[k][e].x);
        const float sa = M[e] == -INFINITY ? 0.f : ex2(M[e] - mn);
        const float sb = ex2(ml[k][e].x - mn);
        Lsum[e] = Lsum[e] * sa + ml[k][e].y * sb;
        acc[e].x = acc[e].x * sa + v[k][e].x * sb;
        acc[e].y = acc[e].y * sa + v[k][e].y * sb;
        acc[e].z = acc[e].z * sa + v[k][e].z * sb;
        acc[e].w = acc[e].w * sa + v[k][e].w * sb;
        M[e] = mn;
      }
  }
  const bool has_prefix = MODE == kSuffix && dsc.has_prefix;
  float2 xm[kPer];
  float4 xa[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {                // the prefix partials, all loads at once
    const int i = tid + kThr * e;
    xm[e] = make_float2(-INFINITY, 0.f);
    xa[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (has_prefix && i < nel) {
      const long long row = out_row<MODE>(a, dsc.seq, dsc.kvh, i / kF4);
      xm[e] = __ldcg(a.ext_ml + row);
      xa[e] = __ldcg(reinterpret_cast<const float4*>(a.ext_acc + row * D) + i % kF4);
    }
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int i = tid + kThr * e;
    if (i >= nel) continue;
    const int h = i / kF4, d4 = i % kF4;           // query column, 4-dim group
    const long long row = out_row<MODE>(a, dsc.seq, dsc.kvh, h);
    if (row < 0) continue;
    float v[4] = {acc[e].x, acc[e].y, acc[e].z, acc[e].w};
    const float x4[4] = {xa[e].x, xa[e].y, xa[e].z, xa[e].w};
    finish_row<T, MODE, D>(a, row, M[e], Lsum[e], v, d4 * 4, 4, xm[e], x4);
  }
}

template <typename T, int D, int BS, int NT, int MODE, bool KV8 = false, bool KSC = false>
__global__ void __launch_bounds__(kThreads, ctas_per_sm(KV8, NT, BS))
    pa_decode_split_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                           const __grid_constant__ CUtensorMap tmv) {
  using L = Layout<D, KV8, ctas_per_sm(KV8, NT, BS), MODE == kAppend, KSC, BS == 1>;
  constexpr int kStages = L::kStages;
  constexpr int kSegW = seg_weight(BS);
  static_assert(!KV8 || D == 128 || D == 64, "8-bit caches: head_dim 128 or 64");
  static_assert(!KV8 || MODE == kPlain || KSC,
                "8-bit caches: the cascade and fused-append modes use per-block scales");
  static_assert(!KSC || KV8, "per-block scales belong to 8-bit caches");
  static_assert(ctas_per_sm(KV8, NT, BS) == 2 || NT == 1, "the 3-CTA layout holds 8 columns");
  // MMA operand type: the cache's 16-bit type, or fp16 for E4M3 (exact there)
  constexpr bool kBF16 = !KV8 && std::is_same_v<T, __nv_bfloat16>;
  constexpr int kFullCount = 1;        // the producer's expect_tx arrival
  constexpr int kConsumerThreads = 32 * kConsumerWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + L::kMetaOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff);
  volatile int* last_flag = abort_flag + 1;
  long long* total_s = reinterpret_cast<long long*>(smem + L::kMiscOff + 8);
  SplitDesc* desc = reinterpret_cast<SplitDesc*>(smem + L::kDescOff);
  float2* mls = reinterpret_cast<float2*>(smem + L::kMlOff);

  // block size 1: the producer issues the K gathers and consumer warp kHelperWarp the V
  // gathers of every fill (a warp issues TMA loads at a bounded rate, and at four rows a
  // load this path is bound by it).  A gather load moves four 128-byte pieces (a column
  // half of a 16-bit row, or a whole 8-bit row; a 64-byte 8-bit row is one piece of its
  // own size).
  constexpr int kHelperWarp = kConsumerWarps - 1;
  constexpr int kGParts = D * (KV8 ? 1 : 2) >= 128 ? D * (KV8 ? 1 : 2) / 128 : 1;
  constexpr int kGPieceB = KV8 ? (D < 128 ? D : 128) : 128;
  uint64_t* yready = reinterpret_cast<uint64_t*>(smem + L::kYBarOff);
  volatile int* ymark = reinterpret_cast<volatile int*>(smem + L::kYMarkOff);
  volatile int* yseen = ymark + kStages;
  int* ycoord = reinterpret_cast<int*>(smem + L::kYOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], kFullCount);
      mbar_init(&empty[i], kConsumerWarps);
      if constexpr (BS == 1) mbar_init(&yready[i], 1);
    }
    if constexpr (BS == 1) *yseen = 0;
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  __syncthreads();
  // Nothing global is written, and nothing a previous kernel may write is read, before the
  // previous grid is done.  The producer of every CTA but CTA 0 (which writes the rows of
  // sequences without units) computes its schedule first: that reads only the launch's
  // lengths, starts and block tables, which no kernel of this library writes.  A late-wait
  // suffix launch's previous grid is the cascade's prefix pass, which writes nothing this
  // launch touches but the external partials, so it waits for that grid only before it
  // reads them (CTA 0's rows without units, every end-of-portion merge) and before it
  // exits; it overlaps the prefix pass's end and still completes after it.
  const bool late_wait = MODE == kSuffix && a.late_wait;
  if (warp != 0 && !late_wait) pdl_wait();
  if (warp != 0) pdl_trigger();

  const int G = gridDim.x, c = blockIdx.x;
  const int Hkv = a.num_kv_heads, group = a.group;

  if (warp == 0) {
    // ============================== producer ==============================
    if (c == 0) pdl_wait();
    const int B = a.num_seqs;
    // pass 1 over the batch: total units; CTA 0 also writes the zero rows of empty
    // sequences (they own no unit).  For B <= 32 the lane values are kept for pass 2.
    long long run = 0;
    int keep_ctx = 0, keep_first = 0, keep_u = 0, keep_x = 0;
#pragma unroll 4
    for (int base = 0; base < B; base += 32) {
      const int s = base + lane;
      SeqSpan sp{0, 0};
      if (s < B) sp = span_of<MODE>(a, s, c == 0 ? a.status : nullptr);
      const int ctx = sp.ctx;
      const int u = (ctx - sp.first + kUnit - 1) / kUnit;
      int x = u ? u + kSegW : 0;                     // weight of each of its segments
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      keep_ctx = ctx;
      keep_first = sp.first;
      keep_u = u;
      keep_x = x;
      run += __shfl_sync(0xffffffffu, x, 31);
      if (c == 0) {
        unsigned zero = __ballot_sync(0xffffffffu, s < B && u == 0);
        while (zero) {
          const int src = __ffs(zero) - 1;
          zero &= zero - 1;
          const int f = MODE == kSuffix ? __shfl_sync(0xffffffffu, sp.first, src) : 0;
          empty_rows<T, MODE, D>(a, base + src, f, lane);
        }
      }
    }
    const long long total = (long long)Hkv * run;
    const long long start = total ? cta_start(c, total, G) : 0;
    const long long end = total ? cta_start(c + 1, total, G) : 0;

    // pass 2: the sequence holding unit `start`
    int s_a = 0, u_a = 0, ctx_a = 0, first_a = 0;
    long long pb_a = 0;
    if (start < end) {
      long long r2 = 0;
      bool got_a = false;
      for (int base = 0; base < B && !got_a; base += 32) {
        const int s = base + lane;
        int ctx = keep_ctx, first = keep_first, u = keep_u, x = keep_x;
        if (B > 32) {
          SeqSpan sp{0, 0};
          if (s < B) sp = span_of<MODE>(a, s, nullptr);
          ctx = sp.ctx;
          first = sp.first;
          u = (ctx - first + kUnit - 1) / kUnit;
          x = u ? u + kSegW : 0;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
          }
        }
        const int wt = u ? u + kSegW : 0;
        const long long lo = (long long)Hkv * (r2 + x - wt), hi = (long long)Hkv * (r2 + x);
        const unsigned ha = __ballot_sync(0xffffffffu, s < B && u > 0 && lo <= start && start < hi);
        if (ha) {
          const int src = __ffs(ha) - 1;
          s_a = base + src;
          u_a = __shfl_sync(0xffffffffu, u, src);
          ctx_a = __shfl_sync(0xffffffffu, ctx, src);
          if constexpr (MODE == kSuffix) first_a = __shfl_sync(0xffffffffu, first, src);
          pb_a = __shfl_sync(0xffffffffu, lo, src);
          got_a = true;
        }
        r2 += __shfl_sync(0xffffffffu, x, 31);
      }
    }
    if (lane == 0) *total_s = total;
    __syncwarp();
    if (c != 0 && !late_wait) pdl_wait();

    const uint64_t policy = policy_evict_first();
    const int rows_total = a.num_blocks * Hkv * BS;
    int st = 0, nq = 0;
    uint32_t ph = 0;
    bool ok = true;
    [[maybe_unused]] int nfill = 0;                  // block size 1: coordinate sets published
    {
      long long x = start;
      const long long xend = end;
      int s_cur = s_a, u_cur = u_a, ctx_cur = ctx_a, first_cur = first_a;
      // the table window at the start of sequence s_win's segments, kept for its next kv
      // head (whose segment starts at the same token), so only a CTA's first portion of a
      // sequence waits on table reads
      int s_win = -1, sw0 = 0, sw1 = 0, sn0 = 0, sn1 = 0;
      int sm0 = 0, sm1 = 0, sp0 = 0, sp1 = 0;         // block_size 1: the deeper windows
      const int32_t* s_trow = a.block_tables;
      long long pbase = pb_a;
      while (ok && x < xend) {
        // a segment spans u_cur units and then kSegW virtual ones (weight w_cur)
        while (x >= pbase + (long long)Hkv * (u_cur ? u_cur + kSegW : 0)) {   // next sequence
          pbase += (long long)Hkv * (u_cur ? u_cur + kSegW : 0);
          ++s_cur;
          const SeqSpan sp = span_of<MODE>(a, s_cur, nullptr);
          ctx_cur = sp.ctx;
          if constexpr (MODE == kSuffix) first_cur = sp.first;
          u_cur = (ctx_cur - first_cur + kUnit - 1) / kUnit;
        }
        const int w_cur = u_cur + kSegW;
        const int kvh = (int)((x - pbase) / w_cur);
        const long long seg0 = pbase + (long long)kvh * w_cur, seg1 = seg0 + u_cur;
        if (x >= seg1) {                              // on the segment's virtual tail
          x = seg0 + w_cur;
          continue;
        }
        const long long pe = seg1 < xend ? seg1 : xend;
        const bool complete = seg0 >= start && seg1 <= end;
        const int pidx = c * 2 + (start < seg0 ? 1 : 0);
        int qslot = 0;
        if (!complete) {
          qslot = nq++;
          if (lane == 0) {
            const int cf = cta_of(seg0, total, G), cl = cta_of(seg1 - 1, total, G);
            int ncontrib = 0;
            for (int cc = cf; cc <= cl; ++cc)
              ncontrib += cta_start(cc, total, G) < cta_start(cc + 1, total, G);
            desc[qslot] = SplitDesc{s_cur, kvh, cf, cl, ncontrib, first_cur > 0 ? 1 : 0, seg0};
          }
        }
        // Block-table window: lane l holds entries wb+l, wb+32+l (w0, w1) and the next 64
        // entries (n0, n1), loaded 64 blocks before they are needed, so no stage waits on a
        // table read except the portion's first.  With block_size 1 a stage uses a whole
        // window of 64 entries, so two more windows (m, p) are kept: every entry is loaded
        // three stages before its stage, which hides a table read that misses L2.
        const int nblk = (ctx_cur + BS - 1) / BS;
        int wb = (first_cur + (int)(x - seg0) * kUnit) / BS;
        const int32_t* trow;
        int w0, w1, n0, n1, m0 = -1, m1 = -1, p0 = -1, p1 = -1;
        if (x == seg0 && s_cur == s_win) {            // warp-uniform
          trow = s_trow;
          w0 = sw0;
          w1 = sw1;
          n0 = sn0;
          n1 = sn1;
          if constexpr (BS == 1) {
            m0 = sm0;
            m1 = sm1;
            p0 = sp0;
            p1 = sp1;
          }
        } else {
          // a chunk of a prefix launch reads the prefix through its first member's table
          const long long trow_seq =
              MODE == kPrefix ? (long long)chunk_member(a, s_cur, 0) : s_cur;
          trow = a.block_tables + trow_seq * a.max_blocks;
          w0 = wb + lane < nblk ? trow[wb + lane] : -1;
          w1 = wb + 32 + lane < nblk ? trow[wb + 32 + lane] : -1;
          n0 = wb + 64 + lane < nblk ? trow[wb + 64 + lane] : -1;
          n1 = wb + 96 + lane < nblk ? trow[wb + 96 + lane] : -1;
          if constexpr (BS == 1) {
            m0 = wb + 128 + lane < nblk ? trow[wb + 128 + lane] : -1;
            m1 = wb + 160 + lane < nblk ? trow[wb + 160 + lane] : -1;
            p0 = wb + 192 + lane < nblk ? trow[wb + 192 + lane] : -1;
            p1 = wb + 224 + lane < nblk ? trow[wb + 224 + lane] : -1;
          }
          if (x == seg0) {
            s_win = s_cur;
            s_trow = trow;
            sw0 = w0;
            sw1 = w1;
            sn0 = n0;
            sn1 = n1;
            if constexpr (BS == 1) {
              sm0 = m0;
              sm1 = m1;
              sp0 = p0;
              sp1 = p1;
            }
          }
        }
        for (long long tu = x; tu < pe; tu += kUnitsPerStage) {
          const int nun = (int)((pe - tu) < kUnitsPerStage ? (pe - tu) : kUnitsPerStage);
          const int tok0 = first_cur + (int)(tu - seg0) * kUnit;
          if (tok0 / BS >= wb + 64) {                 // warp-uniform: slide the window
            w0 = n0;
            w1 = n1;
            wb += 64;
            if constexpr (BS == 1) {
              n0 = m0;
              n1 = m1;
              m0 = p0;
              m1 = p1;
              p0 = wb + 192 + lane < nblk ? trow[wb + 192 + lane] : -1;
              p1 = wb + 224 + lane < nblk ? trow[wb + 224 + lane] : -1;
            } else {
              n0 = wb + 64 + lane < nblk ? trow[wb + 64 + lane] : -1;
              n1 = wb + 96 + lane < nblk ? trow[wb + 96 + lane] : -1;
            }
          }
          const int flags = (tu == x ? F_FIRST : 0) | (tu + kUnitsPerStage >= pe ? F_LAST : 0) |
                            (complete ? F_COMPLETE : 0) |
                            (MODE == kSuffix && first_cur > 0 ? F_PREFIX : 0);
          // the query rows of this kv head: group consecutive heads of each new token,
          // one bulk copy per token, stored as columns c = token * group + head
          const uint32_t qrow_bytes = (uint32_t)(group * D * 2);
          const uint32_t qbytes = (flags & F_FIRST) ? qrow_bytes * (uint32_t)a.q_len : 0u;
          const T* qsrc = static_cast<const T*>(a.q) +
                          ((long long)s_cur * a.q_len * a.num_q_heads + (long long)kvh * group) * D;
          // source of query-row token jq (in a prefix launch: the chunk's jq-th member; a
          // padding slot repeats the first member's rows and its results are dropped)
          auto qrow_src = [&](int jq) -> const T* {
            if constexpr (MODE == kPrefix) {
              int mem = chunk_member(a, s_cur, jq);
              if (mem < 0) mem = (int)((trow - a.block_tables) / a.max_blocks);   // first member
              return static_cast<const T*>(a.q) +
                     ((long long)mem * a.num_q_heads + (long long)kvh * group) * D;
            } else {
              return qsrc + (long long)jq * a.num_q_heads * D;
            }
          };
          // fused append: the stage holding a segment's newest token (position ctx-1)
          // stages that token's K/V rows from k_new/v_new; its consumer patches them into
          // the tile and writes them to the cache row found here
          int newrow = -1;
          if (MODE == kAppend && tok0 <= ctx_cur - 1 &&
              ctx_cur - 1 < tok0 + nun * kUnit) {      // warp-uniform
            const int tn = ctx_cur - 1;
            int blk_n;
            if constexpr (BS != 1) {
              const int wi = tn / BS - wb;
              if ((tok0 + kTileTokens - 1) / BS >= wb + 64)
                blk_n = win_lookup(w0, w1, n0, wi);
              else
                blk_n = win_lookup(w0, w1, w1, wi);
            } else {
              const int r = tn - tok0;
              blk_n = __shfl_sync(0xffffffffu, r >= 32 ? w1 : w0, r & 31);
            }
            if ((unsigned)blk_n < (unsigned)a.num_blocks) newrow = (blk_n * Hkv + kvh) * BS + tn % BS;
          }
          const uint32_t nbytes = newrow >= 0 ? (uint32_t)L::kNewBytes : 0u;
          auto stage_new = [&](uint64_t* bar) {       // lane 0: the two staged rows
            uint8_t* dst = smem + L::kNewOff + st * L::kNewBytes;
            const long long src = ((long long)s_cur * Hkv + kvh) * D;
            bulk_load(dst, static_cast<const T*>(a.k_new) + src, D * 2, bar);
            bulk_load(dst + D * 2, static_cast<const T*>(a.v_new) + src, D * 2, bar);
          };
          if constexpr (BS != 1) {
            constexpr int H = BS < 16 ? BS : 16;     // rows per TMA box
            constexpr int BPU = kUnit / H;           // boxes per unit and column half
            constexpr int kParts = KV8 ? 1 : L::kHalves;   // boxes per row of a token
            constexpr int kRowB = KV8 ? D : 128;     // tile bytes per row and box
            constexpr int kBoxBytes = H * kRowB;     // D 8-bit values or 64 16-bit
            static_assert(kUnitsPerStage * BPU * kParts * 2 <= 32, "one box per lane");
            // this lane's box and its block-table entry, read before the slot wait
            const int nbox = nun * BPU * kParts * 2;
            const int kv = lane & 1;
            const int hf = (lane >> 1) % kParts;
            const int jb = (lane >> 1) / kParts;
            const int j = jb / BPU, b = jb % BPU;
            const int t = tok0 + j * kUnit + b * H;
            const bool mine = lane < nbox && t < ctx_cur;
            // the stage spans blocks tok0/BS .. +64/BS-1 < wb + 72: w0, w1 and, only when it
            // runs past the window, n0 (whose load was issued 64 blocks ago)
            const int wi = mine ? t / BS - wb : 0;
            int blk;
            if ((tok0 + kTileTokens - 1) / BS >= wb + 64)   // warp-uniform
              blk = win_lookup(w0, w1, n0, wi);
            else
              blk = win_lookup(w0, w1, w1, wi);       // never touches n0 while it loads
            int y = 0;
            float scv = 0.f;                           // KSC: this box's block scale
            if (mine) {
              if ((unsigned)blk < (unsigned)a.num_blocks) {
                y = (blk * Hkv + kvh) * BS + (t % BS);
                if constexpr (KSC) scv = __ldg((kv ? a.v_bscale : a.k_bscale) + blk * Hkv + kvh);
              } else {
                if (a.status) atomicOr(a.status, DEV_BAD_BLOCK_ID);
                y = rows_total;                        // out of range: TMA fills zeros
              }
            }
            uint32_t bytes = qbytes + nbytes;
            for (int jj = 0; jj < nun; ++jj) {
              const int rem = ctx_cur - (tok0 + jj * kUnit);
              const int nb = (rem + H - 1) / H;
              bytes += (uint32_t)((nb < BPU ? nb : BPU) * kBoxBytes * kParts * 2);
            }
            if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, kWaitLimitNs)) {
              ok = false;
              break;
            }
            uint8_t* sK = smem + st * L::kStageBytes;
            uint8_t* sV = sK + L::kKvBytes;
            uint8_t* sQ = sV + L::kKvBytes;
            if constexpr (KSC) {
              // every row's K / V scale: box lane (kv, j, b) covers rows j*16 + b*H .. +H-1
              // of pool kv (0 for rows past the valid tokens)
              if (lane < kUnitsPerStage * BPU * 2) {
                float* sc = reinterpret_cast<float*>(smem + L::kScOff + st * L::kScBytes) +
                            kv * kTileTokens + j * kUnit + b * H;
#pragma unroll
                for (int rr = 0; rr < H; ++rr) sc[rr] = scv;
              }
              __syncwarp();
            }
            if (lane == 0) {
              meta[st] = StageMeta{s_cur, kvh, tok0, nun, ctx_cur, flags, pidx, qslot, newrow};
              mbar_arrive_expect_tx(&full[st], bytes);
              if (qbytes)
                for (int jq = 0; jq < a.q_len; ++jq)
                  bulk_load(sQ + jq * qrow_bytes, qrow_src(jq), qrow_bytes, &full[st]);
              if (nbytes) stage_new(&full[st]);
            }
            __syncwarp();
            if (mine) {
              uint8_t* dst = (kv ? sV : sK) + hf * (kTileTokens * 128) + (j * kUnit + b * H) * kRowB;
              tma_load_2d(dst, kv ? &tmv : &tmk, &full[st], KV8 ? 0 : hf * 64, y, policy);
            }
          } else {
            // block_size 1: every token is its own block.  The rows come in by TMA
            // gather4 loads, four rows of 128 bytes each (a column half of a 16-bit row, or
            // a whole 8-bit row) from four table entries, into the same 128-byte-swizzled
            // tile rows the box loads produce (the swizzle follows the shared-memory address,
            // and each load's four rows are consecutive 128-byte lines).  Sixteen-byte
            // cp.async copies, one warp issuing them all, were limited to ~0.4 of HBM
            // bandwidth here.  Stages are 64 tokens, so the window (w0, w1) holds exactly
            // this stage's table entries, handed out by shuffle.
            constexpr int kParts = kGParts, kPieceB = kGPieceB;
            const int ntok = nun * kUnit;
            // KSC: the K / V scales of rows lane and 32+lane (this stage's table entries
            // are w0, w1), read before the slot wait
            float sck0 = 0.f, sck1 = 0.f, scv0 = 0.f, scv1 = 0.f;
            if constexpr (KSC) {
              const int nv = ntok < ctx_cur - tok0 ? ntok : ctx_cur - tok0;
              if (lane < nv && (unsigned)w0 < (unsigned)a.num_blocks) {
                sck0 = __ldg(a.k_bscale + w0 * Hkv + kvh);
                scv0 = __ldg(a.v_bscale + w0 * Hkv + kvh);
              }
              if (32 + lane < nv && (unsigned)w1 < (unsigned)a.num_blocks) {
                sck1 = __ldg(a.k_bscale + w1 * Hkv + kvh);
                scv1 = __ldg(a.v_bscale + w1 * Hkv + kvh);
              }
            }
            if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, kWaitLimitNs)) {
              ok = false;
              break;
            }
            uint8_t* sK = smem + st * L::kStageBytes;
            uint8_t* sV = sK + L::kKvBytes;
            uint8_t* sQ = sV + L::kKvBytes;
            if constexpr (KSC) {
              float* sc = reinterpret_cast<float*>(smem + L::kScOff + st * L::kScBytes);
              sc[lane] = sck0;
              sc[32 + lane] = sck1;
              sc[kTileTokens + lane] = scv0;
              sc[kTileTokens + 32 + lane] = scv1;
              __syncwarp();
            }
            // load items: (group of 4 rows g, piece hf, pool kv), at most 16 * 2 * 2 = 64,
            // two a lane; rows past the valid tokens (or with a bad block id) read row
            // rows_total, out of range, which the TMA fills with zeros
            const int nvalid = ntok < ctx_cur - tok0 ? ntok : ctx_cur - tok0;
            const int nitems = ((nvalid + 3) >> 2) * kParts * 2;
            static_assert(kTileTokens / 4 * kParts * 2 <= 64, "two load items a lane");
            if (lane == 0) {
              meta[st] = StageMeta{s_cur, kvh, tok0, nun, ctx_cur, flags, pidx, qslot, newrow};
              mbar_arrive_expect_tx(&full[st], qbytes + nbytes + (uint32_t)nitems * (4u * kPieceB));
              if (qbytes)
                for (int jq = 0; jq < a.q_len; ++jq)
                  bulk_load(sQ + jq * qrow_bytes, qrow_src(jq), qrow_bytes, &full[st]);
              if (nbytes) stage_new(&full[st]);
            }
            // every row's coordinate (rows lane and 32+lane), published for the helper warp
            int* yc = ycoord + st * kTileTokens;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int r = h * 32 + lane, blk = h ? w1 : w0;
              int y = rows_total;
              if (r < nvalid) {
                if ((unsigned)blk < (unsigned)a.num_blocks) y = blk * Hkv + kvh;
                else if (a.status) atomicOr(a.status, DEV_BAD_BLOCK_ID);
              }
              yc[r] = y;
            }
            __syncwarp();
            if (lane == 0) {
              ymark[st] = (nvalid + 3) >> 2;
              mbar_arrive(&yready[st]);                 // releases the coordinates
            }
            ++nfill;
            // the K gathers: (group of 4 rows g, piece hf), one a lane
            static_assert(kTileTokens / 4 * kParts <= 32, "one K load item a lane");
            if (lane < nitems / 2) {
              const int hf = lane % kParts, g = lane / kParts;
              tma_gather4(sK + hf * (kTileTokens * 128) + g * 4 * kPieceB, &tmk, &full[st], hf * 64,
                          yc[4 * g], yc[4 * g + 1], yc[4 * g + 2], yc[4 * g + 3], policy);
            }
          }
          if (++st == kStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        x = pe == seg1 ? seg0 + w_cur : pe;          // past the virtual tail
      }
    }
    if (ok) ok = mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, kWaitLimitNs);
    if (ok) {
      if (lane == 0) meta[st].flags = F_END;
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[st]);
      if constexpr (BS == 1) {
        // the V-gather warp waits for the next fill of every slot: one more arrival on each
        // slot's barrier, with no groups, tells it there is none.  It must have taken every
        // earlier arrival first (two phases completing before its wait would read as none,
        // and the group count would be overwritten), which its count shows.
        bool seen = true;
        if (lane == 0) seen = wait_count_bounded(yseen, nfill, abort_flag, kWaitLimitNs);
        seen = __shfl_sync(0xffffffffu, seen, 0);
        if (seen && lane < kStages) {
          ymark[lane] = 0;
          mbar_arrive(&yready[lane]);
        }
        if (!seen && lane == 0) {
          *abort_flag = 1;
          if (a.status) atomicOr(a.status, DEV_TIMEOUT);
        }
      }
    } else {
      if (lane == 0) {
        *abort_flag = 1;
        if (a.status) atomicOr(a.status, DEV_TIMEOUT);
      }
    }
    if (late_wait) pdl_wait();
    return;
  }

  // ============================== consumers ==============================
  const int cw = warp - 1;
  const int gid = lane >> 2, tig = lane & 3;
  const int tid = cw * 32 + lane;
  constexpr int KS = D / 16;            // k-steps of QK, m-tiles of PV
  // With 16 query columns (NT = 2) a warp holding both n-tiles of O and q runs out of
  // registers (spills in the unit loop), so the warps of a pair split the columns: warp
  // cw takes n-tile cw & 1 of units 2 (cw >> 1) and 2 (cw >> 1) + 1 of every stage.
  constexpr bool kColSplit = NT == 2;
  constexpr int NTW = kColSplit ? 1 : NT;       // n-tiles a warp holds
  constexpr int UPW = kColSplit ? 2 : 1;        // units a warp takes per stage
  const int nb = kColSplit ? (cw & 1) : 0;      // its first n-tile
  constexpr int NREGW = KS * NTW * 4;           // O^T accumulator registers a thread holds
  // the end-of-portion merge stages every warp's O in the stage's K and V tiles
  static_assert(kConsumerWarps * NREGW * 32 * 4 <= 2 * L::kKvBytes,
                "merge scratch must fit in the stage's K and V tiles");
  float o[KS][NTW][4];
  float m[NTW][2], l[NTW][2];
  uint32_t qf[KS][NTW][2];
#pragma unroll
  for (int i = 0; i < KS; ++i)
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
      qf[i][n][0] = qf[i][n][1] = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[i][n][e] = 0.f;
    }
#pragma unroll
  for (int n = 0; n < NTW; ++n) m[n][0] = m[n][1] = -INFINITY, l[n][0] = l[n][1] = 0.f;
  // new-token index of this lane's two accumulator columns per n-tile
  int jcol[NTW][2];
#pragma unroll
  for (int n = 0; n < NTW; ++n) {
    jcol[n][0] = ((nb + n) * 8 + 2 * tig) / group;
    jcol[n][1] = ((nb + n) * 8 + 2 * tig + 1) / group;
  }

  // block size 1, warp kHelperWarp: take the next fill of slot s (the producer's arrival
  // of parity par on yready[s]) and issue its V gathers, one (group of 4 rows, piece) a
  // lane, into the slot's V tile; false when the wait gave up
  [[maybe_unused]] auto take_fill = [&](int s, uint32_t par) -> bool {
    if (!mbar_wait_bounded(&yready[s], par, abort_flag, kWaitLimitNs)) return false;
    const int ngrp = __shfl_sync(0xffffffffu, lane == 0 ? ymark[s] : 0, 0);
    if (lane == 0) {
      __threadfence_block();                        // the count is read before it is taken
      *yseen = *yseen + 1;
    }
    if (lane < ngrp * kGParts) {
      const int hf = lane % kGParts, g = lane / kGParts;
      const int* yc = ycoord + s * kTileTokens + 4 * g;
      uint8_t* sV = smem + s * L::kStageBytes + L::kKvBytes;
      tma_gather4(sV + hf * (kTileTokens * 128) + g * 4 * kGPieceB, &tmv, &full[s], hf * 64,
                  yc[0], yc[1], yc[2], yc[3], policy_evict_first());
    }
    return true;
  };
  // a failed wait leaves this warp in the loop (the others may reach a named barrier with
  // it); the abort flag ends every later wait
  auto helper_abort = [&]() {
    if (lane == 0) {
      *abort_flag = 1;
      if (a.status) atomicOr(a.status, DEV_TIMEOUT);
    }
  };
  if constexpr (BS == 1) {
    if (cw == kHelperWarp) {
      bool okh = true;
      for (int s = 0; s < kStages && okh; ++s) okh = take_fill(s, 0u);
      if (!okh) helper_abort();
    }
  }

  int st = 0;
  uint32_t ph = 0;
  for (;;) {
    if (!mbar_wait_bounded(&full[st], ph, abort_flag, kWaitLimitNs)) {
      if (lane == 0) {
        *abort_flag = 1;
        if (a.status) atomicOr(a.status, DEV_TIMEOUT);
      }
      break;
    }
    const StageMeta mt = meta[st];
    if (mt.flags & F_END) break;
    uint8_t* sK = smem + st * L::kStageBytes;
    uint8_t* sV = sK + L::kKvBytes;
    const uint8_t* sQ = sV + L::kKvBytes;
    if (mt.flags & F_FIRST) {
#pragma unroll
      for (int n = 0; n < NTW; ++n) {
        const int cq = (nb + n) * 8 + gid;           // this lane's query column
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0 = 0u, b1 = 0u;
          if (cq < a.ncol) {
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(sQ + cq * D * 2);
            if constexpr (KV8) {
              // k-step ks pairs with the 16 cache bytes of dims 16ks..16ks+15 as the
              // converted fragments order them: logical k (2c, 2c+1) is dims (4c, 4c+1),
              // logical k (2c+8, 2c+9) is dims (4c+2, 4c+3); q converted to fp16
              const uint32_t u0 = qrow[(ks * 16 + 4 * tig) >> 1];
              const uint32_t u1 = qrow[(ks * 16 + 4 * tig + 2) >> 1];
              const float2 f0 = unpack2<T>(u0), f1 = unpack2<T>(u1);
              b0 = pack2<__half>(f0.x, f0.y);
              b1 = pack2<__half>(f1.x, f1.y);
            } else {
              b0 = qrow[(ks * 16 + 2 * tig) >> 1];
              b1 = qrow[(ks * 16 + 8 + 2 * tig) >> 1];
            }
          }
          qf[ks][n][0] = b0;
          qf[ks][n][1] = b1;
#pragma unroll
          for (int e = 0; e < 4; ++e) o[ks][n][e] = 0.f;
        }
        m[n][0] = m[n][1] = -INFINITY;
        l[n][0] = l[n][1] = 0.f;
      }
    }
    bool patched = false;
#pragma unroll 1
    for (int uk = 0; uk < UPW; ++uk) {
      const int u = kColSplit ? (cw >> 1) * 2 + uk : cw;   // unit of the stage
      if (u < mt.nunits) {
        const int t0 = mt.tok0 + u * kUnit;
        const int valid = (mt.ctx - t0) < kUnit ? (mt.ctx - t0) : kUnit;
        // causal limit: new token j sees unit rows < ctx - q_len + 1 + j - t0 (a prefix
        // launch's columns are different sequences: no mask)
        const int lim0 = MODE == kPrefix ? (1 << 30) : mt.ctx - a.q_len + 1 - t0;
        if (MODE == kAppend && KV8 && mt.newrow >= 0 && (mt.ctx - 1 - mt.tok0) / kUnit == u) {
          // fused append into 8-bit pools with per-(block, kv head) scales: D/16 lanes
          // quantise the new K row and as many the V row, 16 values (one 16-byte chunk of
          // codes) each, exactly as the block-scaled append does; a token at offset 0 of its
          // block first fixes the block's scale from its own row.  The codes go into the tile
          // row and the cache row, the scale into the stage's scale row and, for offset 0,
          // the scale array.  With split columns both warps compute the same bytes; the
          // first writes global memory.
          constexpr int CPR8 = D / 16;                  // 16-byte chunks of codes per row
          const int rn = mt.ctx - 1 - mt.tok0;          // row in the stage tile
          const int kv = (lane / CPR8) & 1, ch = lane % CPR8;
          const bool act = lane < 2 * CPR8;
          const uint4* src = reinterpret_cast<const uint4*>(smem + L::kNewOff + st * L::kNewBytes +
                                                            kv * D * 2 + ch * 32);
          uint4 in[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
          if (act) {
            in[0] = src[0];
            in[1] = src[1];
          }
          const uint32_t* w = reinterpret_cast<const uint32_t*>(in);
          float x[16];
          float am = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 f = unpack2<T>(w[e]);
            x[2 * e] = f.x;
            x[2 * e + 1] = f.y;
            am = fmaxf(am, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
#pragma unroll
          for (int o = 1; o < CPR8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
          float* scs = reinterpret_cast<float*>(smem + L::kScOff + st * L::kScBytes) + kv * kTileTokens;
          const bool fresh = mt.newrow % BS == 0;       // offset 0: this token fixes the scale
          const float sc = fresh ? e4m3_block_scale(am) : scs[rn];
          __syncwarp();
          if (act) {
            uint32_t q[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              q[e] = f32x2_to_e4m3x2(__fdiv_rn(x[4 * e], sc), __fdiv_rn(x[4 * e + 1], sc)) |
                     (f32x2_to_e4m3x2(__fdiv_rn(x[4 * e + 2], sc), __fdiv_rn(x[4 * e + 3], sc)) << 16);
            const uint4 codes = make_uint4(q[0], q[1], q[2], q[3]);
            *reinterpret_cast<uint4*>((kv ? sV : sK) + rn * D + ((ch ^ kv8_swz<D>(rn)) << 4)) = codes;
            if (ch == 0 && fresh) scs[rn] = sc;
            if (nb == 0) {
              uint8_t* cache = static_cast<uint8_t*>(const_cast<void*>(kv ? a.v_cache : a.k_cache));
              *reinterpret_cast<uint4*>(cache + (long long)mt.newrow * D + ch * 16) = codes;
              if (ch == 0 && fresh)
                const_cast<float*>(kv ? a.v_bscale : a.k_bscale)[mt.newrow / BS] = sc;
            }
          }
          __syncwarp();
          patched = true;
        } else if (MODE == kAppend && !KV8 && mt.newrow >= 0 && (mt.ctx - 1 - mt.tok0) / kUnit == u) {
          // fused append: this unit holds the newest token; its K/V rows come from the
          // staging area (the cache row the TMA read may still be old) and are written to
          // the cache.  With split columns both warps of the unit patch their tile copy
          // with the same bytes before reading it; the first writes the cache row.
          constexpr int CPR = D * 2 / 16;               // 16-byte chunks per row
          const int rn = mt.ctx - 1 - mt.tok0;          // row in the stage tile
          if (lane < 2 * CPR) {
            const int kv = lane / CPR, ch = lane % CPR, hf = ch >> 3, cc = ch & 7;
            const uint4 val = *reinterpret_cast<const uint4*>(smem + L::kNewOff + st * L::kNewBytes +
                                                              kv * D * 2 + ch * 16);
            *reinterpret_cast<uint4*>((kv ? sV : sK) + hf * (kTileTokens * 128) + rn * 128 +
                                      ((cc ^ (rn & 7)) << 4)) = val;
            if (nb == 0) {
              T* cache = static_cast<T*>(const_cast<void*>(kv ? a.v_cache : a.k_cache));
              *reinterpret_cast<uint4*>(cache + (long long)mt.newrow * D + ch * 8) = val;
            }
          }
          __syncwarp();
          patched = true;
        }
        const uint32_t kbase = smem_u32(sK), vbase = smem_u32(sV);
        // ---- S^T[16 tokens][8*NT heads] = K_unit . q^T
        float sacc[NTW][4];
#pragma unroll
        for (int n = 0; n < NTW; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
        if constexpr (KV8) {
          // one ldmatrix.x4 = rows 0-7 / 8-15 of two 16-byte chunks (k-steps ks, ks+1); a
          // thread's 32 bits are 4 codes, dims 4c..4c+3 of its row, converted in two halves
          const int j = lane >> 3, i = lane & 7;
          const int r = u * kUnit + (j & 1) * 8 + i;
#pragma unroll
          for (int ks = 0; ks < KS; ks += 2) {
            const int chunk = ks + (j >> 1);
            const uint32_t addr = kbase + r * D + ((chunk ^ kv8_swz<D>(r)) << 4);
            uint32_t m0, m1, m2, m3;
            ldsm_x4(addr, m0, m1, m2, m3);
            uint32_t x0, x1, x2, x3, y0, y1, y2, y3;
            e4m3x4_to_f16x2x2(m0, x0, x2);
            e4m3x4_to_f16x2x2(m1, x1, x3);
            e4m3x4_to_f16x2x2(m2, y0, y2);
            e4m3x4_to_f16x2x2(m3, y1, y3);
#pragma unroll
            for (int n = 0; n < NTW; ++n) {
              mma16816<false>(sacc[n], x0, x1, x2, x3, qf[ks][n][0], qf[ks][n][1]);
              mma16816<false>(sacc[n], y0, y1, y2, y3, qf[ks + 1][n][0], qf[ks + 1][n][1]);
            }
          }
        } else {
          const int j = lane >> 3, i = lane & 7;
          const int r = u * kUnit + (j & 1) * 8 + i;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const int d = ks * 16 + (j >> 1) * 8;
            const uint32_t addr =
                kbase + (d >> 6) * (kTileTokens * 128) + r * 128 + ((((d & 63) >> 3) ^ (r & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(addr, a0, a1, a2, a3);
#pragma unroll
            for (int n = 0; n < NTW; ++n) mma16816<kBF16>(sacc[n], a0, a1, a2, a3, qf[ks][n][0], qf[ks][n][1]);
          }
        }
        // ---- online softmax (base 2) per query column
        // KSC: this lane's two rows (gid, gid + 8) carry their blocks' K scales into the
        // scores and their V scales into P (the row sums keep the unscaled weights)
        float sl_lo = a.scale_log2, sl_hi = a.scale_log2, vs_lo = 1.f, vs_hi = 1.f;
        if constexpr (KSC) {
          const float* sc = reinterpret_cast<const float*>(smem + L::kScOff + st * L::kScBytes);
          const int r0 = u * kUnit + gid;
          sl_lo = a.scale_log2 * sc[r0];
          sl_hi = a.scale_log2 * sc[r0 + 8];
          // a row past the valid tokens has p = 0; its scale may be that of a block whose
          // offset 0 was never written (anything, NaN included), so it must not reach P
          vs_lo = gid < valid ? sc[kTileTokens + r0] : 0.f;
          vs_hi = gid + 8 < valid ? sc[kTileTokens + r0 + 8] : 0.f;
        }
        uint32_t bhi[NTW][2], blo[NTW][2];
#pragma unroll
        for (int n = 0; n < NTW; ++n) {
          float xs[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = gid + (e >= 2 ? 8 : 0);
            const int lim = lim0 + jcol[n][e & 1];
            xs[e] = (row < valid && row < lim) ? sacc[n][e] * (e >= 2 ? sl_hi : sl_lo) : -INFINITY;
          }
          float alpha[2], p[4];
          bool grew = false;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float mx = fmaxf(xs[cc], xs[cc + 2]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mnew = fmaxf(m[n][cc], mx);
            // a column with no visible row yet keeps max -inf: use 0 as the reference
            const float mref = mnew == -INFINITY ? 0.f : mnew;
            grew |= mnew != m[n][cc];
            alpha[cc] = ex2(m[n][cc] - mref);
            m[n][cc] = mnew;
            p[cc] = ex2(xs[cc] - mref);
            p[cc + 2] = ex2(xs[cc + 2] - mref);
            l[n][cc] = l[n][cc] * alpha[cc] + p[cc] + p[cc + 2];
          }
          // 8-bit caches (ALU-bound): rescale O only when a column's running max moved in
          // this warp (alpha is exactly 1 otherwise)
          if (!KV8 || __any_sync(0xffffffffu, grew)) {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              o[ks][n][0] *= alpha[0];
              o[ks][n][1] *= alpha[1];
              o[ks][n][2] *= alpha[0];
              o[ks][n][3] *= alpha[1];
            }
          }
          using TM = std::conditional_t<KV8, __half, T>;   // MMA operand type
          const uint32_t h01 = pack2<TM>(p[0] * vs_lo, p[1] * vs_lo);
          const uint32_t h23 = pack2<TM>(p[2] * vs_hi, p[3] * vs_hi);
          bhi[n][0] = movmatrix_t(h01);
          bhi[n][1] = movmatrix_t(h23);
          if constexpr (!KV8) {
            // the rounding residual of P as a second 16-bit operand (~16 bits of P in all)
            const float2 f01 = unpack2<TM>(h01), f23 = unpack2<TM>(h23);
            const uint32_t l01 = pack2<TM>(p[0] - f01.x, p[1] - f01.y);
            const uint32_t l23 = pack2<TM>(p[2] - f23.x, p[3] - f23.y);
            blo[n][0] = movmatrix_t(l01);
            blo[n][1] = movmatrix_t(l23);
          } else {
            blo[n][0] = blo[n][1] = 0u;   // fp16 P: 11 bits, next to 3-bit cache values
          }
        }
        // ---- O^T[D][8*NT] += V_unit^T . P^T
        uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;   // token masks for V rows >= valid
        if (valid < kUnit) {
          const int t_a = 2 * tig, t_b = 8 + 2 * tig;
          mlo = (t_a < valid ? 0x0000ffffu : 0u) | (t_a + 1 < valid ? 0xffff0000u : 0u);
          mhi = (t_b < valid ? 0x0000ffffu : 0u) | (t_b + 1 < valid ? 0xffff0000u : 0u);
        }
        // the PV product; with 8-bit caches (ALU-bound) the token masks are applied only to
        // a unit with fewer than 16 valid rows (a lambda instantiated with and without them)
        auto pv = [&](auto masked) {
          if constexpr (KV8) {
            // ldmatrix.x4.trans of tokens 0-7 / 8-15 of two 16-byte chunks; a thread gets the
            // codes of dims (2g, 2g+1) for tokens (2c, 2c+1): regrouped per dim they give the
            // A fragments with M-row g = dim 2g and M-row g+8 = dim 2g+1 of the chunk
            const int j = lane >> 3, i = lane & 7;
            const int r = u * kUnit + (j & 1) * 8 + i;
#pragma unroll
            for (int mtile = 0; mtile < KS; mtile += 2) {
              const int chunk = mtile + (j >> 1);
              const uint32_t addr = vbase + r * D + ((chunk ^ kv8_swz<D>(r)) << 4);
              uint32_t m[4];
              ldsm_x4_t(addr, m[0], m[1], m[2], m[3]);
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const uint32_t p0 = __byte_perm(m[2 * hh], 0u, 0x3120);       // tokens 2c, 2c+1
                const uint32_t p1 = __byte_perm(m[2 * hh + 1], 0u, 0x3120);   // tokens 8+2c, ...
                uint32_t a0, a1, a2, a3;
                e4m3x4_to_f16x2x2(p0, a0, a1);
                e4m3x4_to_f16x2x2(p1, a2, a3);
                if constexpr (decltype(masked)::value) {
                  a0 &= mlo;
                  a1 &= mlo;
                  a2 &= mhi;
                  a3 &= mhi;
                }
#pragma unroll
                for (int n = 0; n < NTW; ++n)
                  mma16816<false>(o[mtile + hh][n], a0, a1, a2, a3, bhi[n][0], bhi[n][1]);
              }
            }
          } else {
            const int j = lane >> 3, i = lane & 7;
            const int r = u * kUnit + (j >> 1) * 8 + i;
#pragma unroll
            for (int mtile = 0; mtile < KS; ++mtile) {
              const int d = mtile * 16 + (j & 1) * 8;
              const uint32_t addr =
                  vbase + (d >> 6) * (kTileTokens * 128) + r * 128 + ((((d & 63) >> 3) ^ (r & 7)) << 4);
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(addr, a0, a1, a2, a3);
              if constexpr (decltype(masked)::value) {
                a0 &= mlo;
                a1 &= mlo;
                a2 &= mhi;
                a3 &= mhi;
              }
#pragma unroll
              for (int n = 0; n < NTW; ++n) {
                mma16816<kBF16>(o[mtile][n], a0, a1, a2, a3, bhi[n][0], bhi[n][1]);
                mma16816<kBF16>(o[mtile][n], a0, a1, a2, a3, blo[n][0], blo[n][1]);
              }
            }
          }
        };
        if constexpr (KV8) {
          if (valid < kUnit) pv(std::true_type{});
          else pv(std::false_type{});
        } else {
          pv(std::true_type{});
        }
      }
    }
    if (mt.flags & F_LAST) {
      if (late_wait) pdl_wait();                 // the prefix partials are complete
      // ---- merge the four warps' (m, l, O) for this segment portion
#pragma unroll
      for (int n = 0; n < NTW; ++n)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float v = l[n][cc];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          l[n][cc] = v;
        }
      named_bar_sync(1, kConsumerThreads);         // all warps are done with this stage's K/V
      float* scr = reinterpret_cast<float*>(sK);   // K and V tiles reused as scratch
      // every warp stores the n-tiles it holds; its (max, sum) of a column it does not
      // hold is empty (-inf, 0)
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int n = 0; n < NTW; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            scr[(cw * NREGW + (ks * NTW + n) * 4 + e) * 32 + lane] = o[ks][n][e];
      if (gid == 0) {
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int w = n - nb;
            mls[cw * kMaxGroup + n * 8 + 2 * tig + cc] =
                (w >= 0 && w < NTW) ? make_float2(m[w < NTW ? w : 0][cc], l[w < NTW ? w : 0][cc])
                                    : make_float2(-INFINITY, 0.f);
          }
      }
      named_bar_sync(1, kConsumerThreads);
      const bool complete = mt.flags & F_COMPLETE;
      const bool has_prefix = MODE == kSuffix && complete && (mt.flags & F_PREFIX);
      // Thread tid of warp cw combines accumulator register e = cw of every (ks, n) tile of
      // lane `lane` over the warps holding n-tile n: query column h_n = n*8 + 2*(lane%4) +
      // cw%2 and head dim d = ks*16 + lane/4 + 8*(cw/2).  So the column statistics (max,
      // weights, sum) are computed once per n, and the loop over the dims only sums and
      // stores.
      constexpr int kIt = KS * NT;                  // accumulator values per thread
      static_assert(kConsumerWarps == 4, "register e of a tile is combined by warp e");
      float cM[NT], cL[NT], cs[NT][kConsumerWarps];
      long long crow[NT];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int h = n * 8 + 2 * (lane & 3) + (cw & 1);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mls[w * kMaxGroup + h].x);
        float Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float2 ml = mls[w * kMaxGroup + h];
          cs[n][w] = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);
          Ls += ml.y * cs[n][w];
        }
        cM[n] = M;
        cL[n] = Ls;
        crow[n] = (complete && h < a.ncol) ? out_row<MODE>(a, mt.seq, mt.kvh, h) : -1ll;
      }
      float2 xm[NT];
      float xv[kIt];
#pragma unroll
      for (int n = 0; n < NT; ++n)
        xm[n] = (MODE == kSuffix && has_prefix && crow[n] >= 0) ? __ldcg(a.ext_ml + crow[n])
                                                                 : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int it = 0; it < kIt; ++it) {            // the prefix partials, all loads at once
        const int n = it % NT, ks = it / NT;
        const int d = ks * 16 + (KV8 ? 2 * (lane >> 2) + (cw >= 2 ? 1 : 0)
                                     : (lane >> 2) + (cw >= 2 ? 8 : 0));
        xv[it] = (MODE == kSuffix && has_prefix && crow[n] >= 0) ? __ldcg(a.ext_acc + crow[n] * D + d)
                                                                  : 0.f;
      }
#pragma unroll
      for (int it = 0; it < kIt; ++it) {
        const int n = it % NT, ks = it / NT;
        const int h = n * 8 + 2 * (lane & 3) + (cw & 1);   // query column
        if (h >= a.ncol) continue;
        // head dim of this accumulator value (8-bit caches order the PV rows 2g, 2g+1)
        const int d = ks * 16 + (KV8 ? 2 * (lane >> 2) + (cw >= 2 ? 1 : 0)
                                     : (lane >> 2) + (cw >= 2 ? 8 : 0));
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const int nl = n - (kColSplit ? (w & 1) : 0);    // n-tile n in warp w's registers
          if (nl >= 0 && nl < NTW)
            acc += scr[(w * NREGW + (ks * NTW + nl) * 4 + cw) * 32 + lane] * cs[n][w];
        }
        if (complete) {
          // column h = new token (or chunk member) h / group, head kvh * group + h % group;
          // a row that sees no token at all (a new token before the context start) is zero
          if (crow[n] >= 0)
            finish_row<T, MODE, D>(a, crow[n], cM[n], cL[n], &acc, d, 1, xm[n], &xv[it]);
        } else {
          a.part_acc[((long long)mt.pidx * kMaxGroup + h) * D + d] = acc;
          if (d == 0) {
            a.part_ml[((long long)mt.pidx * kMaxGroup + h) * 2 + 0] = cM[n];
            a.part_ml[((long long)mt.pidx * kMaxGroup + h) * 2 + 1] = cL[n];
          }
        }
      }
      if (!complete) {
        // ---- arrival on the segment's counter: bar.sync orders every thread's partial
        // stores before thread 0's release at GPU scope; its acquire orders the other
        // CTAs' partials before the reads below (they load through L2, bypassing L1).
        named_bar_sync(1, kConsumerThreads);
        const SplitDesc dsc = desc[mt.qslot];
        if (tid == 0) {
          // One round trip in the usual case: the last arrival resets the counter to 0,
          // and the first CTA of a segment (whose portion is the end of its range) is
          // usually the last to arrive, the others the first.  A wrong guess only costs
          // a retry with the value the CAS returned.
          unsigned long long* ctr = a.counters + dsc.cf;
          unsigned long long old =
              dsc.cf == c ? ((unsigned long long)a.epoch << 32) | (uint32_t)(dsc.ncontrib - 1) : 0ull,
              nxt;
          for (;;) {
            nxt = (uint32_t)(old >> 32) == a.epoch ? old + 1
                                                    : ((unsigned long long)a.epoch << 32) | 1ull;
            const unsigned long long prev = cas_acq_rel_gpu(ctr, old, nxt);
            if (prev == old) break;
            old = prev;
          }
          const bool last = (int)(uint32_t)nxt == dsc.ncontrib;
          if (last) st_relaxed_gpu(ctr, 0ull);     // every contributor has arrived
          *last_flag = last;
        }
        named_bar_sync(1, kConsumerThreads);
        if (*last_flag) merge_split<T, D, NT, MODE>(a, dsc, *total_s, G, group, tid);
      }
      fence_proxy_async_smem();   // generic writes above precede the next TMA fill
    }
    if (patched) fence_proxy_async_smem();   // the patched row precedes the next TMA fill
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    if constexpr (BS == 1)
      if (cw == kHelperWarp && !take_fill(st, ph ^ 1u)) helper_abort();
    if (++st == kStages) {
      st = 0;
      ph ^= 1u;
    }
  }
  if (late_wait) pdl_wait();
}

}  // namespace pkv
