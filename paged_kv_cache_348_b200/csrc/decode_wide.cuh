// decode_wide.cuh -- paged decode for many query rows per kv head on tcgen05 tensor cores.
//
// Same operation as decode.cuh ("Paged Attention and Memory Efficiency in Production LLM
// Serving", section "How PagedAttention borrows OS paging": the kernel resolves each
// request's block table at run time and computes the plain softmax(scale q K^T) V), for
// the launches whose query rows per kv head -- the GQA group times the new tokens of a
// sequence ("PagedAttention -- The KV Cache Problem", "Why This Matters for Production":
// beam search and parallel sampling), or the members of a shared-prefix chunk -- number
// 9..64.  There the contraction is a real dense tile (up to 64 flop per KV byte), too
// much for warp-level mma.sync with register accumulators, so it runs on the
// 5th-generation tensor cores:
//
//  * One persistent CTA per SM takes an equal range of the batch's 16-token units (the
//    schedule of decode.cuh: segments = (sequence, kv head), weighted split, partials of
//    segments shared between CTAs merged by the last arrival).
//  * Warp 0 streams 128-token K tiles into a 3-stage ring with 4-D TMA copies whose row
//    coordinate comes from the block table (128-byte swizzle, tokens as rows, a unit's two
//    column halves in one box; at block_size 1 gather4 loads of four rows), and the
//    segment's query rows into a Q tile with cp.async (same swizzle); with 32 query
//    columns or fewer warp 10 walks the same schedule and issues the V tiles (one warp
//    issuing every load capped the stream at ~0.8 of HBM bandwidth with no compute at all;
//    at 64 columns the extra warp's registers cost the softmax more than it gains).
//  * Warp 1 (one thread) issues the MMAs: S^T[128 tokens][N] = K . Q^T with the tokens on
//    M = 128 and the query rows on N = 16..64 (no padding of the query side to 64 or 128),
//    accumulated in tensor memory (one S^T buffer per ring slot); then O^T[D][N] +=
//    V^T . P^T with V read MN-major from the same tile.  It is event driven: a stage's
//    QK^T goes out as soon as its tiles land, its PV as soon as the softmax is done.
//  * The softmax warps (warps 2..9, two warpgroups) split the query columns: a thread owns
//    one token row of S^T (one TMEM lane) and half of the columns.  Base 2, fp32, with
//    a lazily moved reference maximum per query row (a stage moves it only when some score
//    exceeds it by more than 2^8, which after a portion's first stage is rare; O^T is then
//    rescaled in tensor memory).  P^T is written in 16 bits into the stage's K tile, which
//    QK^T no longer needs; with bf16 its rounding residual goes beside it as NC more
//    columns, so one PV pass (N = 2 NC) accumulates both and ~16 bits of P count.  Row sums stay per thread and are reduced once per portion.  The same
//    warps read O^T back at the end of a portion (one thread per head dim and column half)
//    and write the output or the split partial.  The column count NC (16, 32 or 64, the
//    query rows rounded up) is a template parameter, so these loops are exactly as long
//    as a launch needs: with one CTA per SM the softmax has only two warps per scheduler
//    to hide latency with, and unused columns or runtime guards cost real time there.
//  * Every wait is bounded; tensor memory is released on every exit path.
#pragma once
#include "decode.cuh"

namespace pkv {

constexpr int kWideCols = 64;                     // query rows per kv head handled (MMA N)
constexpr int kWideTile = 128;                    // tokens per stage (MMA M of QK^T)
constexpr int kWideUnits = kWideTile / kUnit;     // 16-token units per stage
constexpr int kWideStages = 3;
// softmax warpgroups (warps 2 .. 1 + 4 * SWG): two, each owning half of the NC query columns.
// Four (16 columns each at NC 64) measured slower: the 576-thread CTA caps a thread at 96
// registers and the softmax spilled.
__host__ __device__ constexpr int wide_swg(int) { return 2; }
__host__ __device__ constexpr int wide_soft_threads(int nc) { return 128 * wide_swg(nc); }
// warps: 0 producer (K, Q; V too at 64 columns), 1 MMA, 2 .. 1 + 4 * SWG softmax, then at
// up to 32 columns the V producer
__host__ __device__ constexpr bool wide_vprod(int nc) { return nc <= 32; }
__host__ __device__ constexpr int wide_threads(int nc) {
  return 64 + wide_soft_threads(nc) + (wide_vprod(nc) ? 32 : 0);
}
// tensor memory: one S^T buffer per ring slot (columns 64 s .. 64 s + NC - 1) and O^T from
// column 256 (NC columns, or 2 NC when P's residual is a second column block)
constexpr uint32_t kWideTmemCols = 512;
constexpr uint32_t kOCol = 256;
constexpr float kRescaleLog2 = 8.f;               // a reference max moves past this gap only
// see pa_decode_wide_kernel: a portion's fixed cost grows with its query columns (the
// epilogue's row sums and output writes)
__host__ __device__ constexpr int wide_seg_weight(int nc) { return nc <= 16 ? 24 : (nc <= 32 ? 40 : 56); }

// K and V tiles: token row r, 64-dim half h (128 bytes, 128-byte swizzle) at
// ((r / 8) * kHalves + h) * 1024 + (r % 8) * 128: 8-row atoms with the halves side by side,
// so one TMA box (a 4-D view of the pool) brings a 16-row unit's both halves, and the
// MMA descriptors see 8-row groups at a stride of kHalves * 1024 bytes.
template <int D>
struct WideLayout {
  static constexpr int kHalves = D / 64;                        // 128-byte column halves
  static constexpr int kKvBytes = kHalves * kWideTile * 128;    // one K or V tile
  static constexpr int kGroupBytes = kHalves * 1024;            // one 8-row group, all halves
  static constexpr int kPBytes = kWideTile * 128;               // P^T high or low part
  // P^T (high, low) goes to the stage's K tile once QK^T has read it, when it fits
  static constexpr bool kPInK = kKvBytes >= 2 * kPBytes;
  static constexpr int kPOff = kPInK ? 0 : 2 * kKvBytes;
  static constexpr int kStageBytes = 2 * kKvBytes + (kPInK ? 0 : 2 * kPBytes);
  static constexpr int kQOff = kWideStages * kStageBytes;
  static constexpr int kQBytes = kHalves * kWideCols * 128;
  static constexpr int kMetaOff = kQOff + kQBytes;
  static constexpr int kBarOff = (kMetaOff + kWideStages * (int)sizeof(StageMeta) + 15) / 16 * 16;
  // full[3], empty[3], sfull[3], pfull[3], qempty, drain
  static constexpr int kNumBars = 4 * kWideStages + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;       // tmem base, abort, last, total
  static constexpr int kDescOff = kMiscOff + 32;
  static constexpr int kMrefOff = (kDescOff + 2 * (int)sizeof(SplitDesc) + 15) / 16 * 16;
  // float [5][64]: two reference-max buffers, a row of -inf (a portion's first stage), and
  // the two buffers again with -inf replaced by 0 (the reference p is computed against)
  static constexpr int kRedOff = kMrefOff + 5 * kWideCols * 4;  // float [64 cols][4 warps]
  static constexpr int kAlphaOff = kRedOff + kWideCols * 4 * 4;
  // per query column: new token (or chunk member) j and head g within the group
  static constexpr int kColOff = kAlphaOff + kWideCols * 4;
  static constexpr int kBytes = kColOff + 2 * kWideCols * 4;
  static constexpr int kDynSmem = kBytes + 1024;                // slack for 1024-byte alignment
  static_assert(kStageBytes % 1024 == 0 && kQOff % 1024 == 0 && kKvBytes % 1024 == 0,
                "tiles need 1024-byte alignment (128-byte swizzle atoms)");
  static_assert(kBarOff % 8 == 0 && kMiscOff % 8 == 0 && kDescOff % 8 == 0 && kMrefOff % 16 == 0,
                "mbarriers and 64-bit fields need 8-byte alignment");
  static_assert(kDynSmem <= 232448, "one CTA per SM must fit");
};

// Last arrival of a split segment (see merge_split in decode.cuh), for up to 64 query
// columns: out = (sum_k acc_k 2^(m_k - M)) / (sum_k l_k 2^(m_k - M)), contributors folded
// in CTA order.  Thread tid owns elements (column, 4 dims) e = tid + 256 i, 4 at a time.
template <typename T, int D, int MODE, int kWideSoftThreads>
__device__ __forceinline__ void merge_wide(const DecodeArgs& a, const SplitDesc& dsc,
                                           long long total, int G, int tid) {
  constexpr int kF4 = D / 4;
  constexpr int kB = 4;                                  // elements per batch
  const int nel = a.ncol * kF4;
  for (int e0 = tid; e0 < nel; e0 += kB * kWideSoftThreads) {
    float M[kB], Ls[kB];
    float4 acc[kB];
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      M[b] = -INFINITY;
      Ls[b] = 0.f;
      acc[b] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int cc = dsc.cf; cc <= dsc.cl; ++cc) {
      const int pk = partial_slot(cc, dsc.seg0, total, G);
      if (pk < 0) continue;
      float2 ml[kB];
      float4 v[kB];
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int e = e0 + b * kWideSoftThreads;
        ml[b] = make_float2(-INFINITY, 0.f);
        v[b] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < nel) {
          const long long row = (long long)pk * kWideCols + e / kF4;
          ml[b] = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + row);
          v[b] = __ldcg(reinterpret_cast<const float4*>(a.part_acc + row * D) + e % kF4);
        }
      }
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        if (ml[b].x == -INFINITY) continue;
        const float mn = fmaxf(M[b], ml[b].x);
        const float sa = M[b] == -INFINITY ? 0.f : ex2(M[b] - mn);
        const float sb = ex2(ml[b].x - mn);
        Ls[b] = Ls[b] * sa + ml[b].y * sb;
        acc[b].x = acc[b].x * sa + v[b].x * sb;
        acc[b].y = acc[b].y * sa + v[b].y * sb;
        acc[b].z = acc[b].z * sa + v[b].z * sb;
        acc[b].w = acc[b].w * sa + v[b].w * sb;
        M[b] = mn;
      }
    }
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      const int e = e0 + b * kWideSoftThreads;
      if (e >= nel) continue;
      const long long row = out_row<MODE>(a, dsc.seq, dsc.kvh, e / kF4);
      if (row < 0) continue;
      float v4[4] = {acc[b].x, acc[b].y, acc[b].z, acc[b].w};
      finish_row<T, MODE, D>(a, row, M[b], Ls[b], v4, (e % kF4) * 4, 4, make_float2(-INFINITY, 0.f),
                             v4);
    }
  }
}

// 8 consecutive 32-bit TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
               "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
}

template <typename T, int D, int BS, int MODE, int NC>
__global__ void __launch_bounds__(wide_threads(NC), 1)
    pa_decode_wide_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv) {
  using L = WideLayout<D>;
  static_assert(MODE == kPlain || MODE == kPrefix || MODE == kAppend,
                "wide decode: plain (multi-token), prefix or fused append");
  static_assert(NC == 16 || NC == 32 || NC == 64, "16, 32 or 64 query columns");
  constexpr int kWideSoftThreads = wide_soft_threads(NC);
  constexpr int CW = NC / wide_swg(NC);             // columns of one softmax warpgroup
  // bf16 P keeps ~16 bits as a high part (columns 0..NC-1 of P^T and O^T) plus its rounding
  // residual (columns NC..2NC-1, summed when O^T is read back); fp16 P has 11, enough here
  constexpr bool kSplit = std::is_same_v<T, __nv_bfloat16>;
  constexpr int kNPV = kSplit ? 2 * NC : NC;        // MMA N of PV
  // a segment's schedule weight beyond its units: a portion's fixed cost here (first stage
  // with its reference-max pass and Q load, end-of-portion epilogue) is worth about this
  // many 16-token units of streaming, several stages' worth (measured per CTA with
  // global-timer stamps, then timed: at 16 columns 24 against 16, 20, 32 and 48), far
  // more than in the mma.sync kernel
  constexpr int kSegW = wide_seg_weight(NC);
  constexpr uint32_t kAB = std::is_same_v<T, __nv_bfloat16> ? 1u : 0u;
  constexpr int kFullCount = 33;       // lane 0's expect_tx arrival + 32 cp.async arrivals
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + L::kMetaOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + kWideStages;
  uint64_t* sfull = empty + kWideStages;
  uint64_t* pfull = sfull + kWideStages;
  uint64_t* qempty = pfull + kWideStages;
  uint64_t* drain = qempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  volatile int* last_flag = abort_flag + 1;
  long long* total_s = reinterpret_cast<long long*>(smem + L::kMiscOff + 16);
  SplitDesc* desc = reinterpret_cast<SplitDesc*>(smem + L::kDescOff);
  float* mref = reinterpret_cast<float*>(smem + L::kMrefOff);      // [5][64]
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);        // [64][4]
  float* alph = reinterpret_cast<float*>(smem + L::kAlphaOff);     // [64]
  int* colj = reinterpret_cast<int*>(smem + L::kColOff);           // [64] column -> j
  int* colg = colj + kWideCols;                                    // [64] column -> head in group
  uint8_t* sQ = smem + L::kQOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the V producer (none: an index no warp has)
  constexpr int kVWarp = wide_vprod(NC) ? 2 + kWideSoftThreads / 32 : -1;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kWideStages; ++i) {
      mbar_init(&full[i], kFullCount);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kWideStages; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], kWideSoftThreads);
    }
    mbar_init(qempty, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < kWideCols; ++i) mref[2 * kWideCols + i] = -INFINITY;
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kWideTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + kWideCols) {
    const int cq = threadIdx.x - 64;
    colj[cq] = cq / a.group;
    colg[cq] = cq % a.group;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // Nothing global is written, and nothing a previous kernel may write is read, before the
  // previous grid is done; the producers of every CTA but CTA 0's K producer (which writes
  // the rows of sequences without units) compute their schedule first, from the launch's
  // lengths and chunk members, which no kernel of this library writes.
  if (warp != 0 && warp != kVWarp) {
    pdl_wait();
    pdl_trigger();
  }

  const int G = gridDim.x, c = blockIdx.x;
  const int Hkv = a.num_kv_heads, group = a.group;

  if (warp == 0 || warp == kVWarp) {
    // ============================== producers ==============================
    // Both walk the CTA's schedule; warp 0 (kw) issues the K tiles and the Q tile, sets each
    // stage's meta and byte count and ends the ring, the V warp issues the V tiles.  Each
    // waits for a slot's release on its own; the V loads of a fill may land before warp 0's
    // expect_tx (the transaction count goes negative, and the phase still waits for warp
    // 0's arrival).  Without a V warp, warp 0 issues both pools' tiles.
    const bool kw = warp == 0;
    constexpr int nkv = wide_vprod(NC) ? 1 : 2;    // pools this warp loads: kv0 .. kv0+nkv-1
    const int kv0 = kw ? 0 : 1;
    if (c == 0 && kw) pdl_wait();
    const int B = a.num_seqs;
    long long run = 0;
    int keep_ctx = 0, keep_u = 0, keep_x = 0;
    for (int base = 0; base < B; base += 32) {
      const int s = base + lane;
      SeqSpan sp{0, 0};
      if (s < B) sp = span_of<MODE>(a, s, c == 0 && kw ? a.status : nullptr);
      const int u = (sp.ctx + kUnit - 1) / kUnit;
      int x = u ? u + kSegW : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      keep_ctx = sp.ctx;
      keep_u = u;
      keep_x = x;
      run += __shfl_sync(0xffffffffu, x, 31);
      if (c == 0 && kw) {
        unsigned zero = __ballot_sync(0xffffffffu, s < B && u == 0);
        while (zero) {
          const int src = __ffs(zero) - 1;
          zero &= zero - 1;
          empty_rows<T, MODE, D>(a, base + src, 0, lane);
        }
      }
    }
    const long long total = (long long)Hkv * run;
    const long long start = total ? cta_start(c, total, G) : 0;
    const long long end = total ? cta_start(c + 1, total, G) : 0;

    int s_a = 0, u_a = 0, ctx_a = 0;
    long long pb_a = 0;
    if (start < end) {
      long long r2 = 0;
      bool got_a = false;
      for (int base = 0; base < B && !got_a; base += 32) {
        const int s = base + lane;
        int ctx = keep_ctx, u = keep_u, x = keep_x;
        if (B > 32) {
          SeqSpan sp{0, 0};
          if (s < B) sp = span_of<MODE>(a, s, nullptr);
          ctx = sp.ctx;
          u = (ctx + kUnit - 1) / kUnit;
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
          pb_a = __shfl_sync(0xffffffffu, lo, src);
          got_a = true;
        }
        r2 += __shfl_sync(0xffffffffu, x, 31);
      }
    }
    if (lane == 0 && kw) *total_s = total;
    __syncwarp();
    if (c != 0 || !kw) pdl_wait();

    const uint64_t policy = policy_evict_first();
    const int rows_total = a.num_blocks * Hkv * BS;
    int st = 0, nqs = 0, portions = 0;
    uint32_t ph = 0;
    bool ok = true;
    {
      long long x = start;
      int s_cur = s_a, u_cur = u_a, ctx_cur = ctx_a;
      long long pbase = pb_a;
      while (ok && x < end) {
        while (x >= pbase + (long long)Hkv * (u_cur ? u_cur + kSegW : 0)) {   // next sequence
          pbase += (long long)Hkv * (u_cur ? u_cur + kSegW : 0);
          ++s_cur;
          ctx_cur = span_of<MODE>(a, s_cur, nullptr).ctx;
          u_cur = (ctx_cur + kUnit - 1) / kUnit;
        }
        const int w_cur = u_cur + kSegW;
        const int kvh = (int)((x - pbase) / w_cur);
        const long long seg0 = pbase + (long long)kvh * w_cur, seg1 = seg0 + u_cur;
        if (x >= seg1) {                              // on the segment's virtual tail
          x = seg0 + w_cur;
          continue;
        }
        const long long pe = seg1 < end ? seg1 : end;
        const bool complete = seg0 >= start && seg1 <= end;
        const int pidx = c * 2 + (start < seg0 ? 1 : 0);
        int qslot = 0;
        if (!complete) {
          qslot = nqs++;
          if (lane == 0 && kw) {
            const int cf = cta_of(seg0, total, G), cl = cta_of(seg1 - 1, total, G);
            int ncontrib = 0;
            for (int cc = cf; cc <= cl; ++cc)
              ncontrib += cta_start(cc, total, G) < cta_start(cc + 1, total, G);
            desc[qslot] = SplitDesc{s_cur, kvh, cf, cl, ncontrib, 0, seg0};
          }
        }
        // a chunk of a prefix launch reads the prefix through its first member's table
        const long long trow_seq = MODE == kPrefix ? (long long)chunk_member(a, s_cur, 0) : s_cur;
        const int32_t* trow = a.block_tables + trow_seq * a.max_blocks;
        const int nblk = (ctx_cur + BS - 1) / BS;
        // block_size 1: the table entries of the portion's next stage, loaded while this
        // stage waits for its slot (pv_tok = the token they start at, -1: none loaded)
        int pv[4] = {-1, -1, -1, -1}, pv_tok = -1;
        for (long long tu = x; tu < pe; tu += kWideUnits) {
          const int nun = (int)((pe - tu) < kWideUnits ? (pe - tu) : kWideUnits);
          const int tok0 = (int)(tu - seg0) * kUnit;
          const bool first_stage = tu == x;
          const int flags = (first_stage ? F_FIRST : 0) | (tu + kWideUnits >= pe ? F_LAST : 0) |
                            (complete ? F_COMPLETE : 0);
          uint8_t* sK = smem + st * L::kStageBytes;
          uint8_t* sV = sK + L::kKvBytes;
          if constexpr (MODE == kAppend) {
            // fused append: the stage holding the newest token (position ctx-1) first
            // writes that token's K/V rows (k_new, v_new) to its cache rows, then reads the
            // tile, so the tile holds the new rows.  The stage is this segment's only reader
            // of that row.  Each writing lane fences its stores against the async proxy
            // before the warp issues the tile's TMA loads (an out-of-range block id is
            // flagged by the tile's own table lookups and the row is not written).
            const int tn = ctx_cur - 1;
            if (tn >= tok0 && tn < tok0 + nun * kUnit) {   // warp-uniform
              constexpr int CPR = D * 2 / 16;              // 16-byte chunks per row
              const int blk = __ldg(trow + tn / BS);
              if ((unsigned)blk < (unsigned)a.num_blocks && lane < nkv * CPR) {
                const int kv = kv0 + lane / CPR, ch = lane % CPR;   // this warp's pools
                const long long src = ((long long)s_cur * Hkv + kvh) * D;
                const long long row = ((long long)blk * Hkv + kvh) * BS + tn % BS;
                const T* nrow = static_cast<const T*>(kv ? a.v_new : a.k_new) + src;
                const uint4 val = __ldg(reinterpret_cast<const uint4*>(nrow) + ch);
                T* cache = static_cast<T*>(const_cast<void*>(kv ? a.v_cache : a.k_cache));
                reinterpret_cast<uint4*>(cache + row * D)[ch] = val;
                fence_proxy_async_global();
              }
              __syncwarp();
            }
          }
          if constexpr (BS != 1) {
            constexpr int H = BS < 16 ? BS : 16;     // rows per TMA box (all column halves)
            constexpr int BPU = kUnit / H;           // boxes per unit
            constexpr int kBoxBytes = H * 128 * L::kHalves;
            constexpr int kMaxBox = kWideUnits * BPU;    // of this warp's pool
            constexpr int kRep = (kMaxBox + 31) / 32;
            const int nbox = nun * BPU;
            // this lane's boxes and their block-table entries, read before the slot wait
            int ys[kRep];
#pragma unroll
            for (int rp = 0; rp < kRep; ++rp) {
              const int bi = lane + 32 * rp;
              const int jb = bi;
              const int t = tok0 + (jb / BPU) * kUnit + (jb % BPU) * H;
              ys[rp] = -1;
              if (bi < nbox && t < ctx_cur) {
                const int blk = t / BS < nblk ? __ldg(trow + t / BS) : -1;
                if ((unsigned)blk < (unsigned)a.num_blocks) {
                  ys[rp] = (blk * Hkv + kvh) * BS + (t % BS);
                } else {
                  if (a.status && kw) atomicOr(a.status, DEV_BAD_BLOCK_ID);
                  ys[rp] = rows_total;                 // out of range: TMA fills zeros
                }
              }
            }
            uint32_t bytes = 0;
            for (int jj = 0; jj < nun; ++jj) {
              const int rem = ctx_cur - (tok0 + jj * kUnit);
              const int nb = (rem + H - 1) / H;
              bytes += (uint32_t)((nb < BPU ? nb : BPU) * kBoxBytes * 2);
            }
            if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, kWaitLimitNs)) {
              ok = false;
              break;
            }
            if (lane == 0 && kw) {
              meta[st] = StageMeta{s_cur, kvh, tok0, nun, ctx_cur, flags, pidx, qslot, -1};
              mbar_arrive_expect_tx(&full[st], bytes);
            }
            __syncwarp();
#pragma unroll
            for (int rp = 0; rp < kRep; ++rp) {
              const int jb = lane + 32 * rp;
              if (ys[rp] >= 0) {
                const int row0 = (jb / BPU) * kUnit + (jb % BPU) * H;   // a multiple of 8
#pragma unroll
                for (int kk = 0; kk < nkv; ++kk) {
                  const int kv = kv0 + kk;
                  uint8_t* dst = (kv ? sV : sK) + (row0 >> 3) * L::kGroupBytes;
                  tma_load_4d(dst, kv ? &tmv : &tmk, &full[st], ys[rp] >> 3, policy);
                }
              }
            }
          } else {
            // block_size 1: each token is its own block.  TMA gather4 loads bring four rows
            // of one column half (128 bytes each, four table entries) into four consecutive
            // 128-byte lines of the same swizzled layout the box loads produce (the swizzle
            // follows the shared-memory address).  Lane l holds the table entries of rows
            // l, 32+l, 64+l, 96+l, read during the previous stage of the portion (for its
            // first stage: before the slot wait).
            const int nvalid = (nun * kUnit < ctx_cur - tok0) ? nun * kUnit : ctx_cur - tok0;
            int wv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int r = j * 32 + lane;
              wv[j] = pv_tok == tok0 ? pv[j] : (r < nvalid ? __ldg(trow + tok0 + r) : -1);
            }
            if (tu + kWideUnits < pe) {                // warp-uniform: the next stage's entries
              const int t1 = tok0 + kWideTile;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int r = j * 32 + lane;
                pv[j] = t1 + r < ctx_cur ? __ldg(trow + t1 + r) : -1;
              }
              pv_tok = t1;
            }
            if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, kWaitLimitNs)) {
              ok = false;
              break;
            }
            // load items (group of 4 rows g, half hf) of this warp's pool: at most 32 * 2 =
            // 64, two a lane; rows past the valid tokens or with a bad block id read row
            // rows_total, out of range, which the TMA fills with zeros
            const int nitems = ((nvalid + 3) >> 2) * L::kHalves;
            static_assert(kWideTile / 4 * L::kHalves <= 64, "two load items a lane");
            if (lane == 0 && kw) {
              meta[st] = StageMeta{s_cur, kvh, tok0, nun, ctx_cur, flags, pidx, qslot, -1};
              mbar_arrive_expect_tx(&full[st], (uint32_t)nitems * 2u * 512u);
            }
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 2 * nkv; ++it) {
              const int i = (it & 1) * 32 + lane;
              const int kv = kv0 + (it >> 1), hf = i % L::kHalves, g = i / L::kHalves;
              int y[4];
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const int r = 4 * g + q4;                // < 128 for every item issued
                const int v0 = __shfl_sync(0xffffffffu, wv[0], r & 31);
                const int v1 = __shfl_sync(0xffffffffu, wv[1], r & 31);
                const int v2 = __shfl_sync(0xffffffffu, wv[2], r & 31);
                const int v3 = __shfl_sync(0xffffffffu, wv[3], r & 31);
                const int blk = (r & 127) < 32 ? v0 : ((r & 127) < 64 ? v1 : ((r & 127) < 96 ? v2 : v3));
                y[q4] = rows_total;
                if (i < nitems && r < nvalid) {
                  if ((unsigned)blk < (unsigned)a.num_blocks) {
                    y[q4] = blk * Hkv + kvh;
                  } else if (a.status && hf == 0 && kv == 0) {
                    atomicOr(a.status, DEV_BAD_BLOCK_ID);
                  }
                }
              }
              if (i < nitems)
                tma_gather4((kv ? sV : sK) + ((g >> 1) * L::kHalves + hf) * 1024 + (g & 1) * 512,
                            kv ? &tmv : &tmk, &full[st], hf * 64, y[0], y[1], y[2], y[3], policy);
            }
          }
          if (first_stage && kw) {
            // the segment's query rows: column cq = token (or chunk member) j * group + head,
            // row cq of the Q tile, 128-byte swizzle.  The previous portion's last QK^T must
            // be done with the single Q tile first.
            if (portions > 0 &&
                !mbar_wait_bounded(qempty, (uint32_t)((portions - 1) & 1), abort_flag,
                                   kWaitLimitNs)) {
              ok = false;
              break;
            }
            constexpr int CPQ = D / 8;                 // 16-byte chunks per query row
            const int nchunk = a.ncol * CPQ;
            for (int k = lane; k < nchunk; k += 32) {
              const int cq = k / CPQ, ch = k % CPQ;
              const int jq = cq / group, g = cq % group;
              const T* src;
              if constexpr (MODE == kPrefix) {
                int mem = chunk_member(a, s_cur, jq);
                if (mem < 0) mem = (int)trow_seq;     // padding slot: the first member's rows
                src = static_cast<const T*>(a.q) +
                      ((long long)mem * a.num_q_heads + (long long)kvh * group + g) * D;
              } else {
                src = static_cast<const T*>(a.q) +
                      (((long long)s_cur * a.q_len + jq) * a.num_q_heads + (long long)kvh * group + g) *
                          D;
              }
              uint8_t* dst = sQ + (ch >> 3) * (kWideCols * 128) + cq * 128 + (((ch & 7) ^ (cq & 7)) << 4);
              cp_async_16(dst, src + ch * 8, policy);
            }
            ++portions;
          }
          if (kw) cp_async_mbar_arrive_noinc(&full[st]);
          if (++st == kWideStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        x = pe == seg1 ? seg0 + w_cur : pe;          // past the virtual tail
      }
    }
    if (kw && ok) ok = mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, kWaitLimitNs);
    if (!kw) {
      // the V producer is done with its last fill
    } else if (ok) {
      if (lane == 0) {
        meta[st].flags = F_END;
        mbar_arrive(&full[st]);
      }
      __syncwarp();
      cp_async_mbar_arrive_noinc(&full[st]);
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      if (a.status) atomicOr(a.status, DEV_TIMEOUT);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 1) {
    // ============================== MMA issue ==============================
    // Event driven: QK^T of a stage is issued as soon as its tiles have landed and its
    // slot's S^T buffer is free (at most kWideStages stages ahead of PV), PV as soon as the
    // softmax has written P^T.
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_f16(kAB, 0u, 0u, 128u, (uint32_t)NC);
      const uint32_t idesc_pv = idesc_f16(kAB, 1u, 1u, (uint32_t)D, (uint32_t)kNPV);
      // descriptors of slot 0; slots, k-steps and column halves add to the start-address
      // field (16-byte units, bits 0..13; every address here is below 256 KB, so the sum
      // never carries out of the field)
      const uint64_t dq0 = smem_desc_sw128(smem_u32(sQ), 16u, 1024u);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(smem), 16u, L::kGroupBytes);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(smem + L::kKvBytes), 1024u, L::kGroupBytes);
      const uint64_t dp0 = smem_desc_sw128(smem_u32(smem + L::kPOff), L::kPBytes, 1024u);
      auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
      auto qk = [&](int slot, int flags) {
        const uint32_t so = (uint32_t)(slot * L::kStageBytes);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks & 3) * 32;          // 16 dims = 32 bytes along a row
          tc_mma_f16(tbase + (uint32_t)(slot * 64),
                     adv(dk0, so + (ks >> 2) * 1024 + off),
                     adv(dq0, (ks >> 2) * (kWideCols * 128) + off), idesc_qk, ks > 0);
        }
        tc_commit(&sfull[slot]);
        if (flags & F_LAST) tc_commit(qempty);       // the Q tile may be refilled after this
      };
      auto pv = [&](int slot, bool first) {
        const uint32_t so = (uint32_t)(slot * L::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < kWideTile / 16; ++kk)
          tc_mma_f16(tbase + kOCol, adv(dv0, so + kk * 2 * L::kGroupBytes), adv(dp0, so + kk * 2048),
                     idesc_pv,
                     !(first && kk == 0));
      };
      int q_slot = 0, p_slot = 0, n_qk = 0, n_pv = 0;
      uint32_t q_ph = 0, p_ph = 0;
      int fl[kWideStages] = {0, 0, 0};
      bool q_end = false, ok = true;
      uint64_t idle_since = 0;
      while (ok) {
        bool progress = false;
        if (!q_end && n_qk - n_pv < kWideStages && mbar_try_wait(&full[q_slot], q_ph)) {
          // Q arrives by cp.async: generic-proxy writes the tensor cores read through the
          // async proxy
          fence_proxy_async_smem();
          const int f = meta[q_slot].flags;
          if (f & F_END) {
            q_end = true;
          } else {
            tc_fence_after();
            qk(q_slot, f);
            fl[q_slot] = f;
            ++n_qk;
            if (++q_slot == kWideStages) {
              q_slot = 0;
              q_ph ^= 1u;
            }
          }
          progress = true;
        }
        if (n_pv < n_qk && mbar_try_wait(&pfull[p_slot], p_ph)) {
          tc_fence_after();
          pv(p_slot, fl[p_slot] & F_FIRST);
          tc_commit(&empty[p_slot]);                // frees the stage (K, V and P tiles)
          ++n_pv;
          if (++p_slot == kWideStages) {
            p_slot = 0;
            p_ph ^= 1u;
          }
          progress = true;
        }
        if (q_end && n_pv == n_qk) break;
        if (progress) {
          idle_since = 0;
        } else if (*abort_flag) {
          ok = false;
        } else {
          const uint64_t now = globaltimer_ns();
          if (!idle_since) idle_since = now;
          else if (now - idle_since > kWaitLimitNs) ok = false;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        if (a.status) atomicOr(a.status, DEV_TIMEOUT);
      }
      // nothing issued here may still be running when tensor memory is released (this
      // wait ignores the abort flag: only its time limit ends it)
      tc_commit(drain);
      int no_abort = 0;
      mbar_wait_bounded(drain, 0u, &no_abort, kWaitLimitNs);
    }
    __syncwarp();      // the warp reaches the CTA barrier below together, lane 0 included
  } else {
    // ============================== softmax / epilogue ==============================
    const int wg = (warp - 2) >> 2;                // softmax warpgroup: columns c0 .. c0+CW-1
    const int c0 = wg * CW;
    const int q4 = warp & 3;                       // TMEM lane quadrant of this warp
    const int r = q4 * 32 + lane;                  // token row of S^T (= head dim of O^T at D 128)
    const int tid = threadIdx.x - 64;
    const uint32_t trow_addr = tbase + ((uint32_t)(q4 * 32) << 16);
    float lp[CW];                                  // this row's share of the column sums
#pragma unroll
    for (int j = 0; j < CW; ++j) lp[j] = 0.f;
    int cur = 0;
    int st = 0;
    uint32_t ph = 0;
    int pst = 0;
    uint32_t pph = 0;                              // slot/parity of the previous stage
    auto give_up = [&]() {
      if (lane == 0) {
        *abort_flag = 1;
        if (a.status) atomicOr(a.status, DEV_TIMEOUT);
      }
    };
    // CW consecutive TMEM columns starting at col of this warp's lanes
    auto tld = [&](uint32_t col, float* v) {
      if constexpr (CW == 8) {
        tmem_ld8(trow_addr + col, v);
      } else {
#pragma unroll
        for (int k = 0; k < CW / 16; ++k) {
          float w[16];
          tmem_ld16(trow_addr + col + 16 * k, w);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[16 * k + j] = w[j];
        }
      }
    };
    auto tst = [&](uint32_t col, const float* v) {
      if constexpr (CW == 8) {
        tmem_st8(trow_addr + col, v);
      } else {
#pragma unroll
        for (int k = 0; k < CW / 16; ++k) {
          float w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) w[j] = v[16 * k + j];
          tmem_st16(trow_addr + col + 16 * k, w);
        }
      }
    };
    for (int i = 0;; ++i) {
      if (!mbar_wait_bounded(&full[st], ph, abort_flag, kWaitLimitNs)) {
        give_up();
        break;
      }
      const StageMeta mt = meta[st];
      if (mt.flags & F_END) break;
      const bool first = mt.flags & F_FIRST;
      if (first) {
#pragma unroll
        for (int j = 0; j < CW; ++j) lp[j] = 0.f;
      }
      if (!mbar_wait_bounded(&sfull[st], ph, abort_flag, kWaitLimitNs)) {   // this slot's S^T
        give_up();
        break;
      }
      tc_fence_after();
      float s[CW];
      tld((uint32_t)(st * 64 + c0), s);
      tmem_wait_ld();
      const int nvalid = (mt.nunits * kUnit < mt.ctx - mt.tok0) ? mt.nunits * kUnit : mt.ctx - mt.tok0;
      const bool tv = r < nvalid;
      // causal limit: new token j sees stage rows < lim0 + j (a prefix launch: no mask)
      const int lim0 = MODE == kPrefix ? (1 << 30) : mt.ctx - a.q_len + 1 - mt.tok0;
      // reference maxima in force: a portion's first stage starts from the -inf row.  With
      // x = scale * s (base 2), e = max_j (x_j - m_j) tells whether a reference must move;
      // masked scores are -inf (NaN against a -inf reference, which fmaxf ignores)
      const float sc = a.scale_log2;
      const float* mcur = mref + (first ? 2 : cur) * kWideCols;
      float e = -INFINITY;
      if (tv && (MODE == kPrefix || r < lim0)) {   // every column sees this row
        if (a.ncol < c0 + CW) {                    // padding columns of this warpgroup
#pragma unroll
          for (int j = 0; j < CW; ++j)
            if (c0 + j >= a.ncol) s[j] = -INFINITY;
        }
#pragma unroll
        for (int j = 0; j < CW; j += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(mcur + c0 + j);
          e = fmaxf(e, fmaf(s[j], sc, -m4.x));
          e = fmaxf(e, fmaf(s[j + 1], sc, -m4.y));
          e = fmaxf(e, fmaf(s[j + 2], sc, -m4.z));
          e = fmaxf(e, fmaf(s[j + 3], sc, -m4.w));
        }
      } else {
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const int cq = c0 + j;
          const bool vis = tv && cq < a.ncol && (MODE == kPrefix || r < lim0 + colj[cq]);
          if (!vis) s[j] = -INFINITY;
          e = fmaxf(e, fmaf(s[j], sc, -mcur[cq]));
        }
      }
      const bool slow = bar_red_or(1, kWideSoftThreads, first || e > kRescaleLog2);
      if (slow) {
        // move the reference maxima: this warpgroup's column maxima over the 128 rows
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const float wm = warp_max_f32(s[j] * sc);
          if (lane == j) red[(c0 + j) * 4 + q4] = wm;
        }
        named_bar_sync(1, kWideSoftThreads);
        float* mnext = mref + (cur ^ 1) * kWideCols;
        float* mnext_p = mref + (3 + (cur ^ 1)) * kWideCols;
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const float4 w4 = *reinterpret_cast<const float4*>(red + (c0 + j) * 4);
          const float cm = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
          const float mo = mcur[c0 + j];
          const float mn = fmaxf(mo, cm);
          const float al = (mo == -INFINITY) ? 0.f : ex2(mo - mn);
          lp[j] *= al;
          if (r == j) {
            mnext[c0 + j] = mn;
            mnext_p[c0 + j] = mn == -INFINITY ? 0.f : mn;   // p = 0 while nothing is visible
            alph[c0 + j] = al;
          }
        }
        named_bar_sync(1, kWideSoftThreads);
        cur ^= 1;
        if (!first) {
          // O^T was accumulated against the old maxima: rescale this warpgroup's columns
          // once the previous stage's PV is done (its commit freed that stage's slot)
          if (!mbar_wait_bounded(&empty[pst], pph, abort_flag, kWaitLimitNs)) {
            give_up();
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < (kSplit ? 2 : 1); ++part) {
            float o[CW];
            tld(kOCol + (uint32_t)(part * NC + c0), o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < CW; ++j) o[j] *= alph[c0 + j];
            tst(kOCol + (uint32_t)(part * NC + c0), o);
          }
          tmem_wait_st();
        }
      }
      // P^T row r: p = 2^(x - m), 16 bits per value in 16-byte chunks of 8 columns; P^T
      // column col sits in 64-column block col / 64 (kPBytes apart), 128-byte swizzle
      {
        const float* mc = mref + (3 + cur) * kWideCols;   // -inf replaced by 0
        uint8_t* sP = smem + st * L::kStageBytes + L::kPOff;
        auto put = [&](int col, uint4 v) {
          const int chunk = (col & 63) >> 3;
          *reinterpret_cast<uint4*>(sP + (col >> 6) * L::kPBytes + r * 128 +
                                    ((chunk ^ (r & 7)) << 4)) = v;
        };
#pragma unroll
        for (int ch = 0; ch < CW / 8; ++ch) {
          const float4 m0 = *reinterpret_cast<const float4*>(mc + c0 + ch * 8);
          const float4 m1 = *reinterpret_cast<const float4*>(mc + c0 + ch * 8 + 4);
          const float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            const float p0 = ex2(fmaf(s[ch * 8 + j], sc, -mm[j]));
            const float p1 = ex2(fmaf(s[ch * 8 + j + 1], sc, -mm[j + 1]));
            lp[ch * 8 + j] += p0;
            lp[ch * 8 + j + 1] += p1;
            const uint32_t h = pack2<T>(p0, p1);
            hi[j / 2] = h;
            if constexpr (kSplit) {
              const float2 hf = unpack2<T>(h);
              lo[j / 2] = pack2<T>(p0 - hf.x, p1 - hf.y);
            }
          }
          put(c0 + ch * 8, make_uint4(hi[0], hi[1], hi[2], hi[3]));
          if constexpr (kSplit) put(NC + c0 + ch * 8, make_uint4(lo[0], lo[1], lo[2], lo[3]));
        }
        if (!tv && wg < L::kHalves) {
          // a row past the stage's valid tokens may hold stale or NaN data: P is zero
          // there, and V must be finite (0 x NaN would poison O); warpgroup wg clears
          // column half wg of the row
          uint8_t* sV = smem + st * L::kStageBytes + L::kKvBytes + (r >> 3) * L::kGroupBytes +
                        wg * 1024 + (r & 7) * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4*>(sV + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();                    // P and V rows -> the tensor cores
      tc_fence_before();
      mbar_arrive(&pfull[st]);
      if (mt.flags & F_LAST) {
        // ---- end of a segment portion: row sums, then O^T back from tensor memory
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          float v = lp[j];
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          if (lane == j) red[(c0 + j) * 4 + q4] = v;
        }
        named_bar_sync(1, kWideSoftThreads);
        if (!mbar_wait_bounded(&empty[st], ph, abort_flag, kWaitLimitNs)) {   // this PV done
          give_up();
          break;
        }
        tc_fence_after();
        // head dim of this thread's O^T lane: lane r at D 128; at D 64 (M = 64) dims
        // 16 q4 .. 16 q4 + 15 sit in lanes 0..15 of quadrant q4
        const int d = D == 128 ? r : (lane < 16 ? q4 * 16 + lane : -1);
        const bool complete = mt.flags & F_COMPLETE;
        const float* mc = mref + cur * kWideCols;
        // O^T back 8 columns at a time (the high part plus, with bf16, the residual part)
#pragma unroll 1
        for (int j0 = 0; j0 < CW; j0 += 8) {
          float o[8];
          tmem_ld8(trow_addr + kOCol + (uint32_t)(c0 + j0), o);
          if constexpr (kSplit) {
            float o2[8];
            tmem_ld8(trow_addr + kOCol + (uint32_t)(NC + c0 + j0), o2);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] += o2[j];
          } else {
            tmem_wait_ld();
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int cq = c0 + j0 + j;
            if (cq < a.ncol && d >= 0) {
              const float4 w4 = *reinterpret_cast<const float4*>(red + cq * 4);
              const float Ls = (w4.x + w4.y) + (w4.z + w4.w);
              const float M = mc[cq];
              if (complete) {
                // output row of column cq: out_row without its divisions
                long long row;
                if constexpr (MODE == kPrefix) {
                  const int mem = chunk_member(a, mt.seq, colj[cq]);
                  row = mem < 0 ? -1ll
                                : (long long)mem * a.num_q_heads + (long long)mt.kvh * group + colg[cq];
                } else {
                  row = ((long long)mt.seq * a.q_len + colj[cq]) * a.num_q_heads +
                        (long long)mt.kvh * group + colg[cq];
                }
                if (row >= 0) {
                  if constexpr (MODE == kPrefix) {
                    if (d == 0) a.ext_ml[row] = make_float2(M, Ls);
                    a.ext_acc[row * D + d] = o[j];
                  } else {
                    static_cast<T*>(a.out)[row * D + d] = from_float<T>(Ls > 0.f ? o[j] / Ls : 0.f);
                  }
                }
              } else {
                const long long prow = (long long)mt.pidx * kWideCols + cq;
                a.part_acc[prow * D + d] = o[j];
                if (d == 0) {
                  a.part_ml[prow * 2 + 0] = M;
                  a.part_ml[prow * 2 + 1] = Ls;
                }
              }
            }
          }
        }
        tc_fence_before();
        if (!complete) {
          // arrival on the segment's counter (as in decode.cuh): the last contributor merges
          named_bar_sync(1, kWideSoftThreads);
          const SplitDesc dsc = desc[mt.qslot];
          if (tid == 0) {
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
            if (last) st_relaxed_gpu(ctr, 0ull);
            *last_flag = last;
          }
          named_bar_sync(1, kWideSoftThreads);
          if (*last_flag) merge_wide<T, D, MODE, kWideSoftThreads>(a, dsc, *total_s, G, tid);
        }
        named_bar_sync(1, kWideSoftThreads);       // red[] is reused by the next stage
#pragma unroll
        for (int j = 0; j < CW; ++j) lp[j] = 0.f;  // the next stage starts a portion
      }
      pst = st;
      pph = ph;
      if (++st == kWideStages) {
        st = 0;
        ph ^= 1u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kWideTmemCols);
  }
}

}  // namespace pkv
