/*
 * pagedkv.h -- C ABI of libpagedkv: paged KV-cache decode attention and its two
 * companion kernels, for NVIDIA B200 (sm_100a).
 *
 * Pages the operations come from (cited by page title and section):
 *  [P1] "Paged Attention and Memory Efficiency in Production LLM Serving"
 *  [P2] "PagedAttention in Production: Boosting LLM Serving Throughput with Paged
 *       KV Cache"
 *  [P3] "PagedAttention -- The KV Cache Problem"
 *
 * Conventions shared by every call
 *  - Pointers named *cache*, q, out, k, v, block_tables, context_lens, slot_mapping,
 *    pairs, workspace and dev_status are DEVICE pointers on the current CUDA device;
 *    k_caches / v_caches in pa_copy_blocks are HOST arrays holding device pointers.
 *  - Ownership: the caller owns every buffer, including the workspace.  The library
 *    allocates no device memory and keeps no state between calls.
 *  - Synchrony: every call only enqueues work on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) and returns; results are ready when the stream is.
 *    The kernels are launched as programmatic dependents of the previous kernel on the
 *    stream: a decode kernel may begin reading its context lengths, block tables,
 *    prefix lengths and chunk members while a previous kernel of THIS library is still
 *    running (none of them writes those arrays); everything else waits for it.  A
 *    kernel of other code that writes those arrays must finish before the call (plain
 *    stream order does that, unless that kernel itself releases its dependents early).
 *  - Errors: arguments are validated on the host before anything is enqueued; a
 *    failed check returns an error code and enqueues nothing.  A CUDA launch error
 *    returns PA_ERR_CUDA.  Range violations found on the device (a block id outside
 *    [0, num_blocks), a slot outside [-1, num_blocks*block_size), a pair outside the
 *    pool, a context length outside [0, max_blocks_per_seq*block_size]) never fault:
 *    the offending access is skipped (or the length clamped) and, when dev_status is
 *    not NULL, the matching PA_DEV_* bit is OR-ed into *dev_status.
 *  - KV cache layout, per layer, separately for K and V (the pages only say
 *    "fixed-size blocks"; this layout keeps each (block, kv head) slice contiguous):
 *        cache[num_blocks][num_kv_heads][block_size][head_dim], 16-bit elements.
 *  - Supported: head_dim in {64, 128}; block_size in {1, 8, 16, 32};
 *    num_q_heads % num_kv_heads == 0; q, out and the caches share one dtype.  The query
 *    rows one kv head serves (q heads per kv head x new tokens per sequence, or x chunk
 *    members in a cascade prefix pass) may number up to 64 for pa_decode,
 *    pa_decode_multi, pa_decode_append and the cascade's prefix pass over 16-bit pools,
 *    up to 16 for 8-bit pools and the cascade's per-sequence pass.  Up to 8 rows run on
 *    warp-level tensor-core MMAs; 9 to 64 on the 5th-generation (tcgen05) tensor cores
 *    with the accumulators in tensor memory (PAGEDKV_WIDE_MIN_COLS=n in the environment
 *    moves that threshold, for comparing the two kernels; 8-bit pools and the cascade's
 *    per-sequence pass keep the warp-level kernel up to 16 rows).  Pointers must be
 *    16-byte aligned.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,      /* null/misaligned pointer, bad size, workspace too small */
  PA_ERR_UNSUPPORTED = 2,  /* head_dim, block_size, dtype or group size not built */
  PA_ERR_CUDA = 3,         /* a CUDA runtime/driver call or launch failed */
  PA_ERR_NO_BLOCKS = 4,    /* block manager: not enough free blocks; nothing was changed */
  PA_ERR_NO_MEMORY = 5     /* block manager: host memory allocation failed */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

/* Bits OR-ed into *dev_status by the kernels (see "Errors" above). */
#define PA_DEV_BAD_BLOCK_ID 0x1
#define PA_DEV_BAD_SLOT 0x2
#define PA_DEV_BAD_PAIR 0x4
#define PA_DEV_BAD_CONTEXT_LEN 0x8
#define PA_DEV_TIMEOUT 0x10 /* a pipeline wait gave up after ~2 s; outputs are invalid */

/* Library ABI version (major*100 + minor). */
int pa_version(void);

/* Short English text for a status code (static storage). */
const char* pa_status_string(pa_status status);

/*
 * Bytes of workspace pa_decode needs for `num_seqs` sequences on the CURRENT
 * device (the split schedule is sized by its SM count).  Returns 0 on bad arguments.
 */
size_t pa_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim);

/*
 * pa_decode -- attention of each sequence's newest query token over its paged KV.
 *
 * Defined by [P1] "How PagedAttention borrows OS paging": each request keeps a
 * logical block table that the attention kernel resolves at run time, and the
 * attention arithmetic itself (dot products, softmax, value-weighted sum) is the
 * plain one; [P2] "Core Principle" (logical block i of a request -> physical block
 * block_tables[i]); [P3] "How It Works" (the kernel reads the block table to gather
 * KV from non-contiguous blocks).
 *
 * For sequence s and q head h (kv head kvh = h / (num_q_heads/num_kv_heads)):
 *   K_s[t] = k_cache[block_tables[s][t / block_size]][kvh][t % block_size][:],
 *   V_s[t] likewise, for t in [0, context_lens[s]);
 *   out[s][h][:] = sum_t softmax_t(scale * <q[s][h], K_s[t]>) * V_s[t],
 * computed with an fp32 online softmax and fp32 accumulation, rounded to the dtype.
 * context_lens[s] counts every cached token, the newest one included (append runs
 * first).  A length of 0 gives an all-zero output row.  Block-table entries past
 * ceil(context_lens[s]/block_size) and cache slots past the last token are never read.
 *
 *   out            [num_seqs][num_q_heads][head_dim]            (written)
 *   q              [num_seqs][num_q_heads][head_dim]
 *   k_cache/v_cache  layout above, num_blocks blocks
 *   block_tables   int32 [num_seqs][max_blocks_per_seq]
 *   context_lens   int32 [num_seqs]
 *   workspace      >= pa_decode_workspace_bytes(...) bytes, 256-byte aligned; its
 *                  contents on entry do not matter and are clobbered.
 *   dev_status     int32, nullable (see "Errors").
 *
 * The result is a deterministic function of the logical inputs: it does not depend
 * on which physical blocks hold the data.
 */
pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int max_blocks_per_seq, int num_blocks, float scale, pa_dtype dtype,
                    void* workspace, size_t workspace_bytes, int32_t* dev_status,
                    void* stream);

/*
 * pa_decode_multi -- pa_decode for q_len new tokens per sequence (speculative, beam or
 * chunked decoding), causal among them.
 *
 * Defined, besides the passages cited for pa_decode, by [P1] "Why KV cache memory was
 * the bottleneck": a generated token uses the keys and values of every token before
 * it.  The q_len new tokens of sequence s are its last q_len cached positions (append
 * them first), so new token j sits at position p = context_lens[s] - q_len + j and
 *   out[s][j][h][:] = sum_{t <= p} softmax_t(scale * <q[s][j][h], K_s[t]>) * V_s[t].
 * A new token with p < 0 (context_lens[s] < q_len) sees nothing: its row is zero.
 *
 *   q, out         [num_seqs][q_len][num_q_heads][head_dim]
 *   other arguments as for pa_decode; the workspace size does not depend on q_len.
 * Limits: 1 <= q_len and (num_q_heads/num_kv_heads) * q_len <= 64 (PA_ERR_UNSUPPORTED
 * otherwise).  q_len == 1 gives exactly the bits of pa_decode.
 */
pa_status pa_decode_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                          int q_len, int num_q_heads, int num_kv_heads, int head_dim,
                          int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                          pa_dtype dtype, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, void* stream);

/*
 * pa_decode_append -- pa_cache_append of each sequence's newest token fused into
 * pa_decode: one launch instead of two for the usual decode step.
 *
 * Defined by the passages of pa_cache_append and pa_decode.  For every sequence s with
 * context_lens[s] > 0, the newest token sits at position p = context_lens[s] - 1; its
 * K and V (k_new[s], v_new[s]) are written to the cache row of p,
 *   cache[block_tables[s][p / block_size]][h][p % block_size][:],
 * and out is the pa_decode result over positions 0..p with that token included: the
 * same bits as pa_cache_append (slot of position p) followed by pa_decode.
 *
 *   k_new, v_new   device [num_seqs][num_kv_heads][head_dim], 16-byte aligned
 *   k_cache, v_cache  written at the newest token's rows only
 *   other arguments, workspace and errors as for pa_decode; an out-of-range block id
 *   for position p sets PA_DEV_BAD_BLOCK_ID and that token is not written.
 * The newest token's block must not be shared with another sequence (copy it first,
 * as for pa_cache_append).
 */
pa_status pa_decode_append(void* out, const void* q, void* k_cache, void* v_cache,
                           const void* k_new, const void* v_new, const int32_t* block_tables,
                           const int32_t* context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                           int num_blocks, float scale, pa_dtype dtype, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * 8-bit KV cache (E4M3): half the bytes per cached token.
 *
 * Defined by [P3] "What's Still Unsolved" (FP4/FP8 quantised KV cache: lower precision
 * saves memory).  Format: E4M3 -- 1 sign bit, 4 exponent bits with bias 7, 3 fraction
 * bits, no infinity, S.1111.111 = NaN; largest finite value 448.  A pool holds codes c
 * with value scale * c for one per-tensor scale per pool (k_scale for K, v_scale for V,
 * chosen by the caller, > 0).  Layout as for 16-bit pools with 1-byte elements.
 *
 * pa_cache_append_e4m3 -- pa_cache_append into E4M3 pools: every value x of k (v) is
 * stored as the E4M3 code of x / k_scale (x / v_scale) computed in binary32 with IEEE
 * division, rounded to nearest even, magnitudes above 448 clamped to 448.  k and v are
 * 16-bit (dtype); head_dim a multiple of 16.  Other arguments and errors as for
 * pa_cache_append.
 *
 * pa_decode_e4m3 -- pa_decode over E4M3 pools: K_s[t] = k_scale * code, V_s[t] = v_scale *
 * code, everything else as for pa_decode (q and out 16-bit, dtype).  Inside, the codes
 * are converted exactly to fp16 and the products use fp16 tensor-core MMAs with fp32
 * accumulation (q is converted to fp16: values beyond fp16's range are not supported).
 * head_dim 64 or 128; workspace as for pa_decode.
 */
pa_status pa_cache_append_e4m3(void* k_cache, void* v_cache, const void* k, const void* v,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               float k_scale, float v_scale, int32_t* dev_status, void* stream);
pa_status pa_decode_e4m3(void* out, const void* q, const void* k_cache, const void* v_cache,
                         float k_scale, float v_scale, const int32_t* block_tables,
                         const int32_t* context_lens, int num_seqs, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                         int num_blocks, float scale, pa_dtype dtype, void* workspace,
                         size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * 8-bit KV cache (E4M3) with per-(block, kv head) scales.
 *
 * Defined by [P3] "What's Still Unsolved" (FP8 quantised KV cache); the pages give no
 * format or scale granularity, and this reading gives every (physical block, kv head)
 * slice of a pool its own scale: k_scales / v_scales, float32 [num_blocks][num_kv_heads]
 * device arrays beside the pools (value = scale * code).  A block's scale is fixed when
 * its offset-0 token is written: with amax the largest |x| of that token's row for the
 * head and y = amax / 448 in binary32, scale = 2^(ceil(log2 y) + 3) -- the power of two s
 * with s/16 < y <= s/8, leaving 8x headroom for later tokens of the block (larger values
 * saturate at 448 * s); 1 for an all-zero row.  Blocks fill in order, so every token of a
 * block is quantised with the scale its first token set.
 *
 * pa_cache_append_e4m3_bs -- the quantising append: first every token whose slot is
 * offset 0 of its block sets that block's scales (in the same call, before any value is
 * quantised, whatever the order of the tokens), then every value x becomes the E4M3
 * code of x / scale (binary32 IEEE division, round to nearest even, clamped to 448).
 * Arguments as for pa_cache_append_e4m3, with the scale arrays in place of the two
 * per-pool scales; blocks whose offset 0 is not written keep their scales.  Two tokens at
 * offset 0 of one block in one call are undefined (as are duplicate slots).
 *
 * pa_decode_e4m3_bs -- decode of q_len new tokens per sequence (as pa_decode_multi;
 * q_len = 1 is pa_decode) over such pools: K_s[t] = k_scales[b][h] * code with b the
 * physical block of position t, V likewise.  Inside, each token row's K scale multiplies
 * its scores and its V scale its softmax weights before the fp16 tensor-core PV product.
 * head_dim 64 or 128, (num_q_heads/num_kv_heads) * q_len <= 16; workspace as for
 * pa_decode.
 */
pa_status pa_cache_append_e4m3_bs(void* k_cache, void* v_cache, float* k_scales,
                                  float* v_scales, const void* k, const void* v,
                                  const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                                  int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                                  int32_t* dev_status, void* stream);
pa_status pa_decode_e4m3_bs(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const float* k_scales, const float* v_scales,
                            const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                            int q_len, int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                            pa_dtype dtype, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream);

/*
 * pa_decode_cascade -- pa_decode for a batch in which groups of sequences share a prefix
 * of their KV blocks (parallel sampling, beams, a common system prompt), reading each
 * shared block once per chunk of sharers instead of once per sequence.
 *
 * Defined by [P1] "How PagedAttention borrows OS paging" (requests with an identical
 * prefix point their block tables at the same physical blocks) and [P3] "Why This
 * Matters for Production" (parallel sampling and beam search share KV blocks).  The
 * result is that of pa_decode on the same inputs (one new token per sequence): the
 * softmax over a sequence's tokens is split at prefix_lens[s] into the shared part and
 * the sequence's own part, each reduced to (max, sum, unnormalised acc), and the two
 * are combined exactly (log-sum-exp); only the rounding order differs from pa_decode.
 *
 Two launches on `stream`: pass 1 decodes every chunk's prefix (tokens
 * 0..chunk_prefix_lens[c]-1, read through the block table of the chunk's first member)
 * with the query rows of all its members at once; pass 2 decodes every sequence's
 * tokens prefix_lens[s]..context_lens[s]-1 and merges the prefix result.  Pass 2 waits
 * for pass 1 only where it reads pass 1's partials, so the two overlap.
 *
 *   q, out, caches, block_tables, context_lens   as for pa_decode
 *   prefix_lens        device int32 [num_seqs]: shared-prefix length of each sequence,
 *                      0 for a sequence in no chunk
 *   chunk_members      device int32 [num_chunks][chunk_width]: member sequence ids,
 *                      padded with -1; the first slot must be a member.  1 <= chunk_width
 *                      and (num_q_heads/num_kv_heads) * chunk_width <= 64: a chunk's query
 *                      rows share the MMA N dimension, so the prefix is read once for all
 *                      of them (pa_plan_cascade plans such chunks)
 *   chunk_prefix_lens  device int32 [num_chunks]
 *   workspace          >= pa_decode_cascade_workspace_bytes(...) bytes, 256-byte aligned
 Contract (not checked on the device): every sequence with prefix_lens[s] > 0 is a
 * member of exactly one chunk, whose prefix length equals prefix_lens[s], and the block
 * tables of a chunk's members agree on their first ceil(prefix/block_size) entries; a
 * member's context is at least its prefix, and a prefix that is not a multiple of
 * block_size ends its members' contexts (true of tables kept with copy-on-write, where a
 * block stays shared only while no sharer writes into it; pa_plan_cascade plans such
 * chunks).
 * Member ids outside [0, num_seqs) count as padding; a chunk whose first member is
 * padding is empty.  num_q_heads/num_kv_heads must be <= 16 (the per-sequence pass).
 * Other arguments, limits and errors as for pa_decode.
 */
size_t pa_decode_cascade_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads,
                                         int head_dim);
pa_status pa_decode_cascade(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            const int32_t* prefix_lens, int num_seqs,
                            const int32_t* chunk_members, int chunk_width,
                            const int32_t* chunk_prefix_lens, int num_chunks, int num_q_heads,
                            int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int num_blocks, float scale, pa_dtype dtype,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream);

/*
 * The cascade and the fused append over 8-bit pools with per-(block, kv head) scales
 * (the format of pa_cache_append_e4m3_bs / pa_decode_e4m3_bs; head_dim 64 or 128).
 *
 * pa_decode_cascade_e4m3_bs -- pa_decode_cascade over such pools: the result is that of
 * pa_decode_e4m3_bs (q_len 1) on the same inputs, the softmax split at prefix_lens[s]
 * and recombined exactly as for pa_decode_cascade.  Arguments, contract and errors as
 * for pa_decode_cascade, plus the scale arrays, with one more limit: a chunk holds at
 * most 16 query rows, (num_q_heads/num_kv_heads) * chunk_width <= 16.  Workspace:
 * pa_decode_cascade_workspace_bytes.
 *
 * pa_decode_append_e4m3_bs -- pa_cache_append_e4m3_bs of each sequence's newest token
 * (position p = context_lens[s] - 1, slot of p through block_tables) fused into
 * pa_decode_e4m3_bs (q_len 1): the same cache codes, scales and output bits as the two
 * calls in sequence.  When p is offset 0 of its block the token sets that block's scales
 * (k_scales, v_scales are written there); otherwise they are read.  Arguments and errors
 * as for pa_decode_append, plus the scale arrays; the newest token's block must not be
 * shared with another sequence.
 */
pa_status pa_decode_cascade_e4m3_bs(void* out, const void* q, const void* k_cache,
                                    const void* v_cache, const float* k_scales,
                                    const float* v_scales, const int32_t* block_tables,
                                    const int32_t* context_lens, const int32_t* prefix_lens,
                                    int num_seqs, const int32_t* chunk_members, int chunk_width,
                                    const int32_t* chunk_prefix_lens, int num_chunks,
                                    int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int num_blocks,
                                    float scale, pa_dtype dtype, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, void* stream);
pa_status pa_decode_append_e4m3_bs(void* out, const void* q, void* k_cache, void* v_cache,
                                   float* k_scales, float* v_scales, const void* k_new,
                                   const void* v_new, const int32_t* block_tables,
                                   const int32_t* context_lens, int num_seqs, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int max_blocks_per_seq, int num_blocks, float scale,
                                   pa_dtype dtype, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_status, void* stream);

/*
 * pa_cache_append -- write the new tokens' K and V into their cache slots.
 *
 * Defined by [P1] "How PagedAttention borrows OS paging" (blocks are filled on demand
 * as decoding proceeds) and [P3] "How It Works" (allocate blocks on demand as tokens
 * are generated).  For every token i with slot = slot_mapping[i] >= 0:
 *   k_cache[slot / block_size][h][slot % block_size][:] = k[i][h][:]   for all h,
 * and the same for v.  A negative slot marks a padding token and is skipped.
 *
 *   k, v           [num_tokens][num_kv_heads][head_dim], contiguous
 *   slot_mapping   int64 [num_tokens]
 * Two tokens naming the same slot in one call is undefined (one of them wins).
 */
pa_status pa_cache_append(void* k_cache, void* v_cache, const void* k, const void* v,
                          const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                          int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                          int32_t* dev_status, void* stream);

/*
 * pa_copy_blocks -- the copy-on-write copy of shared blocks.
 *
 * Defined by [P1] "How PagedAttention borrows OS paging" (sequences sharing a prefix
 * point at the same physical blocks; a new block is allocated when one diverges,
 * as in OS copy-on-write) and [P3] "Why This Matters for Production" (parallel
 * sampling and beam search share KV blocks copy-on-write).  For every layer l and
 * pair p: block pairs[p][1] <- block pairs[p][0], byte for byte, in k_caches[l] and
 * in v_caches[l].
 *
 *   k_caches, v_caches  HOST arrays of num_layers device pointers (one pool per layer)
 *   pairs          device int32 [num_pairs][2] = (src, dst)
 *   block_bytes    bytes of one block of one pool (num_kv_heads*block_size*head_dim*2),
 *                  a multiple of 16
 * A dst that is also a src, or appears twice, in one call is undefined.
 */
pa_status pa_copy_blocks(void* const* k_caches, void* const* v_caches, int num_layers,
                         const int32_t* pairs, int num_pairs, int num_blocks,
                         size_t block_bytes, int32_t* dev_status, void* stream);

/*
 * pa_swap_out_blocks / pa_swap_in_blocks -- the data side of preemption (see
 * pa_bm_swap_out): copy n blocks of every layer's K and V pool to a buffer, or back.
 *
 * Defined by [P1] "Why KV cache memory was the bottleneck" (preempting in-flight
 * requests when the cache runs out).  Buffer layout, block_bytes per block (as in
 * pa_copy_blocks):  buf[layer][pool: 0 = K, 1 = V][i][block_bytes]  for i < n, entry i
 * holding pool block blocks[i]; num_layers * 2 * n * block_bytes bytes in all.
 *
 *   host_dst / host_src  page-locked host memory the device can reach (cudaHostAlloc,
 *                  cudaMallocHost, cudaHostRegister) or device memory, 16-byte aligned;
 *                  pageable host memory is refused (PA_ERR_INVALID), not faulted on.
 *   k_caches, v_caches  HOST arrays of num_layers device pointers (one pool per layer)
 *   blocks         device int32 [n]; an id outside [0, num_blocks) sets PA_DEV_BAD_PAIR
 *                  and that entry is skipped
 * Stream-ordered like every call; the buffer is complete when the stream is.
 */
pa_status pa_swap_out_blocks(void* host_dst, void* const* k_caches, void* const* v_caches,
                             int num_layers, const int32_t* blocks, int n, int num_blocks,
                             size_t block_bytes, int32_t* dev_status, void* stream);
pa_status pa_swap_in_blocks(void* const* k_caches, void* const* v_caches, int num_layers,
                            const int32_t* blocks, int n, int num_blocks, const void* host_src,
                            size_t block_bytes, int32_t* dev_status, void* stream);

/*
 * pa_decode_noalloc -- pa_decode without a caller-provided workspace.
 *
 * The pages have no counterpart for this call; it exists for callers that cannot
 * allocate device memory: a plug-in that runs inside a host serving process whose own
 * allocator owns the device memory (most of it already handed to the KV pools, and
 * raw cudaMalloc forbidden by that host), or a C caller on a path where cudaMalloc
 * with its implicit device synchronisation is not allowed.  Such a caller still
 * passes the inputs and the output; the scratch pa_decode takes as `workspace` lives
 * instead in one fixed array of PA_NOALLOC_SCRATCH_BYTES bytes inside the library's
 * device code.  Every GPU that loads the library holds that array until the process
 * exits.  This call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine).
 *
 * Same arguments, results and errors as pa_decode, minus workspace/workspace_bytes,
 * with these differences:
 *  - The scratch holds the split partials, at head_dim <= 128, of at most 444 CTAs of
 *    the warp-level kernel (3 per SM on a 148-SM B200, the most pa_decode schedules
 *    there) or 148 of the tcgen05 kernel (one per SM, 9 to 64 query rows per kv head):
 *    head_dim above 128 returns PA_ERR_UNSUPPORTED, and a GPU with more SMs is
 *    scheduled with at most those numbers of CTAs.
 *    The batch size does not change the scratch; num_seqs above PA_NOALLOC_MAX_SEQS
 *    returns PA_ERR_INVALID as a stated limit of this call, not of the scratch.
 *  - The first call on a device looks up the device address of the array for that
 *    device (cudaGetSymbolAddress, with that device current) and caches it for the life
 *    of the process; make that first call before any stream capture, and do not use
 *    this call after a cudaDeviceReset of that device (the cached address belongs to
 *    the destroyed context).
 *  - All calls share the one array per device and it keeps whatever the previous call
 *    left there.  Nothing in it needs to start at zero (each call writes every value
 *    it later reads), but two calls that can run at the same time on one device (on
 *    different streams, or from different host threads) race on it and give wrong
 *    results: order them on one stream or with events.
 */
#define PA_NOALLOC_SCRATCH_BYTES 9852160
#define PA_NOALLOC_MAX_SEQS 16384
pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int max_blocks_per_seq, int num_blocks, float scale,
                            pa_dtype dtype, int32_t* dev_status, void* stream);

/* ======================================================================================
 * Host block manager (pa_bm_*): the bookkeeping that produces the kernels' inputs.
 *
 * Defined by [P2] "Core Principle" (logical blocks of a request map to physical blocks
 * through its block table; blocks are allocated on demand and returned to the pool when
 * the request finishes), [P1] "How PagedAttention borrows OS paging" (requests with an
 * identical prefix point their tables at the same physical blocks; a new block is
 * allocated only when a sequence diverges -- copy-on-write), [P3] "How It Works" and
 * "Why This Matters for Production" (parallel sampling and beam search share blocks).
 *
 * Host-only: no call touches a GPU, and every pointer below is a HOST pointer.  A
 * manager owns a pool of num_blocks block ids; free ids are handed out first-in
 * first-out in the order given at creation (NULL: 0, 1, 2, ...), and released ids
 * join the back of that queue.  Sequence ids are assigned 0, 1, 2, ... and never
 * reused.  Not thread-safe: serialise calls on one manager.  Errors change nothing.
 * ====================================================================================== */
typedef struct pa_block_manager pa_block_manager;

/* New manager over block ids 0..num_blocks-1 of block_size tokens each.  free_order,
 * if not NULL, is a permutation of 0..num_blocks-1 (PA_ERR_INVALID otherwise). */
pa_status pa_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                       pa_block_manager** out);
void pa_bm_destroy(pa_block_manager* bm);

/* Free blocks in the pool; the reference count of one block (-1: bad id). */
int pa_bm_free_blocks(const pa_block_manager* bm);
int pa_bm_refcount(const pa_block_manager* bm, int block);

/* A new sequence holding num_tokens cached tokens (a prefill): ceil(num_tokens /
 * block_size) fresh blocks.  PA_ERR_NO_BLOCKS if the pool cannot hold them. */
pa_status pa_bm_allocate(pa_block_manager* bm, int num_tokens, int32_t* seq_id);

/* A new sequence sharing every block of `seq` (each block's count goes up by one). */
pa_status pa_bm_fork(pa_block_manager* bm, int32_t seq, int32_t* child);

/* Reserve the slot of the next token of each of seqs[0..n) in order (a sequence may
 * appear more than once).  For token i: slots[i] = physical block * block_size +
 * offset.  A token that starts a new logical block gets a fresh block; a token that
 * lands in a block shared with other sequences gets a private copy: the pair (shared
 * block, fresh block) is written to cow_pairs[2k], cow_pairs[2k+1] (cow_pairs must
 * hold 2n ints) and *num_cow counts them -- pass them to pa_copy_blocks before
 * pa_cache_append.  If the pool cannot serve the whole batch, returns
 * PA_ERR_NO_BLOCKS and changes nothing. */
pa_status pa_bm_append_tokens(pa_block_manager* bm, const int32_t* seqs, int n, int64_t* slots,
                              int32_t* cow_pairs, int* num_cow);

/* Drop a sequence: every block's count goes down by one; blocks reaching zero return
 * to the back of the free queue. */
pa_status pa_bm_release(pa_block_manager* bm, int32_t seq);

/* Cached tokens / blocks held by a sequence (-1: unknown sequence). */
int64_t pa_bm_context_len(const pa_block_manager* bm, int32_t seq);
int pa_bm_num_blocks_of(const pa_block_manager* bm, int32_t seq);

/* Longest block table among seqs[0..n) (-1: an unknown sequence). */
int pa_bm_max_blocks(const pa_block_manager* bm, const int32_t* seqs, int n);

/* Fill tables[n][width] with the block tables of seqs[0..n) (entries past a table's
 * end = fill) and, if not NULL, context_lens[n].  PA_ERR_INVALID if a table is wider
 * than width or a sequence is unknown. */
pa_status pa_bm_block_tables(const pa_block_manager* bm, const int32_t* seqs, int n, int width,
                             int32_t fill, int32_t* tables, int32_t* context_lens);

/* Flat slot of cached position pos (0 <= pos < context length) of seq. */
pa_status pa_bm_slot_of(const pa_block_manager* bm, int32_t seq, int64_t pos, int64_t* slot);

/*
 * Preemption: swap a sequence's KV out of the pool and back.
 *
 * Defined by [P1] "Why KV cache memory was the bottleneck" (when the cache runs out,
 * in-flight requests are preempted) together with the release rule of [P2] "Core
 * Principle".  pa_bm_swap_out writes seq's blocks in table order to blocks[] (HOST,
 * room for pa_bm_num_blocks_of(seq) entries), sets *num_blocks, and then gives them
 * back exactly as pa_bm_release would (a block shared with another sequence stays with
 * it); seq keeps its id and context length but holds no block.  Save the blocks'
 * contents (pa_swap_out_blocks) before anything can reuse them: enqueue that copy
 * before any later write into the pool on the same stream.  pa_bm_swap_in gives a
 * swapped-out seq ceil(len/block_size) fresh blocks from the front of the free queue,
 * written in table order to blocks[]; restore the saved contents into them
 * (pa_swap_in_blocks) before the sequence is decoded.  A swapped-in sequence shares
 * nothing.  Errors: PA_ERR_INVALID for an unknown sequence, swap_out of a swapped-out
 * one or swap_in of a resident one; PA_ERR_NO_BLOCKS (nothing changed) when the pool
 * cannot hold the blocks.  While swapped out, a sequence is refused by fork,
 * append_tokens, block_tables, slot_of and plan_cascade (PA_ERR_INVALID);
 * pa_bm_context_len still reports its length, pa_bm_num_blocks_of 0, and pa_bm_release
 * drops it.
 */
pa_status pa_bm_swap_out(pa_block_manager* bm, int32_t seq, int32_t* blocks, int* num_blocks);
pa_status pa_bm_swap_in(pa_block_manager* bm, int32_t seq, int32_t* blocks, int* num_blocks);

/*
 * Cascade planning: the inputs pa_decode_cascade takes (prefix_lens, chunk_members,
 * chunk_prefix_lens) for a batch, from its block tables.
 *
 * Defined by [P1] "How PagedAttention borrows OS paging" (requests with an identical
 * prefix point their block tables at the same physical blocks) and [P3] "Why This
 * Matters for Production" (parallel sampling and beam search share blocks).  Batch rows
 * with a non-empty context whose first table entry names the same physical block form a
 * sharing group (groups in order of first appearance, members in row order).  A group's
 * prefix is the leading table entries common to all its members, in tokens, capped at
 * its shortest member's context length; a group of one row, or with a prefix of 0,
 * gets no chunk.  Each group is cut, in row order, into chunks of at most W members
 * (the last padded with -1), all with the group's prefix; prefix_lens[i] is the prefix
 * of row i's chunk, 0 for a row in no chunk.  Identical blocks hold identical K/V, so
 * this is exactly the contract pa_decode_cascade states.
 *
 *   group         q heads per kv head (num_q_heads / num_kv_heads), >= 1
 *   chunk_width   W, members per chunk: group * W must be <= 64 (PA_ERR_UNSUPPORTED
 *                 otherwise).  <= 0 fits W to the batch: with Wmax = max(1, 64 / group),
 *                 W is the largest over sharing groups of ceil(m / ceil(m / Wmax)) for
 *                 a group of m members -- each group in the fewest chunks Wmax allows,
 *                 spread evenly -- or Wmax when no group shares a prefix.  The query
 *                 rows of a chunk are MMA columns, so unused member slots cost work.
 *   prefix_lens   HOST int32 [num_seqs] (written)
 *   chunk_members HOST int32 [num_seqs][W] (written, row stride W: the first
 *                 *num_chunks rows; there are never more chunks than rows; with
 *                 chunk_width <= 0 allocate for W = Wmax)
 *   chunk_prefix_lens  HOST int32 [num_seqs] (written: the first *num_chunks entries)
 *   chunk_width_out    HOST int (written: W), or NULL
 * Host-only, no GPU.  pa_plan_cascade reads the tables (HOST int32
 * [num_seqs][max_blocks_per_seq], each holding ceil(context_lens[i]/block_size) valid
 * entries, else PA_ERR_INVALID); pa_bm_plan_cascade reads the manager's tables of
 * seqs[0..n), batch row i = seqs[i] (PA_ERR_INVALID for an unknown sequence).
 */
pa_status pa_plan_cascade(const int32_t* block_tables, int max_blocks_per_seq,
                          const int32_t* context_lens, int num_seqs, int block_size, int group,
                          int chunk_width, int32_t* prefix_lens, int32_t* chunk_members,
                          int32_t* chunk_prefix_lens, int* num_chunks, int* chunk_width_out);
pa_status pa_bm_plan_cascade(const pa_block_manager* bm, const int32_t* seqs, int n, int group,
                             int chunk_width, int32_t* prefix_lens, int32_t* chunk_members,
                             int32_t* chunk_prefix_lens, int* num_chunks, int* chunk_width_out);

/*
 * pa_check_bounded_waits -- a diagnostic of the bounded waits.  Every wait of a decode
 * kernel's pipeline (a stage barrier, a slot release, the count the block-size-1 V-gather
 * warp keeps) gives up after 2 s, sets PA_DEV_TIMEOUT in dev_status and lets the kernel
 * leave, so a pipeline that cannot finish reports an error instead of hanging the GPU.
 * This call runs the same two wait helpers, on one warp, against a barrier that nothing
 * arrives on and a count that nothing raises, each with a limit of limit_us microseconds.
 *   result    DEVICE int32 [4], 4-byte aligned (written): [0] 1 if the barrier wait gave
 *             up, [1] 1 if the count wait gave up (both 1 when the mechanism works),
 *             [2], [3] how long each wait took, in microseconds
 *   limit_us  1 .. 2,000,000
 * PA_ERR_INVALID for a null or misaligned result or a limit out of range.  Stream-ordered
 * like every call; the GPU stays usable afterwards.
 */
pa_status pa_check_bounded_waits(int32_t* result, int limit_us, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDKV_H */
