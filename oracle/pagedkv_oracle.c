/*
 * pagedkv_oracle.c -- plain, slow, obviously-correct CPU reference for paged
 * KV-cache decode.  TEST INFRASTRUCTURE ONLY: it is called from the tests, from
 * the smoke check and from the CPU-baseline leg of the benchmark, never from the
 * product path.  It shares no code, header, table or constant with the CUDA
 * library; both sides only consume the same seeded inputs.
 *
 * Pages this follows (cited by page title and section):
 *  [P1] "Paged Attention and Memory Efficiency in Production LLM Serving"
 *  [P2] "PagedAttention in Production: Boosting LLM Serving Throughput with
 *       Paged KV Cache"
 *  [P3] "PagedAttention -- The KV Cache Problem"
 *
 * Cache layout (the pages only say "fixed-size blocks"; this is the reading the
 * whole repository uses): one K pool and one V pool per layer, each
 * [num_blocks][num_kv_heads][block_size][head_dim] 16-bit elements.
 * Arithmetic is fp64 after exact conversion of the 16-bit inputs.
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F16 0
#define ORC_BF16 1

/* ---- 16-bit float <-> double, written from the IEEE-754 / bfloat16 bit layouts ---- */

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f | 0x400), e - 25); /* (1024+f) * 2^(e-15-10) */
  return sign ? -v : v;
}

/* bfloat16: the upper half of a binary32 (1 sign, 8 exponent bias 127, 7 fraction). */
double orc_bf16_to_f64(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 7) & 0xff;
  int f = b & 0x7f;
  double v;
  if (e == 0)
    v = ldexp((double)f, -133); /* f * 2^-126 * 2^-7 */
  else if (e == 255)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f | 0x80), e - 134); /* (128+f) * 2^(e-127-7) */
  return sign ? -v : v;
}

/* Round |x| to an integer count of `ulp` units, ties to even (x, ulp exact doubles). */
static double rne_units(double ax, double ulp) {
  double q = ax / ulp; /* exact: ulp is a power of two and no underflow here */
  double fl = floor(q);
  double rem = q - fl;
  if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
  return fl;
}

/* Generic round-to-nearest-even of a double into a binary format with
 * `mant` stored fraction bits, exponent bias `bias`, max biased exponent `emax_b`. */
static uint16_t f64_to_small(double x, int mant, int bias, int ebits) {
  uint16_t sign = signbit(x) ? 1 : 0;
  int top = mant + ebits;                   /* bit position of the sign */
  uint16_t exp_all = (uint16_t)((1 << ebits) - 1);
  if (isnan(x)) return (uint16_t)((sign << top) | (exp_all << mant) | (1 << (mant - 1)));
  double ax = fabs(x);
  int emin = 1 - bias;                      /* smallest normal exponent */
  int emax = exp_all - 1 - bias;            /* largest normal exponent */
  if (ax == 0.0) return (uint16_t)(sign << top);
  int e;
  frexp(ax, &e);                            /* ax = m * 2^e, m in [0.5,1) */
  int unbiased = e - 1;                     /* ax in [2^unbiased, 2^(unbiased+1)) */
  if (unbiased < emin) unbiased = emin;     /* subnormal range uses the emin ulp */
  double ulp = ldexp(1.0, unbiased - mant);
  double n = rne_units(ax, ulp);            /* significand in units of ulp */
  double lim = ldexp(1.0, mant + 1);        /* rounding carried to the next binade */
  if (n >= lim) { n /= 2.0; unbiased += 1; }
  if (unbiased > emax) return (uint16_t)((sign << top) | (exp_all << mant)); /* inf */
  uint32_t sig = (uint32_t)n;
  uint32_t biased;
  if (sig < (1u << mant)) biased = 0;       /* subnormal (only possible at emin) */
  else { biased = (uint32_t)(unbiased + bias); sig -= (1u << mant); }
  return (uint16_t)((sign << top) | (biased << mant) | sig);
}

uint16_t orc_f64_to_f16(double x) { return f64_to_small(x, 10, 15, 5); }
uint16_t orc_f64_to_bf16(double x) { return f64_to_small(x, 7, 127, 8); }

/* ---- 8-bit E4M3 (1 sign, 4 exponent bits with bias 7, 3 fraction bits; no infinity;
 *      S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448) ------- */
double orc_e4m3_to_f64(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 0xf;
  int f = b & 7;
  double v;
  if (e == 15 && f == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)f, -9);              /* subnormal: f/8 * 2^-6 */
  else
    v = ldexp((double)(f | 8), e - 10);    /* (8+f)/8 * 2^(e-7) */
  return sign ? -v : v;
}

/* Round to nearest, ties to even, then clamp magnitudes above 448 to 448 ("satfinite");
 * NaN stays NaN. */
uint8_t orc_f64_to_e4m3(double x) {
  uint8_t sign = signbit(x) ? 0x80 : 0;
  if (isnan(x)) return (uint8_t)(sign | 0x7f);
  double ax = fabs(x);
  if (ax == 0.0) return sign;
  if (isinf(ax)) return (uint8_t)(sign | 0x7e);
  int e;
  frexp(ax, &e);
  int unbiased = e - 1;                    /* ax in [2^unbiased, 2^(unbiased+1)) */
  if (unbiased < -6) unbiased = -6;        /* subnormals share the 2^-9 step */
  if (unbiased > 8) return (uint8_t)(sign | 0x7e);
  double ulp = ldexp(1.0, unbiased - 3);
  double n = rne_units(ax, ulp);           /* significand in units of ulp, 0..16 */
  if (n >= 16.0) { n /= 2.0; unbiased += 1; }
  if (unbiased > 8 || (unbiased == 8 && n > 14.0)) return (uint8_t)(sign | 0x7e);
  uint32_t m = (uint32_t)n;
  if (m < 8) return (uint8_t)(sign | m);   /* subnormal (unbiased == -6) */
  return (uint8_t)(sign | (uint32_t)(unbiased + 7) << 3 | (m - 8));
}

/* The quantised code of a 16-bit cache input for a per-tensor scale: x / scale divided
 * in binary32 (round to nearest), then rounded to E4M3 as above. */
uint8_t orc_quantize_e4m3(uint16_t bits, int dtype, float scale) {
  float xf = (float)(dtype == 1 ? orc_bf16_to_f64(bits) : orc_f16_to_f64(bits));
  volatile float q = xf / scale;
  return orc_f64_to_e4m3((double)q);
}

/* ---- per-(block, kv head) scales of an 8-bit cache.  The pages name an FP8 quantised
 *      KV cache ("PagedAttention -- The KV Cache Problem", "What's Still Unsolved") but
 *      no format; the reading: every (physical block, kv head) slice of a pool has its
 *      own scale, fixed by the token written at offset 0 of the block (the first token a
 *      block ever receives, since blocks fill in order): with amax the largest |x| of that
 *      token's row for the head and y = amax / 448 in binary32, the scale is the power of
 *      two 2^(ceil(log2 y) + 3) -- the smallest power of two that maps the row into
 *      E4M3's range, times 8 of headroom for later tokens of the block (larger ones
 *      saturate).  amax of 0 (or not finite) gives scale 1.  A power of two keeps x / scale
 *      exact, so the code is the E4M3 rounding of the scaled value. ----------------- */
float orc_e4m3_block_scale(float amax) {
  volatile float y = amax / 448.0f;
  if (!(y > 0.0f) || isinf(y)) return 1.0f;
  int e;
  float m = frexpf(y, &e);                 /* y = m 2^e, m in [0.5, 1) */
  int c = (m == 0.5f) ? e - 1 : e;         /* ceil(log2 y) */
  c += 3;
  if (c < -126) c = -126;
  if (c > 127) c = 127;
  return ldexpf(1.0f, c);
}

static double to_f64(uint16_t v, int dtype) {
  return dtype == ORC_BF16 ? orc_bf16_to_f64(v) : orc_f16_to_f64(v);
}
static uint16_t from_f64(double v, int dtype) {
  return dtype == ORC_BF16 ? orc_f64_to_bf16(v) : orc_f64_to_f16(v);
}

/* ---- sizing identity: [P1] "Why KV cache memory was the bottleneck..."; [P2]
 *      "Misconception 3" formula with hidden = kv_heads * head_dim ----------------- */
int64_t orc_kv_bytes_per_token(int layers, int kv_heads, int head_dim, int elem_bytes) {
  return (int64_t)layers * 2 /* K and V */ * kv_heads * head_dim * elem_bytes;
}

/* ---- block-table resolve: [P2] "Core Principle" (logical block -> physical block
 *      through the block table), [P3] "How It Works" (the kernel reads the block table
 *      to gather KV from non-contiguous blocks) ------------------------------------ */
/* Element offset of (physical block b, kv head h, in-block offset o, dim 0). */
static int64_t cache_row(int64_t b, int h, int o, int Hkv, int bs, int D) {
  return ((b * Hkv + h) * (int64_t)bs + o) * D;
}

/* Gather the logical rows 0..ctx-1 of one sequence and kv head into out[ctx][D] (fp64).
 * cache_dtype ORC_F16 / ORC_BF16: 16-bit elements; ORC_E4M3: 8-bit codes, each value
 * multiplied by `scale` (the per-tensor dequantisation scale).
 * Returns 0, or -1 if a needed block-table entry lies outside [0, num_blocks). */
#define ORC_E4M3 2
int orc_gather_any(double* out, const void* cache, int cache_dtype, double scale,
                   int num_blocks, int Hkv, int bs, int D, const int32_t* table_row, int ctx,
                   int kvh) {
  for (int t = 0; t < ctx; ++t) {
    int32_t b = table_row[t / bs];          /* logical block t/bs -> physical block */
    int o = t % bs;                         /* position inside the block */
    if (b < 0 || b >= num_blocks) return -1;
    int64_t r = cache_row(b, kvh, o, Hkv, bs, D);
    for (int d = 0; d < D; ++d) {
      double v;
      if (cache_dtype == ORC_E4M3)
        v = scale * orc_e4m3_to_f64(((const uint8_t*)cache)[r + d]);
      else
        v = to_f64(((const uint16_t*)cache)[r + d], cache_dtype);
      out[(int64_t)t * D + d] = v;
    }
  }
  return 0;
}

int orc_gather(double* out, const uint16_t* cache, int dtype, int num_blocks, int Hkv,
               int bs, int D, const int32_t* table_row, int ctx, int kvh) {
  return orc_gather_any(out, cache, dtype, 1.0, num_blocks, Hkv, bs, D, table_row, ctx, kvh);
}

/* Gather over an 8-bit cache with per-(block, kv head) scales bscale[b][kvh]. */
static int gather_block_scaled(double* out, const uint8_t* cache, const float* bscale,
                               int num_blocks, int Hkv, int bs, int D, const int32_t* table_row,
                               int ctx, int kvh) {
  for (int t = 0; t < ctx; ++t) {
    int32_t b = table_row[t / bs];
    int o = t % bs;
    if (b < 0 || b >= num_blocks) return -1;
    double sc = (double)bscale[(int64_t)b * Hkv + kvh];
    int64_t r = cache_row(b, kvh, o, Hkv, bs, D);
    for (int d = 0; d < D; ++d) out[(int64_t)t * D + d] = sc * orc_e4m3_to_f64(cache[r + d]);
  }
  return 0;
}

/* ---- decode attention: [P1] "How PagedAttention borrows OS paging" -- the math is
 *      the plain dot products, softmax and value-weighted sum, only the storage is
 *      paged; so this is softmax(scale * q K^T) V over the gathered rows.
 *      Several new tokens per sequence (q_len > 1): [P1] "Why KV cache memory was the
 *      bottleneck" -- a generated token uses the keys and values of every token before
 *      it.  The q_len new tokens occupy the last q_len cached positions, so new token j
 *      (position ctx - q_len + j) attends to positions 0 .. ctx - q_len + j, i.e. to the
 *      first n_j = ctx - q_len + 1 + j rows; n_j <= 0 gives an all-zero output row. -- */
typedef struct {
  double* out64;
  uint16_t* out16;
  const uint16_t* q;
  const void *k_cache, *v_cache;
  const int32_t *block_tables, *context_lens, *items;
  int n_items, q_len, Hq, Hkv, D, bs, max_blocks, num_blocks, dtype;
  int cache_dtype;                          /* dtype, or ORC_E4M3 with the scales below */
  double k_scale, v_scale;
  const float *k_bscale, *v_bscale;         /* E4M3 with per-(block, kv head) scales */
  double scale;
  atomic_int next;
  atomic_int err;
} decode_job;

static void decode_one(decode_job* J, int s, int j, int h, double* kbuf, double* vbuf, double* w) {
  int D = J->D;
  int group = J->Hq / J->Hkv;
  int kvh = h / group;                      /* consecutive q heads share one kv head */
  int ctx = J->context_lens[s];
  int n = ctx - J->q_len + 1 + j;           /* rows this query token attends to */
  int64_t row = ((int64_t)s * J->q_len + j) * J->Hq + h;
  double* o64 = J->out64 + row * D;
  for (int d = 0; d < D; ++d) o64[d] = 0.0;
  if (n > 0) {
    const int32_t* table_row = J->block_tables + (int64_t)s * J->max_blocks;
    int bad;
    if (J->k_bscale)
      bad = gather_block_scaled(kbuf, (const uint8_t*)J->k_cache, J->k_bscale, J->num_blocks,
                                J->Hkv, J->bs, D, table_row, n, kvh) ||
            gather_block_scaled(vbuf, (const uint8_t*)J->v_cache, J->v_bscale, J->num_blocks,
                                J->Hkv, J->bs, D, table_row, n, kvh);
    else
      bad = orc_gather_any(kbuf, J->k_cache, J->cache_dtype, J->k_scale, J->num_blocks, J->Hkv,
                           J->bs, D, table_row, n, kvh) ||
            orc_gather_any(vbuf, J->v_cache, J->cache_dtype, J->v_scale, J->num_blocks, J->Hkv,
                           J->bs, D, table_row, n, kvh);
    if (bad) {
      atomic_store(&J->err, 1);
      return;
    }
    const uint16_t* qrow = J->q + row * D;
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {           /* x_t = scale * <q, k_t> */
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += to_f64(qrow[d], J->dtype) * kbuf[(int64_t)t * D + d];
      w[t] = J->scale * acc;
      if (w[t] > m) m = w[t];
    }
    double l = 0.0;
    for (int t = 0; t < n; ++t) { w[t] = exp(w[t] - m); l += w[t]; }
    for (int t = 0; t < n; ++t)
      for (int d = 0; d < D; ++d) o64[d] += w[t] * vbuf[(int64_t)t * D + d];
    for (int d = 0; d < D; ++d) o64[d] /= l;
  }
  if (J->out16) {
    uint16_t* o16 = J->out16 + row * D;
    for (int d = 0; d < D; ++d) o16[d] = from_f64(o64[d], J->dtype);
  }
}

static int max_ctx_of(decode_job* J) {
  int mx = 0;
  for (int i = 0; i < J->n_items; ++i) {
    int s = J->items ? J->items[i] : i;
    if (J->context_lens[s] > mx) mx = J->context_lens[s];
  }
  return mx;
}

static void* decode_worker(void* arg) {
  decode_job* J = (decode_job*)arg;
  int mx = max_ctx_of(J);
  size_t n = (size_t)(mx > 0 ? mx : 1);
  double* kbuf = (double*)malloc(n * J->D * sizeof(double));
  double* vbuf = (double*)malloc(n * J->D * sizeof(double));
  double* w = (double*)malloc(n * sizeof(double));
  if (!kbuf || !vbuf || !w) { atomic_store(&J->err, 2); free(kbuf); free(vbuf); free(w); return NULL; }
  int per_seq = J->q_len * J->Hq;
  int total = J->n_items * per_seq;         /* work item = (sequence, new token, q head) */
  for (;;) {
    int it = atomic_fetch_add(&J->next, 1);
    if (it >= total) break;
    int i = it / per_seq, r = it % per_seq;
    int s = J->items ? J->items[i] : i;
    decode_one(J, s, r / J->Hq, r % J->Hq, kbuf, vbuf, w);
  }
  free(kbuf); free(vbuf); free(w);
  return NULL;
}

/* q and out64 are [B][q_len][Hq][D] (out16, if not NULL, gets the round-to-nearest-even
 * 16-bit copy).  `items` (nullable) restricts the work to the listed sequences (sampled
 * checks); rows of other sequences are left untouched.  Returns 0, -1 on a bad block
 * id, -2 on bad arguments or allocation failure. */
static int run_decode(decode_job* J, int B, int nthreads);

/* Decode over an 8-bit E4M3 cache: q and out as for orc_decode_multi (16-bit dtype), the
 * cache values are k_scale * code and v_scale * code. */
int orc_decode_e4m3(double* out64, uint16_t* out16, const uint16_t* q, const uint8_t* k_cache,
                    const uint8_t* v_cache, double k_scale, double v_scale,
                    const int32_t* block_tables, const int32_t* context_lens, int B, int q_len,
                    int Hq, int Hkv, int D, int bs, int max_blocks, int num_blocks, double scale,
                    int dtype, const int32_t* items, int n_items, int nthreads) {
  if (B < 0 || q_len < 1 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0) return -2;
  decode_job J;
  J.out64 = out64; J.out16 = out16; J.q = q; J.k_cache = k_cache; J.v_cache = v_cache;
  J.cache_dtype = ORC_E4M3; J.k_scale = k_scale; J.v_scale = v_scale;
  J.k_bscale = NULL; J.v_bscale = NULL;
  J.block_tables = block_tables; J.context_lens = context_lens;
  J.items = items; J.n_items = items ? n_items : B;
  J.q_len = q_len; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.bs = bs; J.max_blocks = max_blocks;
  J.num_blocks = num_blocks; J.dtype = dtype; J.scale = scale;
  return run_decode(&J, B, nthreads);
}

/* Decode over an 8-bit E4M3 cache with per-(block, kv head) scales: the cached value of
 * (block b, kv head h) is k_bscale[b][h] * code (v likewise); q and out as for
 * orc_decode_multi. */
int orc_decode_e4m3_bs(double* out64, uint16_t* out16, const uint16_t* q, const uint8_t* k_cache,
                       const uint8_t* v_cache, const float* k_bscale, const float* v_bscale,
                       const int32_t* block_tables, const int32_t* context_lens, int B, int q_len,
                       int Hq, int Hkv, int D, int bs, int max_blocks, int num_blocks, double scale,
                       int dtype, const int32_t* items, int n_items, int nthreads) {
  if (B < 0 || q_len < 1 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || !k_bscale ||
      !v_bscale)
    return -2;
  decode_job J;
  J.out64 = out64; J.out16 = out16; J.q = q; J.k_cache = k_cache; J.v_cache = v_cache;
  J.cache_dtype = ORC_E4M3; J.k_scale = 1.0; J.v_scale = 1.0;
  J.k_bscale = k_bscale; J.v_bscale = v_bscale;
  J.block_tables = block_tables; J.context_lens = context_lens;
  J.items = items; J.n_items = items ? n_items : B;
  J.q_len = q_len; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.bs = bs; J.max_blocks = max_blocks;
  J.num_blocks = num_blocks; J.dtype = dtype; J.scale = scale;
  return run_decode(&J, B, nthreads);
}

int orc_decode_multi(double* out64, uint16_t* out16, const uint16_t* q, const uint16_t* k_cache,
                     const uint16_t* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, int B, int q_len, int Hq, int Hkv, int D, int bs,
                     int max_blocks, int num_blocks, double scale, int dtype, const int32_t* items,
                     int n_items, int nthreads) {
  if (B < 0 || q_len < 1 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0) return -2;
  decode_job J;
  J.out64 = out64; J.out16 = out16; J.q = q; J.k_cache = k_cache; J.v_cache = v_cache;
  J.cache_dtype = dtype; J.k_scale = 1.0; J.v_scale = 1.0;
  J.k_bscale = NULL; J.v_bscale = NULL;
  J.block_tables = block_tables; J.context_lens = context_lens;
  J.items = items; J.n_items = items ? n_items : B;
  J.q_len = q_len; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.bs = bs; J.max_blocks = max_blocks;
  J.num_blocks = num_blocks; J.dtype = dtype; J.scale = scale;
  return run_decode(&J, B, nthreads);
}

static int run_decode(decode_job* J, int B, int nthreads) {
  atomic_init(&J->next, 0);
  atomic_init(&J->err, 0);
  for (int i = 0; i < J->n_items; ++i) {
    int s = J->items ? J->items[i] : i;
    if (s < 0 || s >= B) return -2;
    if (J->context_lens[s] < 0 || (int64_t)J->context_lens[s] > (int64_t)J->max_blocks * J->bs)
      return -2;
  }
  if (nthreads < 1) nthreads = 1;
  if (nthreads == 1) {
    decode_worker(J);
  } else {
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    if (!th) return -2;
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, decode_worker, J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
  }
  int e = atomic_load(&J->err);
  return e == 1 ? -1 : (e ? -2 : 0);
}

/* One new token per sequence: q and out are [B][Hq][D]. */
int orc_decode(double* out64, uint16_t* out16, const uint16_t* q, const uint16_t* k_cache,
               const uint16_t* v_cache, const int32_t* block_tables, const int32_t* context_lens,
               int B, int Hq, int Hkv, int D, int bs, int max_blocks, int num_blocks,
               double scale, int dtype, const int32_t* items, int n_items, int nthreads) {
  return orc_decode_multi(out64, out16, q, k_cache, v_cache, block_tables, context_lens, B, 1, Hq,
                          Hkv, D, bs, max_blocks, num_blocks, scale, dtype, items, n_items,
                          nthreads);
}

/* ---- cache append: [P1] "How PagedAttention borrows OS paging" (blocks are filled
 *      on demand as decoding proceeds), [P3] "How It Works" (allocate blocks on
 *      demand).  Token i goes to flat slot s = physical_block*block_size + offset;
 *      a negative slot is a padding token and is skipped. ----------------------- */
int orc_cache_append(uint16_t* k_cache, uint16_t* v_cache, const uint16_t* k, const uint16_t* v,
                     const int64_t* slots, int T, int Hkv, int D, int bs, int num_blocks) {
  for (int i = 0; i < T; ++i) {
    int64_t s = slots[i];
    if (s < 0) continue;
    if (s >= (int64_t)num_blocks * bs) return -1;
    int64_t b = s / bs;
    int o = (int)(s % bs);
    for (int h = 0; h < Hkv; ++h) {
      int64_t dst = cache_row(b, h, o, Hkv, bs, D);
      int64_t src = ((int64_t)i * Hkv + h) * D;
      memcpy(k_cache + dst, k + src, (size_t)D * sizeof(uint16_t));
      memcpy(v_cache + dst, v + src, (size_t)D * sizeof(uint16_t));
    }
  }
  return 0;
}

/* Quantising append into 8-bit E4M3 caches: for every token i with slot >= 0, the codes
 * orc_quantize_e4m3(k[i][h][d], dtype, k_scale) (and likewise v) go to
 * [slot/bs][h][slot%bs][d]; a negative slot is skipped. */
int orc_cache_append_e4m3(uint8_t* k_cache, uint8_t* v_cache, const uint16_t* k, const uint16_t* v,
                          const int64_t* slots, int T, int Hkv, int D, int bs, int num_blocks,
                          int dtype, float k_scale, float v_scale) {
  for (int i = 0; i < T; ++i) {
    int64_t s = slots[i];
    if (s < 0) continue;
    if (s >= (int64_t)num_blocks * bs) return -1;
    int64_t b = s / bs;
    int o = (int)(s % bs);
    for (int h = 0; h < Hkv; ++h) {
      int64_t dst = cache_row(b, h, o, Hkv, bs, D);
      int64_t src = ((int64_t)i * Hkv + h) * D;
      for (int d = 0; d < D; ++d) {
        k_cache[dst + d] = orc_quantize_e4m3(k[src + d], dtype, k_scale);
        v_cache[dst + d] = orc_quantize_e4m3(v[src + d], dtype, v_scale);
      }
    }
  }
  return 0;
}

/* ---- copy-on-write block copy: [P1] "How PagedAttention borrows OS paging" (a new
 *      block is allocated once a sequence diverges from a shared prefix, as in OS
 *      copy-on-write), [P3] "Why This Matters" (parallel sampling / beam search share
 *      blocks copy-on-write).  For every layer and pair: dst block <- src block, K and V. */
int orc_copy_blocks(uint16_t** k_caches, uint16_t** v_caches, int L, const int32_t* pairs,
                    int n_pairs, int64_t block_elems, int num_blocks) {
  for (int p = 0; p < n_pairs; ++p) {
    int32_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return -1;
  }
  for (int l = 0; l < L; ++l)
    for (int p = 0; p < n_pairs; ++p) {
      int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
      memcpy(k_caches[l] + dst * block_elems, k_caches[l] + src * block_elems,
             (size_t)block_elems * sizeof(uint16_t));
      memcpy(v_caches[l] + dst * block_elems, v_caches[l] + src * block_elems,
             (size_t)block_elems * sizeof(uint16_t));
    }
  return 0;
}

/* Quantising append into 8-bit pools with per-(block, kv head) scales (see
 * orc_e4m3_block_scale).  First, every token whose slot is offset 0 of its block fixes
 * that block's scales from its own rows (k_bscale[b][h] from k[i][h][:], v likewise);
 * then every token's values are quantised with its block's scales, exactly as
 * orc_quantize_e4m3 does for one scale.  Blocks whose offset 0 is not written here keep
 * their scales.  Negative slots are padding.  Returns 0, or -1 on a slot outside the pool. */
int orc_cache_append_e4m3_bs(uint8_t* k_cache, uint8_t* v_cache, float* k_bscale,
                             float* v_bscale, const uint16_t* k, const uint16_t* v,
                             const int64_t* slots, int T, int Hkv, int D, int bs, int num_blocks,
                             int dtype) {
  for (int i = 0; i < T; ++i)
    if (slots[i] >= (int64_t)num_blocks * bs) return -1;
  for (int i = 0; i < T; ++i) {
    int64_t s = slots[i];
    if (s < 0 || s % bs) continue;
    int64_t b = s / bs;
    for (int h = 0; h < Hkv; ++h) {
      int64_t src = ((int64_t)i * Hkv + h) * D;
      float ak = 0.0f, av = 0.0f;
      for (int d = 0; d < D; ++d) {
        float xk = fabsf((float)to_f64(k[src + d], dtype));
        float xv = fabsf((float)to_f64(v[src + d], dtype));
        if (xk > ak) ak = xk;
        if (xv > av) av = xv;
      }
      k_bscale[b * Hkv + h] = orc_e4m3_block_scale(ak);
      v_bscale[b * Hkv + h] = orc_e4m3_block_scale(av);
    }
  }
  for (int i = 0; i < T; ++i) {
    int64_t s = slots[i];
    if (s < 0) continue;
    int64_t b = s / bs;
    int o = (int)(s % bs);
    for (int h = 0; h < Hkv; ++h) {
      int64_t dst = cache_row(b, h, o, Hkv, bs, D);
      int64_t src = ((int64_t)i * Hkv + h) * D;
      float sk = k_bscale[b * Hkv + h], sv = v_bscale[b * Hkv + h];
      for (int d = 0; d < D; ++d) {
        k_cache[dst + d] = orc_quantize_e4m3(k[src + d], dtype, sk);
        v_cache[dst + d] = orc_quantize_e4m3(v[src + d], dtype, sv);
      }
    }
  }
  return 0;
}
