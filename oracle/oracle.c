/*
 * oracle.c -- plain, slow, single-threaded CPU oracle for paged KV-cache decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this file's library.  The product
 * (the CUDA library) never calls it, shares no code, header, table or helper
 * with it, and must fail loudly rather than fall back to it.
 *
 * Every floating-point result is computed in fp64.  Every loop runs in the
 * logical order of the definition it follows; there is no blocking, fusion or
 * split-context reordering here.
 *
 * Sources (web pages on KV cache / PagedAttention), cited by title + section:
 *  [Dissect]  "深度解构 LLM 推理优化：从 KV Cache 冗余到 PagedAttention 内存分页映射"
 *  [Evolve]   "现代 AI 的“推理加速之谜”：从 KV Cache 到 PagedAttention 的演进"
 *  [MemMgmt]  "KVCache技术背景与核心挑战 / PageAttention内存管理机制" (intelliparadigm)
 *  [vLLMNote] "vLLM 推理原理 从 KV Cache 到分页与连续批处理"
 * Number formats: bfloat16 (1-8-7, bias 127), OCP 8-bit float E4M3
 * (1-4-3, bias 7, no infinities, S.1111.111 = NaN, max finite 448) and
 * symmetric INT8 (two's complement codes -127..127, value = code x scale).
 * Cache element types are numbered 0 = bf16, 1 = E4M3, 2 = INT8; a quantised
 * cache has one fp32 scale per KV head (a per-tensor scale is the case of
 * equal per-head scales).
 *
 * Pins (what ties each function to something other than itself) live in
 * tests/test_oracle_pins.py; every function below is pinned there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bfloat16 -> value: a bf16 is the upper half of an IEEE binary32. Exact. */
double or_bf16_decode(uint16_t b) { return (double)bits_to_f32((uint32_t)b << 16); }

/* binary32 -> bfloat16, round to nearest, ties to even, on the 16 discarded
 * bits.  NaN stays NaN (quiet, sign kept); overflow rounds to infinity as RNE
 * prescribes. */
uint16_t or_bf16_encode_rne(float x)
{
    uint32_t u = f32_to_bits(x);
    if (isnan(x)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16;
    uint32_t rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

/* E4M3 -> value (exact).  Exponent field 0 is subnormal: m * 2^-9.
 * Exponent field e>0: 2^(e-7) * (1 + m/8).  S.1111.111 is NaN. */
double or_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* value (binary32) -> E4M3, round to nearest even, saturating to +-448
 * (the "satfinite" conversion: anything beyond the largest finite value,
 * infinities included, becomes +-448; NaN stays NaN). */
uint8_t or_e4m3_encode_satfinite(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* Spacing of representable values around a: 2^-9 below the smallest
     * normal 2^-6, else 2^(E-3) in the binade [2^E, 2^(E+1)). */
    double quantum;
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);
    } else {
        int E;
        frexp(a, &E);               /* a = f * 2^E, f in [0.5, 1) */
        quantum = ldexp(1.0, (E - 1) - 3);
    }
    double k = rint(a / quantum);   /* exact division (power of 2); rint = RNE */
    double v = k * quantum;
    if (v >= 448.0) return (uint8_t)(sign | 0x7E);   /* not reachable below 448, kept for clarity */
    if (v == 0.0) return sign;
    uint8_t code;
    if (v < ldexp(1.0, -6)) {
        code = (uint8_t)(int)(v / ldexp(1.0, -9));  /* subnormal mantissa 1..7 */
    } else {
        int E;
        double f = frexp(v, &E);    /* v = (2f) * 2^(E-1), 2f in [1, 2) */
        int e = (E - 1) + 7;
        int m = (int)((2.0 * f - 1.0) * 8.0);
        code = (uint8_t)((e << 3) | m);
    }
    return (uint8_t)(sign | code);
}

/* IEEE binary32 division x / s, correctly rounded (the quantisation input). */
float or_div_f32(float x, float s)
{
    volatile float r = x / s;
    return r;
}

/* Symmetric INT8 code of a binary32 value: the nearest integer, ties to the
 * even one, limited to [-127, 127] (-128 is never produced, so the range is
 * symmetric about zero); NaN gives 0.  The value of a code is code x scale.
 * [Dissect] section 4 item 1 and [Evolve] section 3.C name INT8 KV
 * quantisation; the rounding, the symmetric range and the NaN rule are the
 * readings adopted where the pages give no scheme. */
int8_t or_int8_encode_sat(float x)
{
    if (x != x) return 0;
    if (x >= 127.0f) return 127;
    if (x <= -127.0f) return -127;
    double f = floor((double)x);        /* exact: |x| < 127 */
    double frac = (double)x - f;        /* exact, in [0, 1) */
    double r;
    if (frac > 0.5) r = f + 1.0;
    else if (frac < 0.5) r = f;
    else r = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;   /* tie: the even neighbour */
    return (int8_t)r;
}

double or_int8_decode(int8_t c) { return (double)c; }

/* ------------------------------------------------------------------------ */
/* Closed forms                                                              */
/* ------------------------------------------------------------------------ */

/* Per-token KV bytes: 2 (K and V) x layers x KV heads x head dim x bytes per
 * element.  [Dissect] section 1.1 (显存占用的精确量化), per-token memory
 * equation; [Evolve] section 2 (计算公式). */
uint64_t or_kv_bytes_per_token(int layers, int h_kv, int head_dim, int elem_bytes)
{
    return 2ull * (uint64_t)layers * (uint64_t)h_kv * (uint64_t)head_dim * (uint64_t)elem_bytes;
}

/* KV bytes of one sequence holding T cached tokens: 2 x L x T x H_KV x d_h x b.
 * [vLLMNote] section "KV Cache 缓存的究竟是什么", the M_KV estimate. */
uint64_t or_kv_bytes_sequence(int layers, uint64_t tokens, int h_kv, int head_dim, int elem_bytes)
{
    return (uint64_t)tokens * or_kv_bytes_per_token(layers, h_kv, head_dim, elem_bytes);
}

/* ------------------------------------------------------------------------ */
/* Cache layout used by both sides' data (a documented layout, not shared      */
/* code): cache[NB][H_kv][bs][d], elements of 2 bytes (bf16) or 1 (E4M3).      */
/* ------------------------------------------------------------------------ */

static size_t cache_index(int64_t blk, int h, int off, int i, int h_kv, int bs, int d)
{
    return (((size_t)blk * h_kv + h) * bs + off) * d + i;
}

/* Store the new step's K and V rows into their physical slots.
 * A token's slot is phys_block * bs + offset; slot < 0 means "no write"
 * (padding).  bf16 caches receive the input bits unchanged.  E4M3 caches
 * receive enc(x / scale) with an fp32 division and a saturating RNE encode;
 * INT8 caches the same with the INT8 encode.  scale = k_scales[h] (resp.
 * v_scales[h]) for KV head h; the scale arrays are not read for bf16.
 * [Evolve] section 1 (every step computes only the new token's Q, K, V and
 * keeps K, V in the cache); [vLLMNote] section "KV Cache 缓存的究竟是什么";
 * [Dissect] section 3.2 (FP8 KV cache quantisation) and section 4 item 1
 * (INT8/FP8 KV quantisation).
 * Returns 0, -1 if a slot lies outside the pool, -5 on an unknown type. */
int or_reshape_and_cache(const uint16_t *key, const uint16_t *value,
                         void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int T,
                         int h_kv, int d, int bs, int num_blocks,
                         int cache_dtype, const float *k_scales, const float *v_scales)
{
    if (cache_dtype < 0 || cache_dtype > 2) return -5;
    for (int t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t blk = slot / bs;
        int off = (int)(slot % bs);
        if (blk >= num_blocks) return -1;
        for (int h = 0; h < h_kv; ++h) {
            for (int i = 0; i < d; ++i) {
                size_t src = ((size_t)t * h_kv + h) * d + i;
                size_t dst = cache_index(blk, h, off, i, h_kv, bs, d);
                if (cache_dtype == 1) {
                    float kx = (float)or_bf16_decode(key[src]);
                    float vx = (float)or_bf16_decode(value[src]);
                    ((uint8_t *)k_cache)[dst] = or_e4m3_encode_satfinite(or_div_f32(kx, k_scales[h]));
                    ((uint8_t *)v_cache)[dst] = or_e4m3_encode_satfinite(or_div_f32(vx, v_scales[h]));
                } else if (cache_dtype == 2) {
                    float kx = (float)or_bf16_decode(key[src]);
                    float vx = (float)or_bf16_decode(value[src]);
                    ((int8_t *)k_cache)[dst] = or_int8_encode_sat(or_div_f32(kx, k_scales[h]));
                    ((int8_t *)v_cache)[dst] = or_int8_encode_sat(or_div_f32(vx, v_scales[h]));
                } else {
                    ((uint16_t *)k_cache)[dst] = key[src];
                    ((uint16_t *)v_cache)[dst] = value[src];
                }
            }
        }
    }
    return 0;
}

/* Copy-on-write block copy: for every (src, dst) pair and every layer, the
 * whole physical block of K and of V is copied byte for byte.
 * [Dissect] section 2.3 (CoW on the first divergent write);
 * [MemMgmt] section 3.1 (Copy-on-Write: copy the block, update the mapping).
 * block_bytes = H_kv * bs * d * element size.  Returns 0, or -1 on a bad id. */
int or_copy_blocks(uint8_t *const *k_caches, uint8_t *const *v_caches, int num_layers,
                   const int64_t *pairs, int n, uint64_t block_bytes, int num_blocks)
{
    for (int p = 0; p < n; ++p) {
        int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) return -1;
        for (int l = 0; l < num_layers; ++l) {
            for (uint64_t b = 0; b < block_bytes; ++b) {
                k_caches[l][(uint64_t)dst * block_bytes + b] = k_caches[l][(uint64_t)src * block_bytes + b];
                v_caches[l][(uint64_t)dst * block_bytes + b] = v_caches[l][(uint64_t)src * block_bytes + b];
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode attention                                                           */
/* ------------------------------------------------------------------------ */

/* Value of a cache element: bf16 exactly; a quantised code times its scale. */
static double cache_elem(const void *cache, size_t idx, int cache_dtype, double scale)
{
    if (cache_dtype == 1) return or_e4m3_decode(((const uint8_t *)cache)[idx]) * scale;
    if (cache_dtype == 2) return or_int8_decode(((const int8_t *)cache)[idx]) * scale;
    return or_bf16_decode(((const uint16_t *)cache)[idx]);
}

/* One decode-step output row: out = softmax(scale * q . K^T) . V for query
 * head h of sequence s, with K/V being the sequence's first ctx[s] cached
 * tokens in logical order, each found through the block table:
 * token t lives in physical block table[s][t / bs] at offset t % bs.
 * Query head h reads KV head h / (H_q / H_kv) (contiguous grouping).
 * ctx = 0 gives a zero row.  Quantised caches are read as code x the KV
 * head's scale (k_scales[kvh], v_scales[kvh]), in fp64.
 * [Evolve] section 1 (Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V);
 * [Dissect] section 2.1 (block table: logical -> physical block);
 * [vLLMNote] section "PagedAttention 怎样整理这些缓存" (A's logical blocks map
 * to physical 2, 5, 1; the last block may be partly filled);
 * [Dissect] section 1.1 and [Evolve] section 3.A (GQA: query heads share KV
 * heads group-wise).
 * Returns 0, -1 on an out-of-pool block id, -2 on a context longer than the
 * table row. */
static int decode_one(double *out_row, int s, int h,
                      const uint16_t *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *context_lens,
                      int h_q, int h_kv, int d, int bs, int num_blocks,
                      double scale, int cache_dtype, const float *k_scales, const float *v_scales)
{
    int g = h_q / h_kv;
    int kvh = h / g;
    double k_scale = cache_dtype ? (double)k_scales[kvh] : 1.0;
    double v_scale = cache_dtype ? (double)v_scales[kvh] : 1.0;
    int n = context_lens[s];
    for (int i = 0; i < d; ++i) out_row[i] = 0.0;
    if (n <= 0) return 0;
    if ((n + bs - 1) / bs > max_blocks_per_seq) return -2;

    const uint16_t *qrow = q + ((size_t)s * h_q + h) * d;
    double *logit = (double *)malloc(sizeof(double) * (size_t)n);
    if (!logit) return -3;

    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        int32_t phys = block_tables[(size_t)s * max_blocks_per_seq + t / bs];
        if (phys < 0 || phys >= num_blocks) { free(logit); return -1; }
        int off = t % bs;
        double dot = 0.0;
        for (int i = 0; i < d; ++i)
            dot += or_bf16_decode(qrow[i]) *
                   cache_elem(k_cache, cache_index(phys, kvh, off, i, h_kv, bs, d), cache_dtype, k_scale);
        logit[t] = scale * dot;
        if (logit[t] > m) m = logit[t];
    }
    double denom = 0.0;
    for (int t = 0; t < n; ++t) {
        double w = exp(logit[t] - m);
        int32_t phys = block_tables[(size_t)s * max_blocks_per_seq + t / bs];
        int off = t % bs;
        denom += w;
        for (int i = 0; i < d; ++i)
            out_row[i] += w * cache_elem(v_cache, cache_index(phys, kvh, off, i, h_kv, bs, d), cache_dtype, v_scale);
    }
    for (int i = 0; i < d; ++i) out_row[i] /= denom;
    free(logit);
    return 0;
}

/* All rows: out[B][H_q][d] (fp64). */
int or_paged_decode(double *out, const uint16_t *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                    int B, int h_q, int h_kv, int d, int bs, int num_blocks,
                    double scale, int cache_dtype, const float *k_scales, const float *v_scales)
{
    if (h_kv <= 0 || h_q % h_kv != 0) return -4;
    if (cache_dtype < 0 || cache_dtype > 2) return -5;
    /* Rows are independent.  Built with -fopenmp (the second, multi-core baseline library)
     * they are shared out over the host's threads; built without it the pragma is ignored and
     * the loop runs in order on one thread.  Either way each row's arithmetic is the same. */
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int s = 0; s < B; ++s)
        for (int h = 0; h < h_q; ++h) {
            int rc = decode_one(out + ((size_t)s * h_q + h) * d, s, h, q, k_cache, v_cache,
                                block_tables, max_blocks_per_seq, context_lens, h_q, h_kv, d, bs,
                                num_blocks, scale, cache_dtype, k_scales, v_scales);
            if (rc) {
#pragma omp atomic write
                err = rc;
            }
        }
    return err;
}

/* Selected rows only: pairs[2*i] = sequence, pairs[2*i+1] = query head;
 * out[i][d] (fp64).  Same arithmetic as or_paged_decode. */
int or_paged_decode_rows(double *out, const int32_t *pairs, int npairs,
                         const uint16_t *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                         int h_q, int h_kv, int d, int bs, int num_blocks,
                         double scale, int cache_dtype, const float *k_scales, const float *v_scales)
{
    if (h_kv <= 0 || h_q % h_kv != 0) return -4;
    if (cache_dtype < 0 || cache_dtype > 2) return -5;
    int err = 0;   /* as in or_paged_decode: rows over threads only in the -fopenmp build */
#pragma omp parallel for schedule(dynamic)
    for (int i = 0; i < npairs; ++i) {
        int rc = decode_one(out + (size_t)i * d, pairs[2 * i], pairs[2 * i + 1], q, k_cache, v_cache,
                            block_tables, max_blocks_per_seq, context_lens, h_q, h_kv, d, bs,
                            num_blocks, scale, cache_dtype, k_scales, v_scales);
        if (rc) {
#pragma omp atomic write
            err = rc;
        }
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Prefill / chunked-prefill attention                                        */
/* ------------------------------------------------------------------------ */

/* One prefill output row: query row `row` (of all chunks stacked: q[T][h_q][d]) belongs to
 * sequence s, whose chunk holds rows query_start[s] .. query_start[s+1]-1 and ends at the
 * sequence's last cached token, so row i of the chunk sits at absolute position
 * p = context_lens[s] - chunk_len + i.  The row attends causally: tokens 0..p of sequence s,
 * read through the block table, in fp64.
 * "vLLM 推理原理…" section 一次生成有两个阶段 (prefill processes the input tokens and builds
 * their KV; chunked prefill splits a long input into pieces scheduled with decoding);
 * "现代 AI…" section 1 (attention formula); "深度解构…" section 2.1 (block table). */
static int prefill_row(double *out_row, int s, int i, int h, const uint16_t *qrow,
                       const void *k_cache, const void *v_cache, const int32_t *block_tables,
                       int max_blocks_per_seq, int ctx, int chunk, int h_q, int h_kv, int d, int bs,
                       int num_blocks, double scale, int cache_dtype, const float *k_scales,
                       const float *v_scales)
{
    const int group = h_q / h_kv;
    const int kh = h / group;                 /* KV head of query head h */
    int p = ctx - chunk + i;                  /* absolute position of this query token */
    int n = p + 1;                            /* tokens it attends to */
    const double ks = cache_dtype ? (double)k_scales[kh] : 1.0;
    const double vs = cache_dtype ? (double)v_scales[kh] : 1.0;
    for (int e = 0; e < d; ++e) out_row[e] = 0.0;
    if (p < 0) return -7;
    if ((n + bs - 1) / bs > max_blocks_per_seq) return -2;
    double *score = (double *)malloc(sizeof(double) * (size_t)n);
    if (!score) return -3;
    double top = -INFINITY;
    for (int j = 0; j < n; ++j) {
        const int32_t blk = block_tables[(size_t)s * max_blocks_per_seq + j / bs];
        if (blk < 0 || blk >= num_blocks) { free(score); return -1; }
        double acc = 0.0;
        for (int e = 0; e < d; ++e)
            acc += or_bf16_decode(qrow[e]) *
                   cache_elem(k_cache, cache_index(blk, kh, j % bs, e, h_kv, bs, d), cache_dtype, ks);
        score[j] = acc * scale;
        if (score[j] > top) top = score[j];
    }
    double total = 0.0;
    for (int j = 0; j < n; ++j) {
        const double wj = exp(score[j] - top);
        const int32_t blk = block_tables[(size_t)s * max_blocks_per_seq + j / bs];
        total += wj;
        for (int e = 0; e < d; ++e)
            out_row[e] += wj * cache_elem(v_cache, cache_index(blk, kh, j % bs, e, h_kv, bs, d), cache_dtype, vs);
    }
    for (int e = 0; e < d; ++e) out_row[e] = out_row[e] / total;
    free(score);
    return 0;
}

/* Selected prefill rows: rows[2*r] = query row (0..T-1), rows[2*r+1] = query head;
 * out[r][d] (fp64).  q: [T][h_q][d] bf16 bits; query_start: [B+1]; context_lens: [B] (each
 * including its chunk).  Returns 0, -1 on a bad block id, -2 on a context longer than the
 * table row, -4 on a bad head split, -5 on a bad type, -6 on a row outside every chunk, -7 on
 * a chunk longer than its context. */
int or_paged_prefill_rows(double *out, const int32_t *rows, int nrows, const uint16_t *q,
                          const void *k_cache, const void *v_cache, const int32_t *block_tables,
                          int max_blocks_per_seq, const int32_t *query_start, const int32_t *context_lens,
                          int B, int h_q, int h_kv, int d, int bs, int num_blocks, double scale,
                          int cache_dtype, const float *k_scales, const float *v_scales)
{
    if (h_kv <= 0 || h_q % h_kv != 0) return -4;
    if (cache_dtype < 0 || cache_dtype > 2) return -5;
    for (int r = 0; r < nrows; ++r) {
        int row = rows[2 * r], h = rows[2 * r + 1];
        int s = -1;
        for (int b = 0; b < B; ++b)
            if (row >= query_start[b] && row < query_start[b + 1]) { s = b; break; }
        if (s < 0) return -6;
        int chunk = query_start[s + 1] - query_start[s];
        int rc = prefill_row(out + (size_t)r * d, s, row - query_start[s], h, q + ((size_t)row * h_q + h) * d,
                             k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens[s], chunk,
                             h_q, h_kv, d, bs, num_blocks, scale, cache_dtype, k_scales, v_scales);
        if (rc) return rc;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Array forms of the codecs (plain loops over the scalar definitions above). */
/* ------------------------------------------------------------------------ */

void or_bf16_decode_n(const uint16_t *in, double *out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = or_bf16_decode(in[i]); }

void or_bf16_encode_rne_n(const float *in, uint16_t *out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = or_bf16_encode_rne(in[i]); }

void or_e4m3_decode_n(const uint8_t *in, double *out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = or_e4m3_decode(in[i]); }

void or_e4m3_encode_satfinite_n(const float *in, uint8_t *out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = or_e4m3_encode_satfinite(in[i]); }

void or_int8_encode_sat_n(const float *in, int8_t *out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = or_int8_encode_sat(in[i]); }

void or_int8_decode_n(const int8_t *in, double *out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = or_int8_decode(in[i]); }

void or_div_f32_n(const float *x, float s, float *out, int64_t n)
{ for (int64_t i = 0; i < n; ++i) out[i] = or_div_f32(x[i], s); }
