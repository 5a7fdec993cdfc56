/*
 * Oracle for paged single-token decode attention.  TEST INFRASTRUCTURE ONLY:
 * nothing on the product path may link, load or call this file.  It is the
 * plain, slow, fp64 statement of what the paged decode path computes, written
 * from the method's definition and shared with no GPU code.
 *
 * Sources (page, section):
 *  - lqnn.cn/news/235768 ("为什么大模型推理这么慢"), section 1.2: attention is
 *    softmax(Q K^T / sqrt(d)) V; in decode the current token is Q against the K/V
 *    of every cached token.
 *  - same page, section 2.2 (single-step decode pseudo-code): the new token's
 *    k, v are written at position cache_len first, then attention runs over
 *    cache_len + 1 entries, so the decoded token attends to itself.
 *  - same page, section 3.2, and chanyi.net.cn/article/49 section 三: the cache is
 *    cut into fixed 16-token blocks; a per-request block table maps logical block
 *    i to a physical block; the kernel walks the table in order, so the result
 *    depends only on logical order.
 *  - chanyi.net.cn/article/49 section 三: copy-on-write sharing of prefix blocks.
 *  - chanyi.net.cn/article/49 section 四: tiling with online softmax leaves the
 *    mathematical result unchanged, so the plain two-pass softmax is the target.
 *  - lqnn.cn/news/235768 section 4.1: 8-bit KV with grouped scale factors.
 *  - lqnn.cn/news/235768 section 4.2: GQA, several query heads share one KV head.
 *
 * Readings where the pages are silent:
 *  - seq_lens count the token being decoded (append, then attend).
 *  - GQA grouping is contiguous: query head h reads KV head h / (H_q / H_kv).
 *  - cache layout [num_blocks][H_kv][block_size][head_dim]; only the logical
 *    order matters for the result.
 *  - int8: symmetric, range +-127, one fp32 scale per (block, KV head) for K and
 *    one for V; s = absmax / 127 and q = clamp(rint(x / s), -127, 127) in IEEE fp32
 *    with round-half-even; an all-zero tile gets s = 0 and q = 0.
 *  - seq_len <= 0 gives an all-zero output row.
 *
 * Every function returns 0 on success and a negative code on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_I8 = 3, OR_I4 = 4 };

/* Planted-mistake switch for the pin tests: a build with -DORACLE_MUTATION=n
 * (n > 0) carries one deliberate error, and the tests check that some pin
 * fails on it.  The normal build has ORACLE_MUTATION == 0 and every MUT(n) is
 * a constant false. */
#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif
#define MUT(n) (ORACLE_MUTATION == (n))

/* IEEE 754 binary16 -> double, from the format's definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits). */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/2^10) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t bits = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static size_t elem_bytes(int dt)
{
    switch (dt) {
    case OR_F32: return 4;
    case OR_F16: return 2;
    case OR_BF16: return 2;
    case OR_I8: return 1;
    default: return 0;
    }
}

/* Bytes of a row of d elements of dtype dt (4-bit values pack two per byte). */
static size_t row_bytes(int dt, int d)
{
    return dt == OR_I4 ? (size_t)d / 2 : (size_t)d * elem_bytes(dt);
}

/* Element idx of a buffer of dtype dt, as a double.  For int8 the raw integer;
 * for int4 the integer n - 8 of the 4-bit value n, element 2k being the low
 * half of byte k and element 2k+1 its high half. */
static double load_elem(const void *base, size_t idx, int dt)
{
    switch (dt) {
    case OR_F32: return (double)((const float *)base)[idx];
    case OR_F16: return oracle_half_to_double(((const uint16_t *)base)[idx]);
    case OR_BF16: return oracle_bf16_to_double(((const uint16_t *)base)[idx]);
    case OR_I8: return (double)((const int8_t *)base)[idx];
    case OR_I4: {
        const uint8_t byte = ((const uint8_t *)base)[idx / 2];
        const int hi = MUT(12) ? !(idx & 1) : (int)(idx & 1);
        return (double)((hi ? byte >> 4 : byte & 15) - 8);
    }
    default: return NAN;
    }
}

/*
 * Cache append: token i with slot s >= 0 goes to physical block s / block_size,
 * offset s % block_size, for every KV head.  A byte copy; slot < 0 is padding
 * and is skipped.  k, v are [num_tokens][num_kv_heads][head_dim] with the given
 * token stride in elements.
 */
int oracle_reshape_and_cache(const void *k, const void *v, void *key_cache, void *value_cache,
                             const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int64_t num_blocks, int dtype,
                             int64_t k_token_stride, int64_t v_token_stride)
{
    size_t E = elem_bytes(dtype);
    if (!E || block_size <= 0 || head_dim <= 0 || num_kv_heads <= 0) return -2;
    size_t row = (size_t)head_dim * E;
    for (int64_t i = 0; i < num_tokens; ++i) {
        int64_t s = slot_mapping[i];
        if (s < 0) continue;
        if (s >= num_blocks * block_size) return -3;
        int64_t blk = s / block_size, off = s % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t dst = (size_t)(((blk * num_kv_heads + h) * block_size + off)) * row;
            const char *ks = (const char *)k + ((size_t)i * k_token_stride + (size_t)h * head_dim) * E;
            const char *vs = (const char *)v + ((size_t)i * v_token_stride + (size_t)h * head_dim) * E;
            memcpy((char *)key_cache + dst, ks, row);
            memcpy((char *)value_cache + dst, MUT(7) ? ks : vs, row);
        }
    }
    return 0;
}

/*
 * Copy-on-write block copy: for each (src, dst) pair the whole physical block,
 * every KV head and every slot, of K and of V (and the int8 scales when given)
 * is copied byte for byte.  Pairs are applied in order.
 */
int oracle_block_copy(void *key_cache, void *value_cache, float *k_scales, float *v_scales,
                      const int64_t *pairs, int64_t num_pairs, int num_kv_heads, int head_dim,
                      int block_size, int64_t num_blocks, int dtype)
{
    if (!elem_bytes(dtype) && dtype != OR_I4) return -2;
    size_t blk_bytes = (size_t)num_kv_heads * block_size * row_bytes(dtype, head_dim);
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) return -3;
        memcpy((char *)key_cache + dst * blk_bytes, (char *)key_cache + src * blk_bytes, blk_bytes);
        if (!MUT(10))
            memcpy((char *)value_cache + dst * blk_bytes, (char *)value_cache + src * blk_bytes,
                   blk_bytes);
        if (k_scales)
            memcpy(k_scales + dst * num_kv_heads, k_scales + src * num_kv_heads,
                   sizeof(float) * num_kv_heads);
        if (v_scales)
            memcpy(v_scales + dst * num_kv_heads, v_scales + src * num_kv_heads,
                   sizeof(float) * num_kv_heads);
    }
    return 0;
}

/*
 * 8-bit KV with one scale per group, the group being one (block, KV head) tile
 * of block_size * head_dim values.  Symmetric absmax in IEEE fp32:
 *   a = max |x|,  s = a / 127,  q = clamp(rint(x / s), -127, 127)
 * rint() rounds half to even under the default rounding mode.  a = 0 gives
 * s = 0 and q = 0.  src holds fp32, fp16 or bf16 values; every value of those
 * types is exact in fp32.
 */
int oracle_quantize_int8(const void *src, int src_dtype, int8_t *dst, float *scales,
                         int64_t num_blocks, int num_kv_heads, int head_dim, int block_size)
{
    if (src_dtype != OR_F32 && src_dtype != OR_F16 && src_dtype != OR_BF16) return -4;
    size_t tile = (size_t)block_size * head_dim;
    for (int64_t t = 0; t < num_blocks * num_kv_heads; ++t) {
        float a = 0.0f;
        for (size_t i = 0; i < tile; ++i) {
            float x = (float)load_elem(src, t * tile + i, src_dtype);
            float ax = fabsf(x);
            if (ax > a) a = ax;
        }
        float s = MUT(6) ? a / 128.0f : a / 127.0f;
        scales[t] = s;
        for (size_t i = 0; i < tile; ++i) {
            if (a == 0.0f) {
                dst[t * tile + i] = 0;
                continue;
            }
            float x = (float)load_elem(src, t * tile + i, src_dtype);
            float r = rintf(x / s);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            dst[t * tile + i] = (int8_t)r;
        }
    }
    return 0;
}

/*
 * Appending single tokens into an int8 cache (the rescaling the 8-bit grouped-scale
 * KV of lqnn.cn/news/235768 section 4.1 needs once blocks are quantised: the pages
 * do not spell it out; this is the library's reading).  For each token i with
 * slot s = slot_mapping[i] >= 0 (s >= num_blocks * block_size is skipped), block
 * b = s / block_size, slot o = s % block_size, and every KV head h, separately for
 * K (k, key_cache, k_scales) and V:
 *   a = max_j |x_j| over the token's head_dim values,  c = a / 127,
 *   s_old = scales[b][h];  s_new = c > s_old ? c : s_old;
 *   if s_new > s_old: every code of the tile in the other slots is re-rounded,
 *       q <- clamp(rint((q * s_old) / s_new), -127, 127);
 *   the token's codes are clamp(rint(x_j / s_new), -127, 127) (0 when s_new = 0);
 *   scales[b][h] = s_new.
 * All arithmetic in IEEE fp32 (products and quotients rounded to nearest, rint
 * half to even).  So the scale never shrinks, every stored value moves by at
 * most s_new / 2 when re-rounded, and an append that does not raise the scale
 * leaves the other codes untouched.  Tokens are applied in order; the library
 * requires the tokens of one call to fall in distinct blocks.
 */
int oracle_append_int8(const void *k, const void *v, int src_dtype, int8_t *key_cache, int8_t *value_cache,
                       float *k_scales, float *v_scales, const int64_t *slot_mapping, int64_t num_tokens,
                       int num_kv_heads, int head_dim, int block_size, int64_t num_blocks)
{
    if (src_dtype != OR_F32 && src_dtype != OR_F16 && src_dtype != OR_BF16) return -4;
    const size_t tile = (size_t)block_size * head_dim;
    for (int64_t i = 0; i < num_tokens; ++i) {
        const int64_t s = slot_mapping[i];
        if (s < 0 || s >= num_blocks * block_size) continue;
        const int64_t b = s / block_size;
        const int o = (int)(s % block_size);
        for (int kv = 0; kv < 2; ++kv) {
            const void *src = kv ? v : k;
            int8_t *cache = kv ? value_cache : key_cache;
            float *scales = kv ? v_scales : k_scales;
            for (int h = 0; h < num_kv_heads; ++h) {
                const size_t x0 = ((size_t)i * num_kv_heads + h) * head_dim;
                float a = 0.0f;
                for (int j = 0; j < head_dim; ++j) {
                    float ax = fabsf((float)load_elem(src, x0 + j, src_dtype));
                    if (ax > a) a = ax;
                }
                const float c = a / 127.0f;
                const float s_old = scales[b * num_kv_heads + h];
                const float s_new = c > s_old ? c : s_old;
                int8_t *t = cache + ((size_t)b * num_kv_heads + h) * tile;
                if (s_new > s_old) {
                    for (int r = 0; r < block_size; ++r) {
                        if (r == o) continue;
                        for (int j = 0; j < head_dim; ++j) {
                            const float prod = (float)t[(size_t)r * head_dim + j] * s_old;
                            float q = rintf(MUT(14) ? (prod / s_old) : (prod / s_new));
                            if (q > 127.0f) q = 127.0f;
                            if (q < -127.0f) q = -127.0f;
                            t[(size_t)r * head_dim + j] = (int8_t)q;
                        }
                    }
                }
                for (int j = 0; j < head_dim; ++j) {
                    float q = 0.0f;
                    if (s_new != 0.0f) {
                        q = rintf((float)load_elem(src, x0 + j, src_dtype) / s_new);
                        if (q > 127.0f) q = 127.0f;
                        if (q < -127.0f) q = -127.0f;
                    }
                    t[(size_t)o * head_dim + j] = (int8_t)q;
                }
                scales[b * num_kv_heads + h] = s_new;
            }
        }
    }
    return 0;
}

/*
 * 4-bit KV with one scale per group (the pages' second grouped-scale width), the
 * group again one (block, KV head) tile.  Symmetric absmax in IEEE fp32:
 *   a = max |x|,  s = a / 7,  q = clamp(rint(x / s), -7, 7)
 * stored as n = q + 8 in [1, 15]: element 2k in the low four bits of byte k of
 * the tile, element 2k+1 in the high four.  a = 0 gives s = 0 and q = 0.  dst
 * holds num_blocks * num_kv_heads * block_size * head_dim / 2 bytes.
 */
int oracle_quantize_int4(const void *src, int src_dtype, uint8_t *dst, float *scales,
                         int64_t num_blocks, int num_kv_heads, int head_dim, int block_size)
{
    if (src_dtype != OR_F32 && src_dtype != OR_F16 && src_dtype != OR_BF16) return -4;
    if (head_dim % 2) return -2;
    size_t tile = (size_t)block_size * head_dim;
    for (int64_t t = 0; t < num_blocks * num_kv_heads; ++t) {
        float a = 0.0f;
        for (size_t i = 0; i < tile; ++i) {
            float ax = fabsf((float)load_elem(src, t * tile + i, src_dtype));
            if (ax > a) a = ax;
        }
        float s = MUT(13) ? a / 8.0f : a / 7.0f;
        scales[t] = s;
        uint8_t *out = dst + t * (tile / 2);
        for (size_t i = 0; i < tile; ++i) {
            float r = 0.0f;
            if (a != 0.0f) {
                r = rintf((float)load_elem(src, t * tile + i, src_dtype) / s);
                if (r > 7.0f) r = 7.0f;
                if (r < -7.0f) r = -7.0f;
            }
            uint8_t n = (uint8_t)((int)r + 8);
            if (i % 2 == 0)
                out[i / 2] = n;
            else
                out[i / 2] = (uint8_t)(out[i / 2] | (n << 4));
        }
    }
    return 0;
}

/* Common argument block for the decode functions. */
typedef struct {
    const double *q;          /* [B][H_q][d], already upcast to fp64 */
    const void *key_cache;    /* [N_blk][H_kv][bs][d] of kv_dtype */
    const void *value_cache;
    int kv_dtype;
    const float *k_scales;    /* [N_blk][H_kv], int8 only */
    const float *v_scales;
    const int32_t *block_tables; /* [B][max_blocks_per_seq] */
    const int32_t *seq_lens;     /* [B] */
    int num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
    int64_t num_blocks;
    double scale;
} dec_args;

/*
 * Gather step: the logical token t of sequence b, KV head g, read through the
 * block table.  This is exactly the contiguous copy the GPU must not make; here
 * it keeps the definition visible.  K and V are written to rows of Kc, Vc.
 */
static int gather(const dec_args *a, int b, int g, int t0, int t1, double *Kc, double *Vc)
{
    int d = a->head_dim, bs = a->block_size;
    for (int t = t0; t < t1; ++t) {
        int lb = t / bs;
        if (lb >= a->max_blocks_per_seq) return -3;
        int64_t blk = a->block_tables[(size_t)b * a->max_blocks_per_seq + lb];
        if (blk < 0 || blk >= a->num_blocks) return -3;
        int off = MUT(2) ? (t + 1) % bs : t % bs;
        size_t base = (size_t)(((blk * a->num_kv_heads + g) * bs + off)) * d;
        double ks = 1.0, vs = 1.0;
        if (a->kv_dtype == OR_I8 || a->kv_dtype == OR_I4) {
            ks = (double)a->k_scales[blk * a->num_kv_heads + g];
            vs = (double)a->v_scales[blk * a->num_kv_heads + g];
        }
        for (int j = 0; j < d; ++j) {
            Kc[(size_t)(t - t0) * d + j] = load_elem(a->key_cache, base + j, a->kv_dtype) * ks;
            Vc[(size_t)(t - t0) * d + j] = load_elem(a->value_cache, base + j, a->kv_dtype) * vs;
        }
    }
    return 0;
}

/*
 * softmax(scale * q . K^T) . V over tokens [t0, t1) of one (sequence, query head),
 * two-pass in fp64: m = max s, p = exp(s - m), l = sum p, o = sum p V / l.
 * Returns lse = m + log(l) through *lse.
 */
static int attend_q(const dec_args *a, const double *qv, int b, int h, int t0, int t1, double *o,
                    double *lse)
{
    int d = a->head_dim;
    int G = a->num_q_heads / a->num_kv_heads;
    int g = MUT(1) ? h % a->num_kv_heads : h / G;
    int n = t1 - t0;
    double *Kc = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *Vc = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    int rc = (Kc && Vc && s) ? gather(a, b, g, t0, t1, Kc, Vc) : -9;
    if (rc == 0) {
        double m = -INFINITY;
        for (int t = 0; t < n; ++t) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += qv[j] * Kc[(size_t)t * d + j];
            s[t] = MUT(3) ? acc : a->scale * acc;
            if (s[t] > m) m = s[t];
        }
        double l = 0.0;
        for (int t = 0; t < n; ++t) {
            s[t] = exp(s[t] - m);
            l += s[t];
        }
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            const double *W = MUT(8) ? Kc : Vc;
            for (int t = 0; t < n; ++t) acc += s[t] * W[(size_t)t * d + j];
            o[j] = acc / l;
        }
        *lse = MUT(9) ? m : m + log(l);
    }
    free(Kc);
    free(Vc);
    free(s);
    return rc;
}

/* Attention of query row (b, h) of a [B][H_q][d] q over the tokens [t0, t1). */
static int attend_range(const dec_args *a, int b, int h, int t0, int t1, double *o, double *lse)
{
    return attend_q(a, a->q + ((size_t)b * a->num_q_heads + h) * a->head_dim, b, h, t0, t1, o, lse);
}

static int check_dims(const dec_args *a)
{
    if (a->num_seqs < 0 || a->num_q_heads <= 0 || a->num_kv_heads <= 0 || a->head_dim <= 0 ||
        a->block_size <= 0)
        return -2;
    if (a->num_q_heads % a->num_kv_heads) return -2;
    if ((a->kv_dtype == OR_I8 || a->kv_dtype == OR_I4) && (!a->k_scales || !a->v_scales)) return -1;
    if (!elem_bytes(a->kv_dtype) && a->kv_dtype != OR_I4) return -4;
    if (a->kv_dtype == OR_I4 && a->head_dim % 2) return -2;
    return 0;
}

/*
 * Decode: out[b][h][:] = softmax_t(scale * q[b][h] . K[b][t]) . V[b][t] for
 * t = 0 .. seq_lens[b]-1.  If bh_list is non-NULL only the listed
 * (sequence, query head) pairs (bh_list[2i], bh_list[2i+1]) are computed;
 * other rows of out are left as they are.  nthreads > 1 spreads the rows over
 * OpenMP threads.
 */
int oracle_decode(double *out, const double *q, const void *key_cache, const void *value_cache,
                  int kv_dtype, const float *k_scales, const float *v_scales,
                  const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                  int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                  int max_blocks_per_seq, int64_t num_blocks, double scale,
                  const int32_t *bh_list, int64_t num_bh, int nthreads)
{
    dec_args a = {q, key_cache, value_cache, kv_dtype, k_scales, v_scales, block_tables,
                  seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                  max_blocks_per_seq, num_blocks, scale};
    int rc = check_dims(&a);
    if (rc) return rc;
    int64_t rows = bh_list ? num_bh : (int64_t)num_seqs * num_q_heads;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        int b = bh_list ? bh_list[2 * r] : (int)(r / num_q_heads);
        int h = bh_list ? bh_list[2 * r + 1] : (int)(r % num_q_heads);
        double *o = out + ((size_t)b * num_q_heads + h) * head_dim;
        int L = MUT(4) ? seq_lens[b] - 1 : seq_lens[b];
        if (L <= 0) {
            for (int j = 0; j < head_dim; ++j) o[j] = 0.0;
            continue;
        }
        double lse;
        int e = attend_range(&a, b, h, 0, L, o, &lse);
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    return err;
}

/*
 * Decode of query_len > 1 new tokens per sequence (the verification step of
 * speculative decoding, or a chunk of prefill, over the same paged cache):
 * q and out are [B][Q][H_q][d].  seq_lens[b] = L counts every new token, so
 * query token i sits at position L - Q + i and attends causally to the tokens
 * 0 .. L - Q + i:
 *   out[b][i][h][:] = sum_{t <= L-Q+i} softmax_t(scale * q[b][i][h] . K[b][t]) V[b][t].
 * Rows whose range is empty (L - Q + i < 0) are zero.  Q = 1 is oracle_decode.
 */
int oracle_decode_multi(double *out, const double *q, const void *key_cache, const void *value_cache,
                        int kv_dtype, const float *k_scales, const float *v_scales,
                        const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                        int query_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                        int max_blocks_per_seq, int64_t num_blocks, double scale, int nthreads)
{
    dec_args a = {q, key_cache, value_cache, kv_dtype, k_scales, v_scales, block_tables,
                  seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                  max_blocks_per_seq, num_blocks, scale};
    int rc = check_dims(&a);
    if (rc) return rc;
    if (query_len <= 0) return -2;
    int64_t rows = (int64_t)num_seqs * query_len * num_q_heads;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        int h = (int)(r % num_q_heads);
        int i = (int)((r / num_q_heads) % query_len);
        int b = (int)(r / ((int64_t)num_q_heads * query_len));
        double *o = out + (size_t)r * head_dim;
        int end = seq_lens[b] - query_len + i + (MUT(11) ? 0 : 1);  /* tokens 0 .. end-1 */
        if (end <= 0) {
            for (int j = 0; j < head_dim; ++j) o[j] = 0.0;
            continue;
        }
        double lse;
        int e = attend_q(&a, q + (size_t)r * head_dim, b, h, 0, end, o, &lse);
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    return err;
}

/*
 * Split form of the same decode.  Partition p of sequence b covers tokens
 * [p*P, min(L, (p+1)*P)).  For each (b, h, p) with a non-empty partition:
 *   o_part[b][h][p][:] = normalised partial output, lse_part[b][h][p] = m_p + log l_p.
 * Empty partitions get lse = -inf and o = 0.  Shapes [B][H_q][max_parts][d] and
 * [B][H_q][max_parts].
 */
int oracle_decode_partials(double *o_part, double *lse_part, const double *q, const void *key_cache,
                           const void *value_cache, int kv_dtype, const float *k_scales,
                           const float *v_scales, const int32_t *block_tables,
                           const int32_t *seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                           int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                           double scale, int partition_size, int max_parts, int nthreads)
{
    dec_args a = {q, key_cache, value_cache, kv_dtype, k_scales, v_scales, block_tables,
                  seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                  max_blocks_per_seq, num_blocks, scale};
    int rc = check_dims(&a);
    if (rc) return rc;
    if (partition_size <= 0 || max_parts <= 0) return -2;
    int err = 0;
    int64_t rows = (int64_t)num_seqs * num_q_heads * max_parts;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r) {
        int p = (int)(r % max_parts);
        int h = (int)((r / max_parts) % num_q_heads);
        int b = (int)(r / ((int64_t)max_parts * num_q_heads));
        double *o = o_part + (size_t)r * head_dim;
        int L = seq_lens[b];
        int t0 = p * partition_size;
        int t1 = t0 + partition_size < L ? t0 + partition_size : L;
        if (t0 >= t1) {
            for (int j = 0; j < head_dim; ++j) o[j] = 0.0;
            lse_part[r] = -INFINITY;
            continue;
        }
        int e = attend_range(&a, b, h, t0, t1, o, &lse_part[r]);
        if (e) {
#pragma omp atomic write
            err = e;
        }
    }
    return err;
}

/*
 * Log-sum-exp merge of partition results for every (b, h):
 *   M = max_p lse_p,  w_p = exp(lse_p - M),  out = sum_p w_p o_p / sum_p w_p.
 * Partitions with lse = -inf carry weight 0.  A row with no partition gives 0.
 */
int oracle_merge(double *out, const double *o_part, const double *lse_part, int64_t rows,
                 int max_parts, int head_dim)
{
    for (int64_t r = 0; r < rows; ++r) {
        const double *lse = lse_part + r * max_parts;
        double M = -INFINITY;
        for (int p = 0; p < max_parts; ++p)
            if (lse[p] > M) M = lse[p];
        double *o = out + r * head_dim;
        for (int j = 0; j < head_dim; ++j) o[j] = 0.0;
        if (M == -INFINITY) continue;
        double wsum = 0.0;
        for (int p = 0; p < max_parts; ++p) {
            if (lse[p] == -INFINITY) continue;
            double w = exp(lse[p] - M);
            wsum += w;
            const double *op = o_part + (r * max_parts + p) * head_dim;
            for (int j = 0; j < head_dim; ++j) o[j] += w * op[j];
        }
        if (!MUT(5))
            for (int j = 0; j < head_dim; ++j) o[j] /= wsum;
    }
    return 0;
}

/* KV bytes per token: 2 (K and V) x layers x KV heads x head_dim x bytes (lqnn.cn section 2.3). */
int64_t oracle_kv_bytes_per_token(int num_layers, int num_kv_heads, int head_dim, int elem_size)
{
    return (int64_t)2 * num_layers * num_kv_heads * head_dim * elem_size;
}
