/*
 * oracle.c -- plain, slow fp64 CPU statement of one decode step of LLaMA-style
 * attention against a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * Sources (three web pages on writing an LLM inference engine):
 *   [ENGINE]  "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427), chapter 1:
 *             s3.4  KV-cache size formula, fixed 16/32-token pages from a free list,
 *                   attention finds the cached block through the page index;
 *             s4.2  RoPE puts the position into q and k through a rotation;
 *             s4.3  forward with a KV cache: q/k/v views with n_heads / n_kv_heads,
 *                   apply_rotary_emb(q, k, start_pos), append to the cache,
 *                   scores q.k^T / sqrt(head_dim) + causal mask, softmax, times v;
 *             s5.2  check a cache by disabling it and recomputing the whole sequence.
 *   [FLOW]    "大模型推理全流程解析" (stapisi.com/news/4049481), s2.2.2: one query
 *             against all cached keys, scaled, softmax, weighted sum of values.
 *   [WEIGHTS] dpshk.com/news/4990443, s3.2: fp16 q.k products can overflow before the
 *             softmax (so accumulate wide); s5.1: GQA gives k_proj n_kv_heads*head_dim.
 *
 * Storage values are IEEE binary16 or bfloat16 bit patterns (uint16); every
 * function decodes them to double, computes in double, and (where the method
 * stores a result) rounds once, to nearest-even, straight from double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_F16 0
#define ORA_BF16 1

/* ------------------------------------------------------------------------- */
/* storage formats                                                            */
/* ------------------------------------------------------------------------- */

/* IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double ora_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);               /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);   /* 1.f * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: the top 16 bits of an IEEE binary32 (8 exponent bits, bias 127). */
double ora_bf16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);              /* subnormal: f * 2^-133 */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);   /* 1.f * 2^(e-127) */
    return sign ? -v : v;
}

/*
 * Round a double to a binary format with `mbits` fraction bits and exponent
 * bias `bias`, to nearest with ties to even, in one step.  Scaling by a power
 * of two is exact, and rint() rounds to nearest-even in the default mode.
 */
static uint16_t round_to_format(double x, int mbits, int bias, int ebits)
{
    uint16_t sign = signbit(x) ? (uint16_t)(1u << 15) : 0;
    int emax_field = (1 << ebits) - 1;
    if (isnan(x))
        return (uint16_t)(sign | (emax_field << mbits) | (1u << (mbits - 1)));
    double a = fabs(x);
    if (isinf(a))
        return (uint16_t)(sign | (emax_field << mbits));
    if (a == 0.0)
        return sign;
    int e2;
    frexp(a, &e2);                   /* a = m * 2^e2, m in [0.5, 1) */
    int E = e2 - 1;                  /* a = 1.x * 2^E */
    int emin = 1 - bias;
    double units;
    long long bits;
    if (E < emin) {
        /* subnormal range: count units of 2^(emin - mbits) */
        units = rint(ldexp(a, mbits - emin));
        bits = (long long)units;     /* a carry into 2^mbits lands on the min normal */
    } else {
        units = rint(ldexp(a, mbits - E));          /* in [2^mbits, 2^(mbits+1)] */
        bits = ((long long)(E + bias) << mbits) + (long long)units - (1ll << mbits);
    }
    if (bits >= ((long long)emax_field << mbits))
        bits = (long long)emax_field << mbits;     /* overflow to infinity */
    return (uint16_t)(sign | (uint16_t)bits);
}

uint16_t ora_double_to_half(double x) { return round_to_format(x, 10, 15, 5); }
uint16_t ora_double_to_bf16(double x) { return round_to_format(x, 7, 127, 8); }

static double dec(uint16_t h, int dtype)
{
    return dtype == ORA_BF16 ? ora_bf16_to_double(h) : ora_half_to_double(h);
}

static uint16_t enc(double x, int dtype)
{
    return dtype == ORA_BF16 ? ora_double_to_bf16(x) : ora_double_to_half(x);
}

void ora_decode_array(const uint16_t* src, double* dst, int64_t n, int dtype)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = dec(src[i], dtype);
}

void ora_encode_array(const double* src, uint16_t* dst, int64_t n, int dtype)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = enc(src[i], dtype);
}

/* ------------------------------------------------------------------------- */
/* RoPE  [ENGINE] s4.2, s4.3                                                   */
/* ------------------------------------------------------------------------- */

/*
 * Rotary position embedding of one token's heads, in double.
 * x, y: [n_tokens][heads][head_dim].  Pair i of a head is (x[2i], x[2i+1]);
 * it is turned by the angle pos * theta^(-2i/head_dim):
 *   y[2i]   = x[2i] cos a - x[2i+1] sin a
 *   y[2i+1] = x[2i] sin a + x[2i+1] cos a
 * (the pages name a rotation applied at start_pos; the pairing and the
 * frequency ladder are the ones the name apply_rotary_emb refers to).
 */
void ora_rope_f64(const double* x, double* y, const int32_t* positions,
                  int n_tokens, int heads, int head_dim, double theta)
{
    for (int t = 0; t < n_tokens; ++t) {
        for (int h = 0; h < heads; ++h) {
            const double* xs = x + ((int64_t)t * heads + h) * head_dim;
            double* ys = y + ((int64_t)t * heads + h) * head_dim;
            for (int i = 0; i < head_dim / 2; ++i) {
                double freq = pow(theta, -2.0 * i / head_dim);
                double angle = (double)positions[t] * freq;
                double c = cos(angle), s = sin(angle);
                double x0 = xs[2 * i], x1 = xs[2 * i + 1];
                ys[2 * i] = x0 * c - x1 * s;
                ys[2 * i + 1] = x0 * s + x1 * c;
            }
        }
    }
}

/* RoPE on storage values: decode, rotate in double, round once to the dtype.
 * exact_out (optional) receives the unrounded doubles. */
void ora_rope(const uint16_t* x, uint16_t* y, double* exact_out, const int32_t* positions,
              int n_tokens, int heads, int head_dim, double theta, int dtype)
{
    int64_t n = (int64_t)n_tokens * heads * head_dim;
    double* xd = (double*)malloc(sizeof(double) * (size_t)(n ? n : 1));
    double* yd = (double*)malloc(sizeof(double) * (size_t)(n ? n : 1));
    ora_decode_array(x, xd, n, dtype);
    ora_rope_f64(xd, yd, positions, n_tokens, heads, head_dim, theta);
    ora_encode_array(yd, y, n, dtype);
    if (exact_out) memcpy(exact_out, yd, sizeof(double) * (size_t)n);
    free(xd);
    free(yd);
}

/* ------------------------------------------------------------------------- */
/* page table  [ENGINE] s3.4                                                   */
/* ------------------------------------------------------------------------- */

/*
 * Flat slot of the token at `position` of sequence b: the page that the page
 * table names for logical page position/P, and the row position%P inside it.
 * A negative position (a padded batch row) gives slot -1.
 */
void ora_slot_mapping(const int32_t* block_tables, int max_pages_per_seq,
                      const int32_t* positions, int n, int page_size, int64_t* slots)
{
    for (int b = 0; b < n; ++b) {
        int pos = positions[b];
        if (pos < 0) {
            slots[b] = -1;
            continue;
        }
        int logical_page = pos / page_size;
        int row = pos % page_size;
        int64_t physical = block_tables[(int64_t)b * max_pages_per_seq + logical_page];
        slots[b] = physical * page_size + row;
    }
}

/*
 * Cache update of one decode step for one layer ([ENGINE] s4.3 appends the new
 * k and v behind the cached ones; s5.3 asks for a preallocated pool in place of
 * concatenation).  pool: [num_pages][kv_heads][page_size][head_dim];
 * k, v: [n][kv_heads][head_dim]; the token of row b goes to position positions[b]
 * of sequence b.  Values are copied bit for bit.
 */
void ora_kv_append(uint16_t* k_pool, uint16_t* v_pool, const uint16_t* k, const uint16_t* v,
                   const int32_t* block_tables, int max_pages_per_seq, const int32_t* positions,
                   int n, int kv_heads, int page_size, int head_dim)
{
    for (int b = 0; b < n; ++b) {
        int pos = positions[b];
        if (pos < 0) continue;
        int64_t page = block_tables[(int64_t)b * max_pages_per_seq + pos / page_size];
        int row = pos % page_size;
        for (int h = 0; h < kv_heads; ++h) {
            for (int i = 0; i < head_dim; ++i) {
                int64_t dst = ((page * kv_heads + h) * page_size + row) * head_dim + i;
                int64_t src = ((int64_t)b * kv_heads + h) * head_dim + i;
                k_pool[dst] = k[src];
                v_pool[dst] = v[src];
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* attention                                                                   */
/* ------------------------------------------------------------------------- */

/*
 * Copy the first `len` cached tokens of sequence b out of the pages into a
 * contiguous [len][kv_heads][head_dim] array of doubles, in logical order: token
 * t lives in page block_tables[b][t / P], row t % P ([ENGINE] s3.4).
 */
static void gather_sequence(const uint16_t* pool, const int32_t* block_tables, int max_pages_per_seq,
                            int b, int len, int kv_heads, int page_size, int head_dim, int dtype,
                            double* dst)
{
    for (int t = 0; t < len; ++t) {
        int64_t page = block_tables[(int64_t)b * max_pages_per_seq + t / page_size];
        int row = t % page_size;
        for (int h = 0; h < kv_heads; ++h) {
            const uint16_t* src = pool + ((page * kv_heads + h) * page_size + row) * head_dim;
            for (int i = 0; i < head_dim; ++i)
                dst[((int64_t)t * kv_heads + h) * head_dim + i] = dec(src[i], dtype);
        }
    }
}

/*
 * Decode attention of one query token per sequence over its paged cache.
 *   q:   [batch][q_heads][head_dim] (storage), already rotated;
 *   pools: [num_pages][kv_heads][page_size][head_dim] (storage);
 *   context_lens[b]: tokens in the cache, the new one included (0 = padded row);
 *   out: [batch][q_heads][head_dim] double, before any rounding;
 *   weights (optional): [batch][q_heads][max_len] softmax weights, 0 past len.
 * For q head h the key/value head is h / (q_heads / kv_heads) (groups of
 * consecutive query heads share one kv head, [ENGINE] s4.3 n_kv_heads).
 * The single query sits at the last position, so the causal mask keeps every
 * cached token.  Softmax is taken with the maximum subtracted.
 */
void ora_decode_attention(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                          const int32_t* block_tables, int max_pages_per_seq,
                          const int32_t* context_lens, int batch, int q_heads, int kv_heads,
                          int head_dim, int page_size, double scale, int dtype,
                          double* out, double* weights, int max_len)
{
    int group = q_heads / kv_heads;
    for (int b = 0; b < batch; ++b) {
        int len = context_lens[b];
        if (len <= 0) {
            for (int h = 0; h < q_heads; ++h)
                for (int i = 0; i < head_dim; ++i)
                    out[((int64_t)b * q_heads + h) * head_dim + i] = 0.0;
            if (weights)
                for (int h = 0; h < q_heads; ++h)
                    for (int t = 0; t < max_len; ++t)
                        weights[((int64_t)b * q_heads + h) * max_len + t] = 0.0;
            continue;
        }
        size_t n = (size_t)len * kv_heads * head_dim;
        double* K = (double*)malloc(sizeof(double) * n);
        double* V = (double*)malloc(sizeof(double) * n);
        double* s = (double*)malloc(sizeof(double) * (size_t)len);
        gather_sequence(k_pool, block_tables, max_pages_per_seq, b, len, kv_heads, page_size,
                        head_dim, dtype, K);
        gather_sequence(v_pool, block_tables, max_pages_per_seq, b, len, kv_heads, page_size,
                        head_dim, dtype, V);
        for (int h = 0; h < q_heads; ++h) {
            int g = h / group;
            const uint16_t* qh = q + ((int64_t)b * q_heads + h) * head_dim;
            double mx = -INFINITY;
            for (int t = 0; t < len; ++t) {
                double dot = 0.0;
                for (int i = 0; i < head_dim; ++i)
                    dot += dec(qh[i], dtype) * K[((int64_t)t * kv_heads + g) * head_dim + i];
                s[t] = scale * dot;
                if (s[t] > mx) mx = s[t];
            }
            double z = 0.0;
            for (int t = 0; t < len; ++t) {
                s[t] = exp(s[t] - mx);
                z += s[t];
            }
            double* o = out + ((int64_t)b * q_heads + h) * head_dim;
            for (int i = 0; i < head_dim; ++i) {
                double acc = 0.0;
                for (int t = 0; t < len; ++t)
                    acc += s[t] * V[((int64_t)t * kv_heads + g) * head_dim + i];
                o[i] = acc / z;
            }
            if (weights) {
                double* w = weights + ((int64_t)b * q_heads + h) * max_len;
                for (int t = 0; t < max_len; ++t) w[t] = t < len ? s[t] / z : 0.0;
            }
        }
        free(K);
        free(V);
        free(s);
    }
}

/*
 * Decode attention restricted to a list of (b, q head) pairs -- the same
 * arithmetic as ora_decode_attention, for spot checks at sizes where the full
 * batch would take too long.  out: [n_pairs][head_dim].
 */
void ora_decode_attention_pairs(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                                const int32_t* block_tables, int max_pages_per_seq,
                                const int32_t* context_lens, int q_heads, int kv_heads,
                                int head_dim, int page_size, double scale, int dtype,
                                const int32_t* pair_b, const int32_t* pair_h, int n_pairs,
                                double* out)
{
    int group = q_heads / kv_heads;
    /* Each pair is an independent output: the OpenMP build (liboracle_omp.so) hands pairs
     * to threads; the plain build ignores the pragma.  The arithmetic of a pair is the
     * same in both. */
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < n_pairs; ++p) {
        int b = pair_b[p], h = pair_h[p], g = h / group;
        int len = context_lens[b];
        double* o = out + (int64_t)p * head_dim;
        if (len <= 0) {
            for (int i = 0; i < head_dim; ++i) o[i] = 0.0;
            continue;
        }
        const uint16_t* qh = q + ((int64_t)b * q_heads + h) * head_dim;
        double* s = (double*)malloc(sizeof(double) * (size_t)len);
        double mx = -INFINITY;
        for (int t = 0; t < len; ++t) {
            int64_t page = block_tables[(int64_t)b * max_pages_per_seq + t / page_size];
            const uint16_t* kr = k_pool + ((page * kv_heads + g) * page_size + t % page_size) * head_dim;
            double dot = 0.0;
            for (int i = 0; i < head_dim; ++i) dot += dec(qh[i], dtype) * dec(kr[i], dtype);
            s[t] = scale * dot;
            if (s[t] > mx) mx = s[t];
        }
        double z = 0.0;
        for (int t = 0; t < len; ++t) {
            s[t] = exp(s[t] - mx);
            z += s[t];
        }
        for (int i = 0; i < head_dim; ++i) o[i] = 0.0;
        for (int t = 0; t < len; ++t) {
            int64_t page = block_tables[(int64_t)b * max_pages_per_seq + t / page_size];
            const uint16_t* vr = v_pool + ((page * kv_heads + g) * page_size + t % page_size) * head_dim;
            for (int i = 0; i < head_dim; ++i) o[i] += s[t] * dec(vr[i], dtype);
        }
        for (int i = 0; i < head_dim; ++i) o[i] /= z;
        free(s);
    }
}

/*
 * Full causal attention over a whole contiguous sequence, every position a
 * query -- the "no cache, recompute everything" form of [ENGINE] s4.3 / s5.2:
 * S = Q K^T * scale + M with M[i][j] = -inf for j > i, row softmax, times V.
 *   q: [T][q_heads][head_dim], k, v: [T][kv_heads][head_dim] (doubles);
 *   out: [T][q_heads][head_dim].
 * Written with the explicit T x T score matrix and mask, independently of the
 * paged decode routine, so that the last row checks it.
 */
void ora_causal_attention_full(const double* q, const double* k, const double* v, int T,
                               int q_heads, int kv_heads, int head_dim, double scale, double* out)
{
    int group = q_heads / kv_heads;
    double* S = (double*)malloc(sizeof(double) * (size_t)T * (size_t)T);
    for (int h = 0; h < q_heads; ++h) {
        int g = h / group;
        for (int i = 0; i < T; ++i) {
            for (int j = 0; j < T; ++j) {
                double dot = 0.0;
                for (int e = 0; e < head_dim; ++e)
                    dot += q[((int64_t)i * q_heads + h) * head_dim + e] *
                           k[((int64_t)j * kv_heads + g) * head_dim + e];
                double mask = j > i ? -INFINITY : 0.0;
                S[(int64_t)i * T + j] = dot * scale + mask;
            }
        }
        for (int i = 0; i < T; ++i) {
            double* row = S + (int64_t)i * T;
            double mx = -INFINITY;
            for (int j = 0; j < T; ++j)
                if (row[j] > mx) mx = row[j];
            double z = 0.0;
            for (int j = 0; j < T; ++j) {
                row[j] = exp(row[j] - mx);
                z += row[j];
            }
            for (int j = 0; j < T; ++j) row[j] /= z;
            for (int e = 0; e < head_dim; ++e) {
                double acc = 0.0;
                for (int j = 0; j < T; ++j) acc += row[j] * v[((int64_t)j * kv_heads + g) * head_dim + e];
                out[((int64_t)i * q_heads + h) * head_dim + e] = acc;
            }
        }
    }
    free(S);
}

/* ------------------------------------------------------------------------- */
/* KV-cache size  [ENGINE] s3.4                                                */
/* ------------------------------------------------------------------------- */

/* layers x 2 (K and V) x heads x head_dim x tokens x bytes per element */
int64_t ora_kv_cache_bytes(int layers, int heads, int head_dim, int64_t tokens, int elt_bytes)
{
    return (int64_t)layers * 2 * heads * head_dim * tokens * elt_bytes;
}

/* ------------------------------------------------------------------------- */
/* RMSNorm  [ENGINE] s4.2                                                      */
/* ------------------------------------------------------------------------- */

/*
 * RMSNorm of each row, in double: y = x / sqrt(mean(x^2) + eps) * w.  The page is
 * explicit that eps is added to the mean square before the square root (not to the
 * root).  With a residual (optional), the row first becomes h = x + residual, rounded
 * once to the storage type (that rounded sum is also returned), and h is normalised.
 *   x, residual, out: [rows][hidden] storage; w: [hidden]; exact_out (optional): the
 *   unrounded doubles of y; residual_out (when residual is given): the rounded sums.
 */
void ora_rms_norm(const uint16_t* x, const uint16_t* residual, const uint16_t* w, int rows, int hidden,
                  double eps, int dtype, uint16_t* out, double* exact_out, uint16_t* residual_out)
{
    for (int r = 0; r < rows; ++r) {
        const int64_t base = (int64_t)r * hidden;
        double* h = (double*)malloc(sizeof(double) * (size_t)hidden);
        for (int i = 0; i < hidden; ++i) {
            double v = dec(x[base + i], dtype);
            if (residual) {
                uint16_t sum = enc(v + dec(residual[base + i], dtype), dtype);
                residual_out[base + i] = sum;
                v = dec(sum, dtype);
            }
            h[i] = v;
        }
        double ms = 0.0;
        for (int i = 0; i < hidden; ++i) ms += h[i] * h[i];
        ms /= hidden;
        double inv = 1.0 / sqrt(ms + eps);
        for (int i = 0; i < hidden; ++i) {
            double y = h[i] * inv * dec(w[i], dtype);
            out[base + i] = enc(y, dtype);
            if (exact_out) exact_out[base + i] = y;
        }
        free(h);
    }
}

/* ------------------------------------------------------------------------- */
/* chunked prefill  [ENGINE] s4.3                                              */
/* ------------------------------------------------------------------------- */

/*
 * Attention of a chunk of new query tokens per sequence over the paged cache, with
 * the causal mask slice [start_pos, start_pos + seq_len) of the page's forward:
 * sequence b contributes the query rows cu_q[b] .. cu_q[b+1]-1 (n_b = cu_q[b+1] - cu_q[b]);
 * its cache already holds the chunk (context_lens[b] = L_b tokens), so query row i sits at
 * position start_pos + i with start_pos = L_b - n_b and sees keys 0 .. start_pos + i.
 *   q: [cu_q[batch]][q_heads][head_dim] storage; pools and block tables as in
 *   ora_decode_attention; out: [cu_q[batch]][q_heads][head_dim] double.
 */
void ora_prefill_attention(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                           const int32_t* block_tables, int max_pages_per_seq, const int32_t* cu_q,
                           const int32_t* context_lens, int batch, int q_heads, int kv_heads,
                           int head_dim, int page_size, double scale, int dtype, double* out)
{
    int group = q_heads / kv_heads;
    for (int b = 0; b < batch; ++b) {
        int n = cu_q[b + 1] - cu_q[b];
        int len = context_lens[b];
        if (n <= 0) continue;
        int start = len - n;
        double* s = (double*)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
        for (int i = 0; i < n; ++i) {
            int pos = start + i;                     /* keys 0 .. pos are visible */
            for (int h = 0; h < q_heads; ++h) {
                int g = h / group;
                const uint16_t* qh = q + ((int64_t)(cu_q[b] + i) * q_heads + h) * head_dim;
                double* o = out + ((int64_t)(cu_q[b] + i) * q_heads + h) * head_dim;
                double mx = -INFINITY;
                for (int t = 0; t <= pos; ++t) {
                    int64_t page = block_tables[(int64_t)b * max_pages_per_seq + t / page_size];
                    const uint16_t* kr = k_pool + ((page * kv_heads + g) * page_size + t % page_size) * head_dim;
                    double dot = 0.0;
                    for (int e = 0; e < head_dim; ++e) dot += dec(qh[e], dtype) * dec(kr[e], dtype);
                    s[t] = scale * dot;
                    if (s[t] > mx) mx = s[t];
                }
                double z = 0.0;
                for (int t = 0; t <= pos; ++t) {
                    s[t] = exp(s[t] - mx);
                    z += s[t];
                }
                for (int e = 0; e < head_dim; ++e) o[e] = 0.0;
                for (int t = 0; t <= pos; ++t) {
                    int64_t page = block_tables[(int64_t)b * max_pages_per_seq + t / page_size];
                    const uint16_t* vr = v_pool + ((page * kv_heads + g) * page_size + t % page_size) * head_dim;
                    for (int e = 0; e < head_dim; ++e) o[e] += s[t] * dec(vr[e], dtype);
                }
                for (int e = 0; e < head_dim; ++e) o[e] /= z;
            }
        }
        free(s);
    }
}

/* ------------------------------------------------------------------------- */
/* int8 KV pages  [ENGINE] s3.4 (compression: store the cache in a smaller type) */
/* ------------------------------------------------------------------------- */

/*
 * Symmetric int8 quantisation of one head row of k or v (head_dim storage values):
 * amax = max |x_i|; codes q_i = round_half_even(x_i * (127 / amax)) in [-127, 127];
 * scale = amax / 127, so x_i ~ q_i * scale.  An all-zero row gets scale 0 and codes 0.
 * The decisions are taken in fp32 (each operation correctly rounded), the kernel's
 * precision, so that both sides produce the same codes.
 */
void ora_quantize_row_i8(const uint16_t* x, int head_dim, int dtype, int8_t* codes, float* scale_out)
{
    float amax = 0.0f;
    for (int i = 0; i < head_dim; ++i) {
        float a = (float)fabs(dec(x[i], dtype));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        for (int i = 0; i < head_dim; ++i) codes[i] = 0;
        *scale_out = 0.0f;
        return;
    }
    volatile float inv = 127.0f / amax;
    for (int i = 0; i < head_dim; ++i) {
        volatile float prod = (float)dec(x[i], dtype) * inv;
        float r = rintf(prod);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        codes[i] = (int8_t)r;
    }
    volatile float sc = amax / 127.0f;
    *scale_out = sc;
}

/*
 * Cache update into an int8 pool: the token of row b (k, v: [n][kv_heads][head_dim]
 * storage values) goes to position positions[b] of sequence b; each head row is quantised
 * with ora_quantize_row_i8.  Pools: codes [num_pages][kv_heads][page_size][head_dim],
 * scales [num_pages][kv_heads][page_size].
 */
void ora_kv_append_i8(int8_t* k_codes, int8_t* v_codes, float* k_scales, float* v_scales, const uint16_t* k,
                      const uint16_t* v, const int32_t* block_tables, int max_pages_per_seq, const int32_t* positions,
                      int n, int kv_heads, int page_size, int head_dim, int dtype)
{
    for (int b = 0; b < n; ++b) {
        int pos = positions[b];
        if (pos < 0) continue;
        int64_t page = block_tables[(int64_t)b * max_pages_per_seq + pos / page_size];
        int row = pos % page_size;
        for (int h = 0; h < kv_heads; ++h) {
            int64_t dst = (page * kv_heads + h) * page_size + row;
            int64_t src = ((int64_t)b * kv_heads + h) * head_dim;
            ora_quantize_row_i8(k + src, head_dim, dtype, k_codes + dst * head_dim, k_scales + dst);
            ora_quantize_row_i8(v + src, head_dim, dtype, v_codes + dst * head_dim, v_scales + dst);
        }
    }
}

/*
 * Decode attention over an int8 pool: token t's key is k_code * k_scale (and likewise v),
 * taken exactly in double; otherwise as ora_decode_attention_pairs.  q: storage values.
 */
void ora_decode_attention_i8_pairs(const uint16_t* q, const int8_t* k_codes, const int8_t* v_codes,
                                   const float* k_scales, const float* v_scales, const int32_t* block_tables,
                                   int max_pages_per_seq, const int32_t* context_lens, int q_heads, int kv_heads,
                                   int head_dim, int page_size, double scale, int dtype, const int32_t* pair_b,
                                   const int32_t* pair_h, int n_pairs, double* out)
{
    int group = q_heads / kv_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < n_pairs; ++p) {
        int b = pair_b[p], h = pair_h[p], g = h / group;
        int len = context_lens[b];
        double* o = out + (int64_t)p * head_dim;
        for (int i = 0; i < head_dim; ++i) o[i] = 0.0;
        if (len <= 0) continue;
        const uint16_t* qh = q + ((int64_t)b * q_heads + h) * head_dim;
        double* s = (double*)malloc(sizeof(double) * (size_t)len);
        double mx = -INFINITY;
        for (int t = 0; t < len; ++t) {
            int64_t row = (block_tables[(int64_t)b * max_pages_per_seq + t / page_size] * kv_heads + g) * page_size +
                          t % page_size;
            double dot = 0.0;
            for (int i = 0; i < head_dim; ++i)
                dot += dec(qh[i], dtype) * ((double)k_codes[row * head_dim + i] * (double)k_scales[row]);
            s[t] = scale * dot;
            if (s[t] > mx) mx = s[t];
        }
        double z = 0.0;
        for (int t = 0; t < len; ++t) {
            s[t] = exp(s[t] - mx);
            z += s[t];
        }
        for (int t = 0; t < len; ++t) {
            int64_t row = (block_tables[(int64_t)b * max_pages_per_seq + t / page_size] * kv_heads + g) * page_size +
                          t % page_size;
            for (int i = 0; i < head_dim; ++i)
                o[i] += s[t] * ((double)v_codes[row * head_dim + i] * (double)v_scales[row]);
        }
        for (int i = 0; i < head_dim; ++i) o[i] /= z;
        free(s);
    }
}

/*
 * Thread count of the pair routines: the OpenMP build uses n threads (n >= 1) and reports
 * how many it will use; the plain build always reports 1.
 */
#ifdef _OPENMP
#include <omp.h>
int ora_set_threads(int n)
{
    if (n >= 1) omp_set_num_threads(n);
    return omp_get_max_threads();
}
#else
int ora_set_threads(int n)
{
    (void)n;
    return 1;
}
#endif
