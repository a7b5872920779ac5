/*
 * Plain fp64 CPU oracle for the PagedAttention decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file: only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or helper with the CUDA
 * library; the two only ever see the same seeded input arrays.
 *
 * Sources (the pages this restates, by title and section):
 *   - comfyai.app "6.4 PagedAttention", 6.4.1 Mechanism: a sequence's KV is
 *     split into fixed-length blocks; a block table maps logically contiguous
 *     blocks onto physically non-contiguous ones.
 *   - brentwoodlivery.com "5.3.18 LLM serving, vLLM, quantized inference",
 *     "Common mistake: PagedAttention makes the attention math faster": the
 *     attention computation is unchanged, only memory layout/allocation is.
 *     The same page gives the KV size formula 2*B*S*L*d_model*p.
 *   - polomodov.tech "vLLM and PagedAttention", slide 9 (the kernel fetches
 *     K and V from non-contiguous blocks by their addresses), slide 10 (the
 *     block table, logical 0-3 -> physical 7, 1, 3, unallocated), slide 11
 *     (a new physical block only once the previous one is full), slide 13
 *     (copy-on-write copies only the last block).
 *   - comfyai.app 6.4.2/6.4.3: shared blocks are read-only; a write to a
 *     shared block first copies it (copy-on-write).
 *
 * Everything is computed in double.  Every fp16 input is widened exactly to
 * double by the IEEE 754 binary16 definition (oracle_half_to_double).
 *
 * Readings where the pages are silent (the plainest reading in each case):
 *   - slot encoding: slot = physical_block * block_size + offset_in_block;
 *     a negative slot marks a padding token that is not written.
 *   - decode attends over positions t < context_len, no causal mask (one
 *     query per sequence and head); positions >= context_len are never read.
 *   - context_len == 0 gives an all-zero output.
 *   - multi-head attention with as many K/V heads as query heads.
 *
 * Return codes: 0 ok, 1 invalid argument, 2 out-of-range block id or slot.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_RANGE 2

/* IEEE 754 binary16 -> double, from the format's definition:
 * sign(1) | exponent(5, bias 15) | fraction(10).  exponent 0: subnormal
 * fraction * 2^-24; exponent 31: inf / NaN; otherwise (1024 + fraction) *
 * 2^(exponent - 25). */
double oracle_half_to_double(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 1024), expo - 25);
    return sign ? -v : v;
}

/* All 65536 binary16 values, decoded once by oracle_half_to_double (so the
 * table is that definition evaluated, not a second decoder). */
static double half_table[1 << 16];
static pthread_once_t half_table_once = PTHREAD_ONCE_INIT;

static void fill_half_table(void)
{
    for (uint32_t i = 0; i < (1u << 16); ++i)
        half_table[i] = oracle_half_to_double((uint16_t)i);
}

static inline double h2d(uint16_t bits)
{
    return half_table[bits];
}

/* KV cache size in bytes, brentwoodlivery.com 5.3.18 ("KV cache size bytes
 * mein formula"): 2 (K and V) * batch * sequence length * layers * d_model *
 * bytes per element. */
int64_t oracle_kv_cache_bytes(int64_t batch, int64_t seq_len, int64_t layers,
                              int64_t d_model, int64_t bytes_per_elem)
{
    return 2 * batch * seq_len * layers * d_model * bytes_per_elem;
}

/* Cache write (polomodov.tech slide 11: the new token goes into the next free
 * slot of the sequence's last block).  For token i with slot >= 0, copy its
 * H x D fp16 key and value rows into cache[slot / bs, h, slot % bs, :].
 * Layouts: key/value [N, H, D]; caches [NB, H, bs, D]; all fp16 bit patterns. */
int oracle_reshape_and_cache(const uint16_t *key, const uint16_t *value,
                             uint16_t *k_cache, uint16_t *v_cache,
                             const int64_t *slot_mapping, int num_tokens,
                             int num_heads, int head_dim, int block_size,
                             int num_blocks)
{
    if (num_tokens < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0)
        return ORACLE_ERR_ARG;
    const int64_t H = num_heads, D = head_dim, bs = block_size;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * bs)
            return ORACLE_ERR_RANGE;
        int64_t block = slot / bs;
        int64_t offset = slot % bs;
        for (int64_t h = 0; h < H; ++h) {
            const uint16_t *ks = key + ((int64_t)i * H + h) * D;
            const uint16_t *vs = value + ((int64_t)i * H + h) * D;
            uint16_t *kd = k_cache + ((block * H + h) * bs + offset) * D;
            uint16_t *vd = v_cache + ((block * H + h) * bs + offset) * D;
            memcpy(kd, ks, (size_t)D * sizeof(uint16_t));
            memcpy(vd, vs, (size_t)D * sizeof(uint16_t));
        }
    }
    return ORACLE_OK;
}

/* Copy-on-write block copy (comfyai.app 6.4.2-6.4.3; polomodov.tech slide 13):
 * for each pair (src, dst), every element of physical block src is copied to
 * physical block dst, in both caches.  block_mapping is [P, 2] (src, dst). */
int oracle_copy_blocks(uint16_t *k_cache, uint16_t *v_cache,
                       const int64_t *block_mapping, int num_pairs,
                       int num_heads, int head_dim, int block_size,
                       int num_blocks)
{
    if (num_pairs < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0)
        return ORACLE_ERR_ARG;
    const int64_t block_elems = (int64_t)num_heads * block_size * head_dim;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks)
            return ORACLE_ERR_RANGE;
        memmove(k_cache + dst * block_elems, k_cache + src * block_elems,
                (size_t)block_elems * sizeof(uint16_t));
        memmove(v_cache + dst * block_elems, v_cache + src * block_elems,
                (size_t)block_elems * sizeof(uint16_t));
    }
    return ORACLE_OK;
}

/* One (sequence, head) of paged decode attention, in double.
 *   K_t = k_cache[block_tables[b][t / bs], h, t % bs, :]   (same for V_t)
 *   s_t = scale * sum_d q[b,h,d] * K_t[d]
 *   w_t = exp(s_t - max_t s_t)
 *   out = sum_t w_t V_t / sum_t w_t
 * The attention itself is the ordinary softmax attention (the paging changes
 * only where K_t and V_t are read from).  probs, if non-null, receives the
 * normalised weights w_t / sum w (context_len entries).  scores is scratch of
 * context_len doubles. */
static int decode_one(double *out, double *probs, double *scores,
                      const uint16_t *q, const uint16_t *k_cache,
                      const uint16_t *v_cache, const int32_t *table, int len,
                      int h, int64_t H, int64_t D, int64_t bs, int64_t NB,
                      double scale)
{
    for (int64_t d = 0; d < D; ++d)
        out[d] = 0.0;
    if (len == 0)
        return ORACLE_OK;

    double m = -INFINITY;
    for (int t = 0; t < len; ++t) {
        int64_t p = table[t / bs];
        if (p < 0 || p >= NB)
            return ORACLE_ERR_RANGE;
        const uint16_t *k = k_cache + ((p * H + h) * bs + t % bs) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d)
            dot += h2d(q[d]) * h2d(k[d]);
        scores[t] = scale * dot;
        if (scores[t] > m)
            m = scores[t];
    }

    double l = 0.0;
    for (int t = 0; t < len; ++t) {
        scores[t] = exp(scores[t] - m);
        l += scores[t];
    }

    for (int t = 0; t < len; ++t) {
        int64_t p = table[t / bs];
        const uint16_t *v = v_cache + ((p * H + h) * bs + t % bs) * D;
        for (int64_t d = 0; d < D; ++d)
            out[d] += scores[t] * h2d(v[d]);
    }
    for (int64_t d = 0; d < D; ++d)
        out[d] /= l;
    if (probs)
        for (int t = 0; t < len; ++t)
            probs[t] = scores[t] / l;
    return ORACLE_OK;
}

/* Paged decode attention for every (sequence, head).
 *   out   [B, H, D] double
 *   probs [B, H, probs_stride] double or NULL (the softmax weights)
 *   q     [B, H, D] fp16; caches [NB, H, bs, D] fp16
 *   block_tables [B, max_blocks_per_seq] int32; context_lens [B] int32
 * Only the table entries t / bs for t < context_len are read. */
int oracle_paged_decode(double *out, double *probs, int64_t probs_stride,
                        const uint16_t *q, const uint16_t *k_cache,
                        const uint16_t *v_cache, const int32_t *block_tables,
                        int max_blocks_per_seq, const int32_t *context_lens,
                        int num_seqs, int num_heads, int head_dim,
                        int block_size, int num_blocks, double scale)
{
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq < 0)
        return ORACLE_ERR_ARG;
    const int64_t H = num_heads, D = head_dim, bs = block_size;
    for (int b = 0; b < num_seqs; ++b) {
        int len = context_lens[b];
        if (len < 0 || (int64_t)len > (int64_t)max_blocks_per_seq * bs)
            return ORACLE_ERR_ARG;
        if (probs && (int64_t)len > probs_stride)
            return ORACLE_ERR_ARG;
    }

    pthread_once(&half_table_once, fill_half_table);
    int status = ORACLE_OK;
    const int64_t units = (int64_t)num_seqs * H;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : status)
    for (int64_t u = 0; u < units; ++u) {
        int b = (int)(u / H), h = (int)(u % H);
        int len = context_lens[b];
        double *scores = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
        if (!scores) {
            status = status > ORACLE_ERR_ARG ? status : ORACLE_ERR_ARG;
            continue;
        }
        int rc = decode_one(out + u * D, probs ? probs + u * probs_stride : NULL,
                            scores, q + u * D, k_cache, v_cache,
                            block_tables + (int64_t)b * max_blocks_per_seq, len,
                            h, H, D, bs, num_blocks, scale);
        free(scores);
        if (rc > status)
            status = rc;
    }
    return status;
}

/* Multi-query (prefill / chunked prefill) paged attention
 * (brentwoodlivery.com 5.3.18: prefill processes all prompt tokens at once;
 * polomodov.tech slide 11: the prompt's tokens are written into blocks, then
 * decoding continues).  Sequence b holds L = context_lens[b] tokens in the
 * cache, the last n = query_start_loc[b+1] - query_start_loc[b] of which are
 * new.  Query token i of b (row query_start_loc[b] + i of q / out) sits at
 * position p = L - n + i and attends causally to every cached t <= p:
 * out = softmax_t(scale q.K_t) V over t in [0, p] -- the decode arithmetic
 * with context length p + 1.  q, out [num_tokens, H, D]. */
int oracle_paged_prefill(double *out, const uint16_t *q, const uint16_t *k_cache,
                         const uint16_t *v_cache, const int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *context_lens,
                         const int32_t *query_start_loc, int num_seqs, int num_heads,
                         int head_dim, int block_size, int num_blocks, double scale)
{
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq < 0)
        return ORACLE_ERR_ARG;
    pthread_once(&half_table_once, fill_half_table);
    const int64_t H = num_heads, D = head_dim, bs = block_size;
    for (int b = 0; b < num_seqs; ++b) {
        const int n = query_start_loc[b + 1] - query_start_loc[b];
        const int len = context_lens[b];
        if (n < 0 || n > len || (int64_t)len > (int64_t)max_blocks_per_seq * bs)
            return ORACLE_ERR_ARG;
    }
    const int64_t tokens = query_start_loc[num_seqs];
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : status)
    for (int64_t u = 0; u < tokens * H; ++u) {
        const int64_t tok = u / H;
        const int h = (int)(u % H);
        int b = 0;
        while (query_start_loc[b + 1] <= tok)
            ++b;
        const int n = query_start_loc[b + 1] - query_start_loc[b];
        const int pos = context_lens[b] - n + (int)(tok - query_start_loc[b]);
        double *scores = (double *)malloc(sizeof(double) * (size_t)(pos + 1));
        if (!scores) {
            status = status > ORACLE_ERR_ARG ? status : ORACLE_ERR_ARG;
            continue;
        }
        const int rc = decode_one(out + u * D, NULL, scores, q + u * D, k_cache, v_cache,
                                  block_tables + (int64_t)b * max_blocks_per_seq, pos + 1, h, H, D,
                                  bs, num_blocks, scale);
        free(scores);
        if (rc > status)
            status = rc;
    }
    return status;
}

/* ------------------------------------------------------------------------
 * Low-bit KV cache (brentwoodlivery.com "5.3.18 LLM serving, vLLM, quantized
 * inference": the KV cache can be kept in low-bit integer formats; affine
 * quantization s = (r_max - r_min) / (2^b - 1), z = round(-r_min / s),
 * q = round(r / s) + z, r_hat = s (q - z), with one (s, z) per group of
 * values; the page uses groups of 128).  Here a group is one (token, head)
 * row of head_dim values, b = 8, codes stored as uint8 (clamped to
 * [0, 2^b - 1]).  The rounding decisions are taken in fp32, the precision
 * the GPU kernel uses (the page fixes none); round = round half to even.
 * A row whose values are all equal (r_max == r_min = c) has no spread: it
 * uses s = |c| (or 1 when c is 0), so z = -sign(c), every code is 0 and
 * s (0 - z) = c exactly.
 */
static void quantize_row_f32(const uint16_t *x, int64_t D, int bits, uint8_t *codes,
                             float *s_out, float *z_out)
{
    const float qmax = (float)((1 << bits) - 1);
    float rmin = INFINITY, rmax = -INFINITY;
    for (int64_t d = 0; d < D; ++d) {
        const float v = (float)h2d(x[d]);
        if (v < rmin)
            rmin = v;
        if (v > rmax)
            rmax = v;
    }
    float s = (rmax - rmin) / qmax;
    if (s == 0.0f)
        s = rmax != 0.0f ? fabsf(rmax) : 1.0f;
    const float z = rintf(-rmin / s);
    for (int64_t d = 0; d < D; ++d) {
        float q = rintf((float)h2d(x[d]) / s) + z;
        if (q < 0.0f)
            q = 0.0f;
        if (q > qmax)
            q = qmax;
        codes[d] = (uint8_t)q;
    }
    *s_out = s;
    *z_out = z;
}

/* Quantize n rows of D fp16 values: codes [n, D] uint8, params [n, 2] (s, z). */
int oracle_quantize_rows(const uint16_t *x, int n, int D, int bits, uint8_t *codes, float *params)
{
    if (n < 0 || D <= 0 || bits < 2 || bits > 8)
        return ORACLE_ERR_ARG;
    pthread_once(&half_table_once, fill_half_table);
    for (int i = 0; i < n; ++i)
        quantize_row_f32(x + (int64_t)i * D, D, bits, codes + (int64_t)i * D, &params[2 * i],
                         &params[2 * i + 1]);
    return ORACLE_OK;
}

/* Cache write into the int8 cache: token i's key/value row of head h is
 * quantized and stored at (slot / bs, h, slot % bs).  Caches: codes
 * [NB, H, bs, D] uint8, params [NB, H, bs, 2] float (s, z). */
int oracle_reshape_and_cache_int8(const uint16_t *key, const uint16_t *value, uint8_t *k_codes,
                                  uint8_t *v_codes, float *k_params, float *v_params,
                                  const int64_t *slot_mapping, int num_tokens, int num_heads,
                                  int head_dim, int block_size, int num_blocks)
{
    if (num_tokens < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return ORACLE_ERR_ARG;
    pthread_once(&half_table_once, fill_half_table);
    const int64_t H = num_heads, D = head_dim, bs = block_size;
    for (int i = 0; i < num_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * bs)
            return ORACLE_ERR_RANGE;
        const int64_t row0 = (slot / bs) * H * bs + slot % bs;
        for (int64_t h = 0; h < H; ++h) {
            const int64_t row = row0 + h * bs;
            quantize_row_f32(key + ((int64_t)i * H + h) * D, D, 8, k_codes + row * D,
                             &k_params[2 * row], &k_params[2 * row + 1]);
            quantize_row_f32(value + ((int64_t)i * H + h) * D, D, 8, v_codes + row * D,
                             &v_params[2 * row], &v_params[2 * row + 1]);
        }
    }
    return ORACLE_OK;
}

/* Paged decode over the int8 cache: each gathered row is dequantized exactly
 * (r_hat = s (q - z) in double) and the attention is the same as
 * oracle_paged_decode's. */
int oracle_paged_decode_int8(double *out, const uint16_t *q, const uint8_t *k_codes,
                             const uint8_t *v_codes, const float *k_params, const float *v_params,
                             const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *context_lens, int num_seqs, int num_heads,
                             int head_dim, int block_size, int num_blocks, double scale)
{
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq < 0)
        return ORACLE_ERR_ARG;
    pthread_once(&half_table_once, fill_half_table);
    const int64_t H = num_heads, D = head_dim, bs = block_size;
    for (int b = 0; b < num_seqs; ++b)
        if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)max_blocks_per_seq * bs)
            return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    const int64_t units = (int64_t)num_seqs * H;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : status)
    for (int64_t u = 0; u < units; ++u) {
        const int b = (int)(u / H), h = (int)(u % H);
        const int len = context_lens[b];
        const int32_t *table = block_tables + (int64_t)b * max_blocks_per_seq;
        double *o = out + u * D;
        for (int64_t d = 0; d < D; ++d)
            o[d] = 0.0;
        if (len == 0)
            continue;
        double *sc = (double *)malloc(sizeof(double) * (size_t)len);
        if (!sc) {
            status = status > ORACLE_ERR_ARG ? status : ORACLE_ERR_ARG;
            continue;
        }
        double m = -INFINITY;
        int rc = ORACLE_OK;
        for (int t = 0; t < len && rc == ORACLE_OK; ++t) {
            const int64_t p = table[t / bs];
            if (p < 0 || p >= num_blocks) {
                rc = ORACLE_ERR_RANGE;
                break;
            }
            const int64_t row = (p * H + h) * bs + t % bs;
            const double s = k_params[2 * row], z = k_params[2 * row + 1];
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d)
                dot += h2d(q[u * D + d]) * (s * ((double)k_codes[row * D + d] - z));
            sc[t] = scale * dot;
            if (sc[t] > m)
                m = sc[t];
        }
        if (rc == ORACLE_OK) {
            double l = 0.0;
            for (int t = 0; t < len; ++t) {
                sc[t] = exp(sc[t] - m);
                l += sc[t];
            }
            for (int t = 0; t < len; ++t) {
                const int64_t p = table[t / bs];
                const int64_t row = (p * H + h) * bs + t % bs;
                const double s = v_params[2 * row], z = v_params[2 * row + 1];
                for (int64_t d = 0; d < D; ++d)
                    o[d] += sc[t] * (s * ((double)v_codes[row * D + d] - z));
            }
            for (int64_t d = 0; d < D; ++d)
                o[d] /= l;
        }
        free(sc);
        if (rc > status)
            status = rc;
    }
    return status;
}

/* Number of OpenMP threads a parallel region would use (for reporting). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
