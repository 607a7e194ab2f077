/*
 * CPU oracle for paged decode attention and the decode-step KV append.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header, table or constant with
 * the CUDA library; the two meet only in the seeded input generator.
 *
 * Every result is the plain definition, in double precision, one output
 * element at a time, with no blocking, fusion or reordering:
 *
 *   attention   Attention(Q,K,V) = softmax(Q K^T / sqrt(d)) V, for the one new
 *               query of each running sequence against all of its cached keys
 *               and values ("vLLM inference cost optimisation", developer.aliyun.com,
 *               section 2 "what the KV cache actually stores").
 *   paging      the K/V of logical block i of a sequence live in the physical
 *               block named by entry i of its block table; logically contiguous,
 *               physically scattered (same article, section 4 "PagedAttention:
 *               manage the KV cache like virtual memory"; wzjinhao.cn vLLM
 *               write-up, section 2.1: the kernel reads KV block by block
 *               through the table instead of assuming it is contiguous).
 *   GQA         32 query heads over 8 KV heads: a group of query heads shares
 *               one KV head (Aliyun article, KV-cache sizing with GQA/MQA).
 *               Reading: query head g uses KV head g / (num_heads/num_kv_heads).
 *   append      each decode step writes the new token's K and V into the cache
 *               (Aliyun article, section 1 decode loop: "generate new K/V, write
 *               into the KV cache").
 *   FP8 KV      the cache may be stored at 8 bits (Aliyun article, section 15
 *               "the KV cache itself can be quantized"); per-tensor scales
 *               (promptx.wiki inference-optimisation tutorial, quantization
 *               section). Reading: E4M3 as defined by the OCP 8-bit floating
 *               point specification (bias 7, no infinities, S.1111.111 = NaN,
 *               largest finite 448), stored value = encode(x / scale) with the
 *               division in IEEE binary32 and the encode rounding to nearest,
 *               ties to even, saturating to +-448; dequantised value =
 *               decode(code) * scale.
 *               E5M2 (the other OCP 8-bit format; the wzjinhao.cn write-up,
 *               section 2.4, reports its accuracy drift as a KV format):
 *               bias 15, 2-bit mantissa, S.11111.00 = infinity, S.11111.xx
 *               (xx != 0) = NaN, largest finite 57344; the same encode rule
 *               (round to nearest even, magnitudes at or above 57344 saturate
 *               to it, NaN stays NaN).
 *   INT8 KV     the promptx.wiki tutorial's quantisation section also names
 *               8-bit integer KV caches. Reading: symmetric, one scale per
 *               tensor (or per KV head), code = clamp(round-half-even(x /
 *               scale), -127, 127) with the division in binary32, value =
 *               code * scale; NaN encodes to 0.
 *
 * Layouts (a reading: the pages give none):
 *   cache     [num_blocks][num_kv_heads][block_size][head_dim]
 *   q, out    [num_seqs][num_heads][head_dim]
 *   tables    int32 [num_seqs][max_blocks_per_seq]
 *   k, v rows [num_tokens][num_kv_heads][head_dim], slot = block*block_size + offset,
 *             negative slot = no write.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ---------------------------------------------------------------- values */

/* bfloat16 is the upper half of an IEEE binary32 word. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP E4M3: sign, 4-bit exponent with bias 7, 3-bit mantissa.
 * exponent 0 holds the subnormals m/8 * 2^-6; S.1111.111 is NaN. */
double orc_e4m3_value(uint8_t code)
{
    int s = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* The 127 non-negative finite E4M3 values in increasing order (code 0..126). */
static double e4m3_pos[127];
static int e4m3_ready = 0;

static void e4m3_init(void)
{
    if (e4m3_ready)
        return;
    for (int c = 0; c < 127; ++c)
        e4m3_pos[c] = orc_e4m3_value((uint8_t)c);
    e4m3_ready = 1;
}

/* Nearest representable value, ties to the even code, magnitudes above the
 * largest finite value saturate to it; NaN stays NaN (0x7F). */
uint8_t orc_e4m3_encode(float x)
{
    e4m3_init();
    if (isnan(x))
        return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= e4m3_pos[126])
        return sign | 126;
    /* largest code lo with e4m3_pos[lo] <= a (binary search), hi = lo + 1 */
    int lo = 0, hi = 126;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_pos[mid] <= a)
            lo = mid;
        else
            hi = mid;
    }
    double vlo = e4m3_pos[lo], vhi = e4m3_pos[hi];
    double midpoint = 0.5 * (vlo + vhi); /* exact: both are short binary fractions */
    int code;
    if (a < midpoint)
        code = lo;
    else if (a > midpoint)
        code = hi;
    else
        code = (lo & 1) ? hi : lo;
    return sign | (uint8_t)code;
}

void orc_e4m3_encode_array(const float* x, uint8_t* codes, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        codes[i] = orc_e4m3_encode(x[i]);
}

/* OCP E5M2: sign, 5-bit exponent with bias 15, 2-bit mantissa; exponent 0
 * holds the subnormals m/4 * 2^-14; exponent 31 is infinity (m = 0) or NaN. */
double orc_e5m2_value(uint8_t code)
{
    int s = code >> 7;
    int e = (code >> 2) & 0x1F;
    int m = code & 0x3;
    double v;
    if (e == 0x1F)
        v = m == 0 ? INFINITY : NAN;
    else if (e == 0)
        v = ldexp((double)m / 4.0, -14);
    else
        v = ldexp(1.0 + (double)m / 4.0, e - 15);
    return s ? -v : v;
}

/* The 124 non-negative finite E5M2 values in increasing order (code 0..0x7B). */
static double e5m2_pos[124];
static int e5m2_ready = 0;

static void e5m2_init(void)
{
    if (e5m2_ready)
        return;
    for (int c = 0; c < 124; ++c)
        e5m2_pos[c] = orc_e5m2_value((uint8_t)c);
    e5m2_ready = 1;
}

/* Same rule as the E4M3 encoder over the E5M2 value set. */
uint8_t orc_e5m2_encode(float x)
{
    e5m2_init();
    if (isnan(x))
        return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= e5m2_pos[123])
        return sign | 123;
    int lo = 0, hi = 123;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e5m2_pos[mid] <= a)
            lo = mid;
        else
            hi = mid;
    }
    double vlo = e5m2_pos[lo], vhi = e5m2_pos[hi];
    double midpoint = 0.5 * (vlo + vhi);
    int code;
    if (a < midpoint)
        code = lo;
    else if (a > midpoint)
        code = hi;
    else
        code = (lo & 1) ? hi : lo;
    return sign | (uint8_t)code;
}

void orc_e5m2_encode_array(const float* x, uint8_t* codes, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        codes[i] = orc_e5m2_encode(x[i]);
}

/* Symmetric 8-bit integer code: nearest integer to x (ties to even), clamped to +-127. */
int8_t orc_int8_encode(float x)
{
    if (isnan(x))
        return 0;
    if (x >= 127.0f)
        return 127;
    if (x <= -127.0f)
        return -127;
    double r = floor((double)x);
    double frac = (double)x - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))
        r += 1.0;
    return (int8_t)r;
}

/* the 8-bit caches: quantised with a scale */
static int is_fp8(int dtype) { return dtype == ORC_E4M3 || dtype == ORC_E5M2 || dtype == ORC_INT8; }

static double elem(const void* base, int dtype, size_t i, double scale)
{
    switch (dtype) {
    case ORC_F32:
        return (double)((const float*)base)[i];
    case ORC_BF16:
        return bf16_value(((const uint16_t*)base)[i]);
    case ORC_E4M3:
        return orc_e4m3_value(((const uint8_t*)base)[i]) * scale;
    case ORC_E5M2:
        return orc_e5m2_value(((const uint8_t*)base)[i]) * scale;
    case ORC_INT8:
        return (double)((const int8_t*)base)[i] * scale;
    default:
        return NAN;
    }
}

static size_t dtype_size(int dtype)
{
    return dtype == ORC_F32 ? 4 : dtype == ORC_BF16 ? 2 : 1;
}

/* ------------------------------------------------------------- attention */

int orc_paged_decode_lse(double* out, double* lse,
                         const void* q, int q_dtype,
                         const void* k_cache, const void* v_cache, int kv_dtype,
                         const int32_t* block_tables, const int32_t* seq_lens,
                         int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                         int block_size, int max_blocks_per_seq, int num_blocks,
                         double scale, double k_scale, double v_scale,
                         const int32_t* seqs, int n_seqs, int q_len,
                         const float* k_head_scales, const float* v_head_scales)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0 || q_len < 1)
        return ORC_ERR_SHAPE;
    if (is_fp8(q_dtype) || q_dtype < 0 || q_dtype > 4 || kv_dtype < 0 || kv_dtype > 4)
        return ORC_ERR_DTYPE;
    const int group = num_heads / num_kv_heads;
    const int count = seqs ? n_seqs : num_seqs;
    int status = ORC_OK;
    size_t cap = 0;
    double* x = NULL;

    for (int r = 0; r < count; ++r) {
        const int s = seqs ? seqs[r] : r;
        if (s < 0 || s >= num_seqs) {
            status = ORC_ERR_INDEX;
            goto done;
        }
        const int L = seq_lens[s];
        if (L < 0 || L > max_blocks_per_seq * block_size) {
            status = ORC_ERR_INDEX;
            goto done;
        }
        if ((size_t)L > cap) {
            free(x);
            cap = (size_t)L;
            x = (double*)malloc(cap * sizeof(double));
            if (!x) {
                status = ORC_ERR_ALLOC;
                goto done;
            }
        }
        /* query j of the q_len new tokens sits at position L - q_len + j and sees the
         * tokens up to and including itself: Lq = L - q_len + 1 + j of them */
        for (int gq = 0; gq < q_len * num_heads; ++gq) {
            const int j = gq / num_heads, g = gq % num_heads;
            const int Lq = L - q_len + 1 + j;
            double* o = out + ((size_t)r * q_len * num_heads + gq) * head_dim;
            const int h = g / group;
            /* FP8 dequantisation scale: one per tensor, or one per KV head when given */
            const double ksc = k_head_scales ? (double)k_head_scales[h] : k_scale;
            const double vsc = v_head_scales ? (double)v_head_scales[h] : v_scale;
            for (int i = 0; i < head_dim; ++i)
                o[i] = 0.0;
            if (lse)
                lse[(size_t)r * q_len * num_heads + gq] = -INFINITY;
            if (Lq <= 0)
                continue;
            const size_t qoff = ((size_t)s * q_len * num_heads + gq) * head_dim;
            /* scores x_t = scale * q . K_t */
            for (int t = 0; t < Lq; ++t) {
                const int32_t p = block_tables[(size_t)s * max_blocks_per_seq + t / block_size];
                const int off = t % block_size;
                if (p < 0 || p >= num_blocks) {
                    status = ORC_ERR_INDEX;
                    goto done;
                }
                const size_t koff = (((size_t)p * num_kv_heads + h) * block_size + off) * head_dim;
                double dot = 0.0;
                for (int i = 0; i < head_dim; ++i)
                    dot += elem(q, q_dtype, qoff + i, 1.0) * elem(k_cache, kv_dtype, koff + i, ksc);
                x[t] = scale * dot;
            }
            /* softmax weights w_t = exp(x_t - max x) and the weighted sum of V_t */
            double m = x[0];
            for (int t = 1; t < Lq; ++t)
                if (x[t] > m)
                    m = x[t];
            double denom = 0.0;
            for (int t = 0; t < Lq; ++t) {
                const int32_t p = block_tables[(size_t)s * max_blocks_per_seq + t / block_size];
                const int off = t % block_size;
                const size_t voff = (((size_t)p * num_kv_heads + h) * block_size + off) * head_dim;
                const double w = exp(x[t] - m);
                denom += w;
                for (int i = 0; i < head_dim; ++i)
                    o[i] += w * elem(v_cache, kv_dtype, voff + i, vsc);
            }
            for (int i = 0; i < head_dim; ++i)
                o[i] /= denom;
            /* log of the softmax denominator: log sum_t exp(x_t) = m + log sum_t exp(x_t - m) */
            if (lse)
                lse[(size_t)r * q_len * num_heads + gq] = m + log(denom);
        }
    }
done:
    free(x);
    return status;
}

int orc_paged_decode(double* out,
                     const void* q, int q_dtype,
                     const void* k_cache, const void* v_cache, int kv_dtype,
                     const int32_t* block_tables, const int32_t* seq_lens,
                     int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                     int block_size, int max_blocks_per_seq, int num_blocks,
                     double scale, double k_scale, double v_scale,
                     const int32_t* seqs, int n_seqs, int q_len,
                     const float* k_head_scales, const float* v_head_scales)
{
    return orc_paged_decode_lse(out, NULL, q, q_dtype, k_cache, v_cache, kv_dtype, block_tables, seq_lens,
                                num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                                num_blocks, scale, k_scale, v_scale, seqs, n_seqs, q_len, k_head_scales,
                                v_head_scales);
}

/* ---------------------------------------------------------------- append */

int orc_reshape_and_cache(const void* k, const void* v, int in_dtype,
                          void* k_cache, void* v_cache, int kv_dtype,
                          const int64_t* slot_mapping, const int64_t* rows, int64_t n_rows,
                          int num_tokens, int num_kv_heads, int head_dim,
                          int block_size, int num_blocks, float k_scale, float v_scale,
                          const float* k_head_scales, const float* v_head_scales)
{
    if (is_fp8(in_dtype) || in_dtype < 0 || in_dtype > 4 || kv_dtype < 0 || kv_dtype > 4)
        return ORC_ERR_DTYPE;
    if (!is_fp8(kv_dtype) && kv_dtype != in_dtype)
        return ORC_ERR_DTYPE;
    const size_t isz = dtype_size(in_dtype), csz = dtype_size(kv_dtype);
    const int64_t capacity = (int64_t)num_blocks * block_size;
    const int64_t count = rows ? n_rows : num_tokens;
    int status = ORC_OK;
    for (int64_t r = 0; r < count; ++r) {
        const int64_t t = rows ? rows[r] : r;
        if (t < 0 || t >= num_tokens)
            return ORC_ERR_INDEX;
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue; /* padding token: nothing written */
        if (slot >= capacity) {
            status = ORC_ERR_INDEX;
            continue;
        }
        const int64_t blk = slot / block_size, off = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            const size_t src = ((size_t)t * num_kv_heads + h) * head_dim;
            const size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + (size_t)off) * head_dim;
            if (kv_dtype == in_dtype) {
                memcpy((char*)k_cache + dst * csz, (const char*)k + src * isz, head_dim * isz);
                memcpy((char*)v_cache + dst * csz, (const char*)v + src * isz, head_dim * isz);
                continue;
            }
            for (int i = 0; i < head_dim; ++i) {
                const float kx = (float)elem(k, in_dtype, src + i, 1.0);
                const float vx = (float)elem(v, in_dtype, src + i, 1.0);
                const float ky = kx / (k_head_scales ? k_head_scales[h] : k_scale); /* binary32 division */
                const float vy = vx / (v_head_scales ? v_head_scales[h] : v_scale);
                if (kv_dtype == ORC_INT8) {
                    ((int8_t*)k_cache)[dst + i] = orc_int8_encode(ky);
                    ((int8_t*)v_cache)[dst + i] = orc_int8_encode(vy);
                    continue;
                }
                ((uint8_t*)k_cache)[dst + i] = kv_dtype == ORC_E4M3 ? orc_e4m3_encode(ky) : orc_e5m2_encode(ky);
                ((uint8_t*)v_cache)[dst + i] = kv_dtype == ORC_E4M3 ? orc_e4m3_encode(vy) : orc_e5m2_encode(vy);
            }
        }
    }
    return status;
}
