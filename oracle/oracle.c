/*
 * Plain fp64 CPU oracle for attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may build, load or call this file.
 * It shares no code, header, table or helper with the CUDA library; the two
 * meet only through the seeded inputs of paged_kv_attention_34_b200.workloads.
 *
 * What it computes, and where the pages say so:
 *
 *   attention     Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V
 *                 (ybb.press "LLM 推理优化", section 1, the attention formula).
 *                 The scale is an argument (1/sqrt(d) by default).
 *   paging        the cache is a pool of fixed 16-token blocks; a per-request
 *                 page table maps logical page p to a physical block
 *                 (iopencloud "大模型推理加速技术全景", section 3.2 and its
 *                 page-table figure; zhihu roofline page, "显存管理").
 *   varlen        sequences are packed back to back and delimited by a
 *                 cu_seqlens prefix sum; each sequence attends only to itself
 *                 (interview Q&A page, ragged batching answer).
 *   causal        query i of a sequence with q_b new tokens and ctx_b cached
 *                 keys (new tokens included) sits at position ctx_b - q_b + i
 *                 and sees keys 0 .. ctx_b - q_b + i.  The pages do not spell
 *                 out this alignment; it is the reading that makes a decode
 *                 query see its whole context and a chunk see its prefix.
 *   standard      the three-pass form: S = Q K^T materialised, softmax, then
 *                 S V (iopencloud section 2.1).  Used on tiny inputs.
 *   online        the running-max / running-sum recurrence over key blocks,
 *                 normalised once after the last block (iopencloud section
 *                 2.2, pseudocode; the final diag(l)^-1 is read as following
 *                 the loop).
 *   split merge   per-split partial results combined by their log-sum-exp
 *                 (interview Q&A page, FlashDecoding answer: split the KV
 *                 sequence across blocks, then a cross-block reduction).
 *   cache write   scatter of new K/V rows to slot = block*16 + offset; a
 *                 negative slot is a padding token and is skipped.
 *   block copy    copy-on-write of a shared block: all heads and 16 rows of
 *                 K and V of block src are copied to block dst (zhihu roofline
 *                 page, "显存管理": refcounted blocks, copy-on-write).
 *
 * 16-bit inputs are widened exactly to double from their bit patterns
 * (IEEE 754 binary16, and bfloat16 = the upper half of binary32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK 16

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1 };

/* ---- 16-bit formats -------------------------------------------------------- */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp(1.0 + (double)f / 1024.0, e - 15);
    return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_to_f64(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133); /* subnormal: f * 2^-126 * 2^-7 */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp(1.0 + (double)f / 128.0, e - 127);
    return sign ? -v : v;
}

static double widen(uint16_t x, int dtype)
{
    return dtype == ORACLE_F16 ? oracle_f16_to_f64(x) : oracle_bf16_to_f64(x);
}

/* ---- cache write and block copy (exact copies) ---------------------------- */

/* key_cache/value_cache: [num_blocks][H_kv][16][d]; k_new/v_new: [T][H_kv][d].
 * Returns the number of tokens whose slot was out of range (not written). */
int64_t oracle_kv_cache_write(const uint16_t *k_new, const uint16_t *v_new, const int32_t *slot_mapping,
                              int64_t T, uint16_t *key_cache, uint16_t *value_cache, int64_t num_blocks,
                              int H_kv, int d)
{
    int64_t bad = 0;
    for (int64_t t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue; /* padding token */
        if (slot >= num_blocks * ORACLE_BLOCK) {
            ++bad;
            continue;
        }
        int64_t block = slot / ORACLE_BLOCK;
        int64_t offset = slot % ORACLE_BLOCK;
        for (int h = 0; h < H_kv; ++h)
            for (int k = 0; k < d; ++k) {
                int64_t dst = ((block * H_kv + h) * ORACLE_BLOCK + offset) * d + k;
                int64_t src = (t * H_kv + h) * (int64_t)d + k;
                key_cache[dst] = k_new[src];
                value_cache[dst] = v_new[src];
            }
    }
    return bad;
}

/* pairs: [n][2] = (src, dst).  Returns the number of pairs skipped as out of range. */
int64_t oracle_kv_block_copy(uint16_t *key_cache, uint16_t *value_cache, int64_t num_blocks, int H_kv, int d,
                             const int32_t *pairs, int64_t n)
{
    int64_t bad = 0;
    int64_t per_block = (int64_t)H_kv * ORACLE_BLOCK * d;
    for (int64_t i = 0; i < n; ++i) {
        int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
            ++bad;
            continue;
        }
        for (int64_t e = 0; e < per_block; ++e) {
            key_cache[dst * per_block + e] = key_cache[src * per_block + e];
            value_cache[dst * per_block + e] = value_cache[src * per_block + e];
        }
    }
    return bad;
}

/* Swap of whole blocks between the device caches and a host pool (the interview
 * Q&A page, its answer on combining continuous batching with PagedAttention:
 * a preempted request's KV blocks go out to CPU memory and come back when it
 * resumes).  Pair i = (device block, host block); to_host != 0 copies device
 * -> host, else host -> device.  Pairs with an id out of range are skipped and
 * counted. */
int64_t oracle_kv_block_swap(uint16_t *key_cache, uint16_t *value_cache, int64_t num_blocks, uint16_t *host_key,
                             uint16_t *host_value, int64_t host_blocks, int H_kv, int d, const int32_t *pairs,
                             int64_t n, int to_host)
{
    int64_t bad = 0;
    int64_t per_block = (int64_t)H_kv * ORACLE_BLOCK * d;
    for (int64_t i = 0; i < n; ++i) {
        int64_t dev = pairs[2 * i], hst = pairs[2 * i + 1];
        if (dev < 0 || hst < 0 || dev >= num_blocks || hst >= host_blocks) {
            ++bad;
            continue;
        }
        for (int64_t e = 0; e < per_block; ++e) {
            if (to_host) {
                host_key[hst * per_block + e] = key_cache[dev * per_block + e];
                host_value[hst * per_block + e] = value_cache[dev * per_block + e];
            } else {
                key_cache[dev * per_block + e] = host_key[hst * per_block + e];
                value_cache[dev * per_block + e] = host_value[hst * per_block + e];
            }
        }
    }
    return bad;
}

/* ---- attention over the paged cache ---------------------------------------- */

/* One output row: query token t (of sequence b, index i within its q_b new
 * tokens), query head h.  Keys are gathered one by one through the block
 * table.  out_row receives d doubles.  Also returns the natural-log
 * log-sum-exp of the scaled scores when lse != NULL. */
/* Key j of a row is visible: every key up to `last` under the causal rule (tree == NULL); with a
 * tree mask, every cached key before the new tokens and new token j - base when its bit is set. */
static int key_visible(int j, int base, const int32_t *tree)
{
    return !tree || j < base || ((*tree >> (j - base)) & 1);
}

static int attention_row(double *out_row, double *lse, const uint16_t *q, const uint16_t *key_cache,
                         const uint16_t *value_cache, int dtype, const int32_t *block_tables, int max_blocks,
                         int b, int i, int q_b, int ctx_b, int64_t t, int h, int H_q, int H_kv, int d,
                         double scale, double *s /* scratch, >= ctx_b doubles */, const int32_t *tree)
{
    int G = H_q / H_kv;
    int g = h / G; /* consecutive query heads share one KV head */
    int last = ctx_b - q_b + i; /* causal: keys 0 .. last */
    int base = ctx_b - q_b;     /* first new token */
    if (tree)
        last = ctx_b - 1; /* tree verify: the mask decides among the new tokens */
    if (last < 0)
        return -1;
    const uint16_t *qrow = q + (t * H_q + h) * (int64_t)d;

    /* scores s_j = scale * <q, K_j> (masked keys: -inf) */
    for (int j = 0; j <= last; ++j) {
        if (!key_visible(j, base, tree)) {
            s[j] = -INFINITY;
            continue;
        }
        int64_t block = block_tables[(int64_t)b * max_blocks + j / ORACLE_BLOCK];
        int64_t off = j % ORACLE_BLOCK;
        const uint16_t *krow = key_cache + ((block * H_kv + g) * ORACLE_BLOCK + off) * d;
        double acc = 0.0;
        for (int k = 0; k < d; ++k)
            acc += widen(qrow[k], dtype) * widen(krow[k], dtype);
        s[j] = scale * acc;
    }
    /* softmax with the row maximum subtracted */
    double m = -INFINITY;
    for (int j = 0; j <= last; ++j)
        if (s[j] > m)
            m = s[j];
    if (m == -INFINITY)
        return -1; /* no visible key */
    double z = 0.0;
    for (int j = 0; j <= last; ++j) {
        s[j] = exp(s[j] - m);
        z += s[j];
    }
    /* O = sum_j softmax_j V_j */
    for (int k = 0; k < d; ++k)
        out_row[k] = 0.0;
    for (int j = 0; j <= last; ++j) {
        int64_t block = block_tables[(int64_t)b * max_blocks + j / ORACLE_BLOCK];
        int64_t off = j % ORACLE_BLOCK;
        const uint16_t *vrow = value_cache + ((block * H_kv + g) * ORACLE_BLOCK + off) * d;
        if (!key_visible(j, base, tree))
            continue; /* masked key of a tree row (its V may be anything) */
        double w = s[j] / z;
        for (int k = 0; k < d; ++k)
            out_row[k] += w * widen(vrow[k], dtype);
    }
    if (lse)
        *lse = m + log(z);
    return 0;
}

/* out: [n_rows][d] doubles.  rows: flattened (t * H_q + h) row ids to compute,
 * or NULL for all T*H_q rows (then out is [T][H_q][d]).  lse_out: optional
 * [n_rows] natural-log log-sum-exp per row.
 * Returns 0, or -1 if some sequence has ctx_b < q_b or q_b < 0,
 * -2 if H_q is not a multiple of H_kv. */
static int paged_attention_impl(double *out, double *lse_out, const uint16_t *q, const uint16_t *key_cache,
                           const uint16_t *value_cache, int dtype, const int32_t *block_tables, int max_blocks,
                           const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int H_q, int H_kv,
                           int d, double scale, const int64_t *rows, int64_t n_rows, int n_threads,
                                const int32_t *tree_mask)
{
    if (H_kv <= 0 || H_q % H_kv != 0)
        return -2;
    int max_ctx = 0;
    for (int b = 0; b < B; ++b) {
        int q_b = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
        if (q_b < 0 || context_lens[b] < q_b)
            return -1;
        if (context_lens[b] > max_ctx)
            max_ctx = context_lens[b];
    }
    int64_t T = cu_seqlens_q[B];
    int64_t total = rows ? n_rows : T * H_q;
    int status = 0;
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_ctx > 0 ? max_ctx : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < total; ++r) {
            int64_t row = rows ? rows[r] : r;
            int64_t t = row / H_q;
            int h = (int)(row % H_q);
            int b = 0; /* sequence owning token t */
            while (b < B && cu_seqlens_q[b + 1] <= t)
                ++b;
            int i = (int)(t - cu_seqlens_q[b]);
            int q_b = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
            int rc = attention_row(out + r * d, lse_out ? lse_out + r : NULL, q, key_cache, value_cache, dtype,
                                   block_tables, max_blocks, b, i, q_b, context_lens[b], t, h, H_q, H_kv, d,
                                   scale, s, tree_mask ? tree_mask + t : NULL);
            if (rc) {
#pragma omp atomic write
                status = rc;
            }
        }
        free(s);
    }
    return status;
}


int oracle_paged_attention(double *out, double *lse_out, const uint16_t *q, const uint16_t *key_cache,
                           const uint16_t *value_cache, int dtype, const int32_t *block_tables, int max_blocks,
                           const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int H_q, int H_kv,
                           int d, double scale, const int64_t *rows, int64_t n_rows, int n_threads)
{
    return paged_attention_impl(out, lse_out, q, key_cache, value_cache, dtype, block_tables, max_blocks,
                                cu_seqlens_q, context_lens, B, H_q, H_kv, d, scale, rows, n_rows, n_threads, NULL);
}

/* Tree-attention verification (the interview Q&A page, speculative decoding with a draft tree):
 * query token t of sequence b sees every cached key before the sequence's q_b new tokens, and new
 * token j exactly when bit j of tree_mask[t] is set (the drafts on its path from the root).  The
 * causal verify is the chain mask, bits 0 .. i for the i-th new token. */
int oracle_paged_attention_tree(double *out, double *lse_out, const uint16_t *q, const uint16_t *key_cache,
                                const uint16_t *value_cache, int dtype, const int32_t *block_tables, int max_blocks,
                                const int32_t *cu_seqlens_q, const int32_t *context_lens, const int32_t *tree_mask,
                                int B, int H_q, int H_kv, int d, double scale, const int64_t *rows, int64_t n_rows,
                                int n_threads)
{
    return paged_attention_impl(out, lse_out, q, key_cache, value_cache, dtype, block_tables, max_blocks,
                                cu_seqlens_q, context_lens, B, H_q, H_kv, d, scale, rows, n_rows, n_threads,
                                tree_mask);
}

/* ---- dense forms on contiguous fp64 data (tiny inputs) ---------------------- */

/* Standard three-pass attention: S = Q K^T * scale held in full, row softmax,
 * then P V.  q: [n_q][d], k, v: [n_k][d].  Query i sees keys j <= i + offset
 * (offset = n_k - n_q aligns the last query with the last key; a huge offset
 * disables the mask). */
void oracle_dense_attention(double *out, const double *q, const double *k, const double *v, int n_q, int n_k,
                            int d, double scale, int64_t offset)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)n_q * (size_t)n_k);
    for (int i = 0; i < n_q; ++i)
        for (int j = 0; j < n_k; ++j) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += q[(int64_t)i * d + c] * k[(int64_t)j * d + c];
            S[(int64_t)i * n_k + j] = (j <= i + offset) ? scale * acc : -INFINITY;
        }
    for (int i = 0; i < n_q; ++i) {
        double *row = S + (int64_t)i * n_k;
        double m = -INFINITY, z = 0.0;
        for (int j = 0; j < n_k; ++j)
            if (row[j] > m)
                m = row[j];
        for (int j = 0; j < n_k; ++j) {
            row[j] = (row[j] == -INFINITY) ? 0.0 : exp(row[j] - m);
            z += row[j];
        }
        for (int j = 0; j < n_k; ++j)
            row[j] /= z;
    }
    for (int i = 0; i < n_q; ++i)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < n_k; ++j)
                acc += S[(int64_t)i * n_k + j] * v[(int64_t)j * d + c];
            out[(int64_t)i * d + c] = acc;
        }
    free(S);
}

/* Online softmax for one query row over keys in blocks of `block` keys:
 * running max m and running sum l, the accumulator rescaled by
 * exp(m_prev - m_new) whenever the max moves, and one division by l after
 * the last block.  q: [d], k, v: [n_k][d]. */
void oracle_online_softmax(double *out, const double *q, const double *k, const double *v, int n_k, int d,
                           double scale, int block)
{
    double m = -INFINITY, l = 0.0;
    double *o = (double *)calloc((size_t)d, sizeof(double));
    double *s = (double *)malloc(sizeof(double) * (size_t)(block > 0 ? block : 1));
    for (int j0 = 0; j0 < n_k; j0 += block) {
        int nb = (n_k - j0 < block) ? n_k - j0 : block;
        double bmax = -INFINITY;
        for (int j = 0; j < nb; ++j) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += q[c] * k[(int64_t)(j0 + j) * d + c];
            s[j] = scale * acc;
            if (s[j] > bmax)
                bmax = s[j];
        }
        double m_new = m > bmax ? m : bmax;
        double alpha = exp(m - m_new); /* 0 on the first block */
        double rowsum = 0.0;
        for (int j = 0; j < nb; ++j) {
            s[j] = exp(s[j] - m_new);
            rowsum += s[j];
        }
        l = alpha * l + rowsum;
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < nb; ++j)
                acc += s[j] * v[(int64_t)(j0 + j) * d + c];
            o[c] = alpha * o[c] + acc;
        }
        m = m_new;
    }
    for (int c = 0; c < d; ++c)
        out[c] = o[c] / l;
    free(o);
    free(s);
}

/* Attention of one query row restricted to keys [lo, hi): the normalised
 * partial output and its natural-log log-sum-exp (-inf and zeros when the
 * range is empty).  This is one split of split-KV decoding. */
void oracle_attention_partial(double *out, double *lse, const double *q, const double *k, const double *v, int lo,
                              int hi, int d, double scale)
{
    double m = -INFINITY;
    for (int c = 0; c < d; ++c)
        out[c] = 0.0;
    if (hi <= lo) {
        *lse = -INFINITY;
        return;
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)(hi - lo));
    for (int j = lo; j < hi; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
            acc += q[c] * k[(int64_t)j * d + c];
        s[j - lo] = scale * acc;
        if (s[j - lo] > m)
            m = s[j - lo];
    }
    double z = 0.0;
    for (int j = lo; j < hi; ++j) {
        s[j - lo] = exp(s[j - lo] - m);
        z += s[j - lo];
    }
    for (int j = lo; j < hi; ++j)
        for (int c = 0; c < d; ++c)
            out[c] += s[j - lo] / z * v[(int64_t)j * d + c];
    *lse = m + log(z);
    free(s);
}

/* Cross-split reduction: O = sum_s exp(lse_s - lse) O_s with
 * lse = log sum_s exp(lse_s).  Splits with lse_s = -inf contribute nothing.
 * parts: [n_splits][d], lses: [n_splits]. */
void oracle_lse_merge(double *out, double *lse_out, const double *parts, const double *lses, int n_splits, int d)
{
    double m = -INFINITY;
    for (int s = 0; s < n_splits; ++s)
        if (lses[s] > m)
            m = lses[s];
    for (int c = 0; c < d; ++c)
        out[c] = 0.0;
    if (m == -INFINITY) {
        *lse_out = -INFINITY;
        return;
    }
    double z = 0.0;
    for (int s = 0; s < n_splits; ++s)
        z += exp(lses[s] - m);
    for (int s = 0; s < n_splits; ++s) {
        double w = exp(lses[s] - m) / z;
        for (int c = 0; c < d; ++c)
            out[c] += w * parts[(int64_t)s * d + c];
    }
    *lse_out = m + log(z);
}

/* ---- FP8 (E4M3) KV cache ------------------------------------------------------
 * An 8-bit cache with one float scale per stored row (token, KV head): the FP8 KV cache of the
 * serving pages (vLLM's fp8 KV-cache option; FP8 with scaling on the interview Q&A page).  The
 * scale of a row is set when the row is written, amax / 448, so nothing already stored ever has
 * to be requantised.  E4M3 (OCP 8-bit floating point): sign, 4 exponent bits with bias 7, 3
 * mantissa bits, subnormals, no infinities, S.1111.111 = NaN, largest finite 448. */

double oracle_e4m3_to_f64(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6); /* subnormal: 0.m x 2^-6 */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* The E4M3 code nearest to x (ties to the code with an even last bit), saturated to +-448:
 * every finite non-negative code is tried. */
uint8_t oracle_f64_to_e4m3(double x)
{
    if (isnan(x))
        return 0x7f;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0)
        return sign | 0x7e;
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        double err = fabs(a - oracle_e4m3_to_f64((uint8_t)c));
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return sign | (uint8_t)best;
}

/* One row of d 16-bit values -> d codes (code k at dst[k * stride]) and the row's scale:
 * scale = amax / 448 (1 when amax is 0), code_k = e4m3(x_k / scale), both divisions in float
 * rounded to nearest, as the device does. */
static float quant_row(const uint16_t *src, int dtype, int d, uint8_t *dst, int64_t stride)
{
    float amax = 0.0f;
    for (int k = 0; k < d; ++k) {
        float v = fabsf((float)widen(src[k], dtype));
        if (v > amax)
            amax = v;
    }
    float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int k = 0; k < d; ++k) {
        float q = (float)widen(src[k], dtype) / sc;
        dst[k * stride] = oracle_f64_to_e4m3((double)q);
    }
    return sc;
}

/* kv_cache_write into the FP8 cache.  Per (block, KV head): K codes [16 slots][d], V codes
 * transposed, [d][16 slots] (the value-cache layout of vLLM's paged attention kernel); scales
 * [NB][H_kv][16] for each of K and V. */
int64_t oracle_kv_cache_write_fp8(const uint16_t *k_new, const uint16_t *v_new, int dtype,
                                  const int32_t *slot_mapping, int64_t T, uint8_t *key_cache, uint8_t *value_cache,
                                  float *key_scale, float *value_scale, int64_t num_blocks, int H_kv, int d)
{
    int64_t bad = 0;
    for (int64_t t = 0; t < T; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue; /* padding token */
        if (slot >= num_blocks * ORACLE_BLOCK) {
            ++bad;
            continue;
        }
        int64_t block = slot / ORACLE_BLOCK;
        int64_t offset = slot % ORACLE_BLOCK;
        for (int h = 0; h < H_kv; ++h) {
            int64_t row = (block * H_kv + h) * ORACLE_BLOCK + offset;
            int64_t src = (t * H_kv + h) * (int64_t)d;
            uint8_t *vt = value_cache + (block * H_kv + h) * ORACLE_BLOCK * (int64_t)d + offset;
            key_scale[row] = quant_row(k_new + src, dtype, d, key_cache + row * d, 1);
            value_scale[row] = quant_row(v_new + src, dtype, d, vt, ORACLE_BLOCK);
        }
    }
    return bad;
}

/* Attention of one row over the FP8 cache: K_j = e4m3(code) * scale of its row, likewise V (whose
 * codes sit transposed in their block). */
static int attention_row_fp8(double *out_row, const uint16_t *q, int dtype, const uint8_t *key_cache,
                             const uint8_t *value_cache, const float *key_scale, const float *value_scale,
                             const int32_t *block_tables, int max_blocks, int b, int i, int q_b, int ctx_b,
                             int64_t t, int h, int H_q, int H_kv, int d, double scale, double *s)
{
    int G = H_q / H_kv;
    int g = h / G;
    int last = ctx_b - q_b + i; /* causal: keys 0 .. last */
    if (last < 0)
        return -1;
    const uint16_t *qrow = q + (t * H_q + h) * (int64_t)d;
    for (int j = 0; j <= last; ++j) {
        int64_t block = block_tables[(int64_t)b * max_blocks + j / ORACLE_BLOCK];
        int64_t row = (block * H_kv + g) * ORACLE_BLOCK + j % ORACLE_BLOCK;
        double ks = key_scale[row], acc = 0.0;
        for (int k = 0; k < d; ++k)
            acc += widen(qrow[k], dtype) * (oracle_e4m3_to_f64(key_cache[row * d + k]) * ks);
        s[j] = scale * acc;
    }
    double m = -INFINITY;
    for (int j = 0; j <= last; ++j)
        if (s[j] > m)
            m = s[j];
    double z = 0.0;
    for (int j = 0; j <= last; ++j) {
        s[j] = exp(s[j] - m);
        z += s[j];
    }
    for (int k = 0; k < d; ++k)
        out_row[k] = 0.0;
    for (int j = 0; j <= last; ++j) {
        int64_t block = block_tables[(int64_t)b * max_blocks + j / ORACLE_BLOCK];
        int64_t row = (block * H_kv + g) * ORACLE_BLOCK + j % ORACLE_BLOCK;
        double w = s[j] / z, vs = value_scale[row];
        const uint8_t *vt = value_cache + (block * H_kv + g) * ORACLE_BLOCK * (int64_t)d + j % ORACLE_BLOCK;
        for (int k = 0; k < d; ++k)
            out_row[k] += w * (oracle_e4m3_to_f64(vt[k * ORACLE_BLOCK]) * vs);
    }
    return 0;
}

int oracle_paged_attention_fp8(double *out, const uint16_t *q, int dtype, const uint8_t *key_cache,
                               const uint8_t *value_cache, const float *key_scale, const float *value_scale,
                               const int32_t *block_tables, int max_blocks, const int32_t *cu_seqlens_q,
                               const int32_t *context_lens, int B, int H_q, int H_kv, int d, double scale,
                               const int64_t *rows, int64_t n_rows, int n_threads)
{
    if (H_kv <= 0 || H_q % H_kv != 0)
        return -2;
    int max_ctx = 0;
    for (int b = 0; b < B; ++b) {
        int q_b = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
        if (q_b < 0 || context_lens[b] < q_b)
            return -1;
        if (context_lens[b] > max_ctx)
            max_ctx = context_lens[b];
    }
    int64_t T = cu_seqlens_q[B];
    int64_t total = rows ? n_rows : T * H_q;
    int status = 0;
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_ctx > 0 ? max_ctx : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < total; ++r) {
            int64_t row = rows ? rows[r] : r;
            int64_t t = row / H_q;
            int h = (int)(row % H_q);
            int b = 0;
            while (b < B && cu_seqlens_q[b + 1] <= t)
                ++b;
            int i = (int)(t - cu_seqlens_q[b]);
            int q_b = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
            if (attention_row_fp8(out + r * d, q, dtype, key_cache, value_cache, key_scale, value_scale,
                                  block_tables, max_blocks, b, i, q_b, context_lens[b], t, h, H_q, H_kv, d, scale,
                                  s)) {
#pragma omp atomic write
                status = -1;
            }
        }
        free(s);
    }
    return status;
}
