/*
 * fp64 CPU oracle for SegmentAttention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use
 * this file.  It shares no code, header, table or constant with the CUDA path
 * and it is deliberately slow: plain two-pass softmax attention, written from
 * the definitions, with its own walk over the segment lists.
 *
 * What it computes (Flood README, "Introduction" and "Kernels > Seg-attn";
 * the online-softmax state m_i / l_i of the Ascend FlashAttention article,
 * section "bottleneck 2", is the same quantity computed here in one go):
 *
 *   For request r with q_len new queries and k_len = sum of its segment
 *   lengths, logical key j (0 <= j < k_len) lives in pool slot
 *       slot(j) = seg_start[s] + (j - off_s),  off_s = sum of the lengths of
 *   the segments listed before s (list order is logical order).
 *   Query i (0 <= i < q_len) of head h uses kv-head g = h / (Hq / Hkv).
 *   Causal (bottom-right aligned, chunked prefill): it sees keys
 *       j <= (k_len - q_len) + i,   otherwise all keys.
 *   s_j = scale * <q[i,h,:], K[slot(j), g, :]>
 *   m   = max_j s_j,  l = sum_j exp(s_j - m)
 *   out = sum_j exp(s_j - m) V[slot(j), g, :] / l,   lse = m + ln(l)
 *   No visible key: out = 0, lse = -inf.
 *
 * Inputs are bf16 bit patterns widened exactly to double.  Parity: pinned by
 * the CPU tests (brute force on a contiguous copy, closed forms, invariances).
 *
 * ORACLE_MUTANT (compile-time, default 0) plants one deliberate mistake so the
 * tests can show that the pins catch it; the shipped oracle is built with 0.
 *   1 score without the scale        2 top-left causal alignment
 *   3 kv head h % Hkv instead of h / G   4 segments walked in slot order
 *   5 lse without the max            6 output not divided by l
 *   7 V replaced by K in the weighted sum
 */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * FP8 E4M3 code -> value, from the format's definition (1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent 0 is subnormal; S.1111.111 is
 * NaN; there is no infinity; largest finite value 448).
 */
static double e4m3_to_double(uint8_t code) {
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, 1 - 7);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Logical key -> slot list of one request, by walking its segments in list order. */
static int64_t *request_slots(int count, const int32_t *starts, const int32_t *lens, int64_t *k_len_out) {
    int64_t k_len = 0;
    for (int s = 0; s < count; ++s) k_len += lens[s];
    int64_t *slots = (int64_t *)malloc(sizeof(int64_t) * (size_t)(k_len > 0 ? k_len : 1));
    int64_t j = 0;
#if ORACLE_MUTANT == 4
    /* planted mistake: segments taken in slot order instead of list order */
    int *order = (int *)malloc(sizeof(int) * (size_t)(count > 0 ? count : 1));
    for (int s = 0; s < count; ++s) order[s] = s;
    for (int a = 0; a < count; ++a)
        for (int b = a + 1; b < count; ++b)
            if (starts[order[b]] < starts[order[a]]) { int tmp = order[a]; order[a] = order[b]; order[b] = tmp; }
    for (int s = 0; s < count; ++s)
        for (int32_t t = 0; t < lens[order[s]]; ++t) slots[j++] = (int64_t)starts[order[s]] + t;
    free(order);
#else
    for (int s = 0; s < count; ++s)
        for (int32_t t = 0; t < lens[s]; ++t) slots[j++] = (int64_t)starts[s] + t;
#endif
    *k_len_out = k_len;
    return slots;
}

/* One output row: query i of request with the given slot list, head h. */
static void one_row(const uint16_t *qrow, const uint16_t *k_pool, const uint16_t *v_pool,
                    const int64_t *slots, int64_t k_len, int64_t visible, int g, int kv_heads,
                    int d, double scale, double *out, double *lse, double *s_buf) {
    const int64_t n = visible < k_len ? visible : k_len;
    if (n <= 0) {
        for (int t = 0; t < d; ++t) out[t] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        const uint16_t *krow = k_pool + ((size_t)slots[j] * kv_heads + g) * d;
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += bf16_to_double(qrow[t]) * bf16_to_double(krow[t]);
#if ORACLE_MUTANT == 1
        s_buf[j] = acc;
#else
        s_buf[j] = scale * acc;
#endif
        if (s_buf[j] > m) m = s_buf[j];
    }
    double l = 0.0;
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        const double p = exp(s_buf[j] - m);
#if ORACLE_MUTANT == 7
        const uint16_t *vrow = k_pool + ((size_t)slots[j] * kv_heads + g) * d;
#else
        const uint16_t *vrow = v_pool + ((size_t)slots[j] * kv_heads + g) * d;
#endif
        l += p;
        for (int t = 0; t < d; ++t) out[t] += p * bf16_to_double(vrow[t]);
    }
#if ORACLE_MUTANT != 6
    for (int t = 0; t < d; ++t) out[t] /= l;
#endif
#if ORACLE_MUTANT == 5
    *lse = log(l);
#else
    *lse = m + log(l);
#endif
}

/*
 * Rows to compute are given as (packed query token, head) pairs; token indexes
 * the packed query array [sum q_lens, Hq, d].  out: [n_rows, d], lse: [n_rows].
 * Returns 0, or -1 on a bad argument (the oracle checks only what it needs).
 */
int oracle_rows(int batch, const int32_t *q_lens, const int32_t *seg_counts,
                const int32_t *seg_starts, const int32_t *seg_lens,
                const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                int q_heads, int kv_heads, int head_dim, double scale, int causal,
                int64_t n_rows, const int64_t *row_token, const int32_t *row_head,
                double *out, double *lse) {
    if (batch < 0 || q_heads <= 0 || kv_heads <= 0 || q_heads % kv_heads || head_dim <= 0)
        return -1;
    const int group = q_heads / kv_heads;
    /* per-request offsets into the packed queries and the flat segment arrays */
    int64_t *q_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(batch + 1));
    int64_t *s_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(batch + 1));
    q_off[0] = 0;
    s_off[0] = 0;
    for (int r = 0; r < batch; ++r) {
        q_off[r + 1] = q_off[r] + q_lens[r];
        s_off[r + 1] = s_off[r] + seg_counts[r];
    }
    int rc = 0;
    for (int64_t i = 0; i < n_rows; ++i)
        if (row_token[i] < 0 || row_token[i] >= q_off[batch] || row_head[i] < 0 ||
            row_head[i] >= q_heads)
            rc = -1;
    if (rc == 0) {
        /* slot lists per request */
        int64_t **slots = (int64_t **)calloc((size_t)(batch > 0 ? batch : 1), sizeof(int64_t *));
        int64_t *k_lens = (int64_t *)calloc((size_t)(batch > 0 ? batch : 1), sizeof(int64_t));
        int64_t k_max = 1;
        for (int r = 0; r < batch; ++r) {
            slots[r] = request_slots(seg_counts[r], seg_starts + s_off[r], seg_lens + s_off[r],
                                     &k_lens[r]);
            if (k_lens[r] > k_max) k_max = k_lens[r];
        }
#pragma omp parallel
        {
            double *s_buf = (double *)malloc(sizeof(double) * (size_t)k_max);
#pragma omp for schedule(dynamic, 4)
            for (int64_t i = 0; i < n_rows; ++i) {
                const int64_t tok = row_token[i];
                int r = 0; /* request owning this token */
                while (q_off[r + 1] <= tok) ++r;
                const int64_t qi = tok - q_off[r];
#if ORACLE_MUTANT == 2
                const int64_t visible = causal ? qi + 1 : k_lens[r];
#else
                const int64_t visible =
                    causal ? (k_lens[r] - q_lens[r]) + qi + 1 : k_lens[r];
#endif
                const int h = row_head[i];
                one_row(q + ((size_t)tok * q_heads + h) * head_dim, k_pool, v_pool, slots[r],
#if ORACLE_MUTANT == 3
                        k_lens[r], visible, h % kv_heads, kv_heads, head_dim, scale,
#else
                        k_lens[r], visible, h / group, kv_heads, head_dim, scale,
#endif
                        out + (size_t)i * head_dim, lse + i, s_buf);
            }
            free(s_buf);
        }
        for (int r = 0; r < batch; ++r) free(slots[r]);
        free(slots);
        free(k_lens);
    }
    free(q_off);
    free(s_off);
    return rc;
}

/* Every row of every request: out [sum q_lens, Hq, d], lse [sum q_lens, Hq]. */
int oracle_attention(int batch, const int32_t *q_lens, const int32_t *seg_counts,
                     const int32_t *seg_starts, const int32_t *seg_lens, const uint16_t *q,
                     const uint16_t *k_pool, const uint16_t *v_pool, int q_heads, int kv_heads,
                     int head_dim, double scale, int causal, double *out, double *lse) {
    int64_t total = 0;
    for (int r = 0; r < batch; ++r) total += q_lens[r];
    const int64_t n_rows = total * q_heads;
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_rows > 0 ? n_rows : 1));
    int32_t *head = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_rows > 0 ? n_rows : 1));
    for (int64_t i = 0; i < n_rows; ++i) {
        tok[i] = i / q_heads;
        head[i] = (int32_t)(i % q_heads);
    }
    const int rc = oracle_rows(batch, q_lens, seg_counts, seg_starts, seg_lens, q, k_pool, v_pool,
                               q_heads, kv_heads, head_dim, scale, causal, n_rows, tok, head, out,
                               lse);
    free(tok);
    free(head);
    return rc;
}

/*
 * FP8 KV cache variant: pools hold E4M3 codes, K[slot,g,:] = k_scale[g] * code
 * value, V likewise with v_scale[g]; queries stay bf16.  Same attention.
 */
static void one_row_fp8(const uint16_t *qrow, const uint8_t *k_pool, const uint8_t *v_pool,
                        double k_scale, double v_scale, const int64_t *slots, int64_t k_len,
                        int64_t visible, int g, int kv_heads, int d, double scale, double *out,
                        double *lse, double *s_buf) {
    const int64_t n = visible < k_len ? visible : k_len;
    if (n <= 0) {
        for (int t = 0; t < d; ++t) out[t] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        const uint8_t *krow = k_pool + ((size_t)slots[j] * kv_heads + g) * d;
        double acc = 0.0;
        for (int t = 0; t < d; ++t)
            acc += bf16_to_double(qrow[t]) * (k_scale * e4m3_to_double(krow[t]));
        s_buf[j] = scale * acc;
        if (s_buf[j] > m) m = s_buf[j];
    }
    double l = 0.0;
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        const double p = exp(s_buf[j] - m);
        const uint8_t *vrow = v_pool + ((size_t)slots[j] * kv_heads + g) * d;
        l += p;
        for (int t = 0; t < d; ++t) out[t] += p * (v_scale * e4m3_to_double(vrow[t]));
    }
    for (int t = 0; t < d; ++t) out[t] /= l;
    *lse = m + log(l);
}

int oracle_rows_fp8(int batch, const int32_t *q_lens, const int32_t *seg_counts,
                    const int32_t *seg_starts, const int32_t *seg_lens, const uint16_t *q,
                    const uint8_t *k_pool, const uint8_t *v_pool, const double *k_scale,
                    const double *v_scale, int q_heads, int kv_heads, int head_dim, double scale,
                    int causal, int64_t n_rows, const int64_t *row_token, const int32_t *row_head,
                    double *out, double *lse) {
    if (batch < 0 || q_heads <= 0 || kv_heads <= 0 || q_heads % kv_heads || head_dim <= 0)
        return -1;
    const int group = q_heads / kv_heads;
    int64_t *q_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(batch + 1));
    int64_t *s_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(batch + 1));
    q_off[0] = 0;
    s_off[0] = 0;
    for (int r = 0; r < batch; ++r) {
        q_off[r + 1] = q_off[r] + q_lens[r];
        s_off[r + 1] = s_off[r] + seg_counts[r];
    }
    int rc = 0;
    for (int64_t i = 0; i < n_rows; ++i)
        if (row_token[i] < 0 || row_token[i] >= q_off[batch] || row_head[i] < 0 ||
            row_head[i] >= q_heads)
            rc = -1;
    if (rc == 0) {
        int64_t **slots = (int64_t **)calloc((size_t)(batch > 0 ? batch : 1), sizeof(int64_t *));
        int64_t *k_lens = (int64_t *)calloc((size_t)(batch > 0 ? batch : 1), sizeof(int64_t));
        int64_t k_max = 1;
        for (int r = 0; r < batch; ++r) {
            slots[r] = request_slots(seg_counts[r], seg_starts + s_off[r], seg_lens + s_off[r],
                                     &k_lens[r]);
            if (k_lens[r] > k_max) k_max = k_lens[r];
        }
#pragma omp parallel
        {
            double *s_buf = (double *)malloc(sizeof(double) * (size_t)k_max);
#pragma omp for schedule(dynamic, 4)
            for (int64_t i = 0; i < n_rows; ++i) {
                const int64_t tok = row_token[i];
                int r = 0;
                while (q_off[r + 1] <= tok) ++r;
                const int64_t qi = tok - q_off[r];
                const int64_t visible = causal ? (k_lens[r] - q_lens[r]) + qi + 1 : k_lens[r];
                const int h = row_head[i], g = h / group;
                one_row_fp8(q + ((size_t)tok * q_heads + h) * head_dim, k_pool, v_pool,
                            k_scale[g], v_scale[g], slots[r], k_lens[r], visible, g, kv_heads,
                            head_dim, scale, out + (size_t)i * head_dim, lse + i, s_buf);
            }
            free(s_buf);
        }
        for (int r = 0; r < batch; ++r) free(slots[r]);
        free(slots);
        free(k_lens);
    }
    free(q_off);
    free(s_off);
    return rc;
}

/* E4M3 decode exposed for the format pins. */
void oracle_e4m3_decode(const uint8_t *codes, int64_t n, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_double(codes[i]);
}
