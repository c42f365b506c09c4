/*
 * fp64 CPU oracle for segment linear attention (simple GLA) -- TEST
 * INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use
 * this file.  It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (Flood README, "News" 2025/09 and "Kernels > Seg-linear-attn":
 * linear attention of the simple-GLA form, 16 heads, head_dim 128; written here
 * as the recurrence that defines that form):
 *
 *   Every request r owns one recurrent state per head, S (d x d, key index i,
 *   value index j), kept in a state pool slot.  Its new tokens t = 0 .. n_r-1
 *   (rows q_off[r] + t of the packed q, k, v [T, H, d] and g [T, H]) update it
 *   in order:
 *       S <- exp(g[t,h]) * S + k[t,h,:]^T v[t,h,:]        (outer product)
 *       o[t,h,j] = scale * sum_i q[t,h,i] S[i][j]
 *   The state enters from slot in_slot[r] (all zero when in_slot[r] < 0) and
 *   the final state is returned per request.
 *
 * Inputs q, k, v are bf16 bit patterns widened exactly to double; g is given
 * as double.  Parity: pinned by the CPU tests (the parallel closed form in
 * torch fp64, special cases, planted mistakes).
 *
 * ORACLE_MUTANT planted mistakes (default 0):
 *   8 decay dropped                 9 decay applied after the update
 *   10 output from S q (transposed)  11 output without the scale
 *   12 decay of the previous token
 */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double la_bf16(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Recurrence over every request and head.
 *   q_lens [batch]; q, k, v bf16 [T, H, d]; g [T, H] (double);
 *   state_in [num_in, H, d, d] (double, may be NULL when every in_slot < 0),
 *   in_slot [batch] (-1: zero state);
 *   out [T, H, d]; state_out [batch, H, d, d].
 * Returns 0, or -1 on a bad argument.
 */
int oracle_la(int batch, const int32_t *q_lens, const uint16_t *q, const uint16_t *k,
              const uint16_t *v, const double *g, int heads, int d, double scale,
              const double *state_in, int64_t num_in, const int32_t *in_slot, double *out,
              double *state_out) {
    if (batch < 0 || heads <= 0 || d <= 0) return -1;
    int64_t *q_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(batch + 1));
    q_off[0] = 0;
    for (int r = 0; r < batch; ++r) {
        if (q_lens[r] < 0 || in_slot[r] >= num_in || (in_slot[r] >= 0 && !state_in)) {
            free(q_off);
            return -1;
        }
        q_off[r + 1] = q_off[r] + q_lens[r];
    }
    const size_t dd = (size_t)d * d;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int r = 0; r < batch; ++r)
        for (int h = 0; h < heads; ++h) {
            double *S = state_out + ((size_t)r * heads + h) * dd;
            if (in_slot[r] >= 0)
                memcpy(S, state_in + ((size_t)in_slot[r] * heads + h) * dd, sizeof(double) * dd);
            else
                memset(S, 0, sizeof(double) * dd);
            for (int64_t t = 0; t < q_lens[r]; ++t) {
                const int64_t row = q_off[r] + t;
                const uint16_t *qt = q + ((size_t)row * heads + h) * d;
                const uint16_t *kt = k + ((size_t)row * heads + h) * d;
                const uint16_t *vt = v + ((size_t)row * heads + h) * d;
#if ORACLE_MUTANT == 12
                const double decay = t > 0 ? exp(g[(size_t)(row - 1) * heads + h]) : 1.0;
#else
                const double decay = exp(g[(size_t)row * heads + h]);
#endif
                for (int i = 0; i < d; ++i) {
                    const double ki = la_bf16(kt[i]);
                    for (int j = 0; j < d; ++j) {
                        double s = S[(size_t)i * d + j];
#if ORACLE_MUTANT == 8
                        s = s + ki * la_bf16(vt[j]);
#elif ORACLE_MUTANT == 9
                        s = decay * (s + ki * la_bf16(vt[j]));
#else
                        s = decay * s + ki * la_bf16(vt[j]);
#endif
                        S[(size_t)i * d + j] = s;
                    }
                }
                double *o = out + ((size_t)row * heads + h) * d;
                for (int j = 0; j < d; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < d; ++i)
#if ORACLE_MUTANT == 10
                        acc += la_bf16(qt[i]) * S[(size_t)j * d + i];
#else
                        acc += la_bf16(qt[i]) * S[(size_t)i * d + j];
#endif
#if ORACLE_MUTANT == 11
                    o[j] = acc;
#else
                    o[j] = scale * acc;
#endif
                }
            }
        }
    free(q_off);
    return 0;
}
