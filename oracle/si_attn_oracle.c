/*
 * si_attn_oracle.c -- plain fp64 CPU oracle for the sparse attention stage
 * of Compressed Sparse Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library or with the indexer oracle.
 *
 * What it computes (StreamIndex: Memory-Bounded Compressed Sparse Attention
 * via Streaming Top-k, arXiv 2605.02568v1, Abstract): in CSA, after the
 * lightning indexer has chosen the top-k compressed keys of each query, the
 * sparse attention reads only those keys.  The Abstract gives no formula for
 * that attention; this library takes the plainest reading, softmax attention
 * of every query head over the selected compressed key/value entries, which
 * all heads share:
 *
 *     s_j      = scale * sum_d q[b,t,h,d] * K[b,j,d]          for j in J_t
 *     p_j      = exp(s_j) / sum_{i in J_t} exp(s_i)
 *     out[b,t,h,:] = sum_{j in J_t} p_j * V[b,j,:]
 *     lse[b,t,h]   = log sum_{j in J_t} exp(s_j)
 *
 * with J_t the entries idx[b,t,0..k) that are >= 0 (negative entries are
 * padding and are skipped).  A row with no entry gives out = 0 and
 * lse = -infinity.  Every value is computed in fp64 from the exact bf16
 * inputs, with the usual max subtraction (which does not change the result).
 *
 * It also returns, for the acceptance tolerance, absw[b,t,h,:] =
 * sum_j p_j * |V[b,j,:]|, the same weights applied to |V|.
 *
 * Parity pins (tests/test_attn_oracle.py): hand-computed cases, uniform
 * scores (a plain mean), the dense causal special case (a library routine,
 * torch's scaled_dot_product_attention in fp64), a dominant key, permutation
 * and padding invariance.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper half of an IEEE fp32; widening to fp64 is exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Sparse attention of R query rows.
 *
 *   q_rows   bf16 bits [R, H, D]    the rows' query heads
 *   idx_rows int32     [R, k]       selected key indices, < 0 = padding
 *   row_b    int64     [R]          batch of each row
 *   kcache   bf16 bits [B, T, D]    compressed keys
 *   vcache   bf16 bits [B, T, DV]   compressed values
 *   out      fp64      [R, H, DV]
 *   lse      fp64      [R, H]
 *   absw     fp64      [R, H, DV] or NULL
 *
 * Returns 0, or -1 on a bad argument (an index >= T, a bad batch).
 */
int oracle_sparse_attention(const uint16_t* q_rows, const int32_t* idx_rows, const int64_t* row_b, int64_t R,
                            const uint16_t* kcache, const uint16_t* vcache, int64_t B, int64_t T, int H, int D,
                            int DV, int64_t k, double scale, double* out, double* lse, double* absw) {
    if (R < 0 || B < 1 || T < 0 || H < 1 || D < 1 || DV < 1 || k < 1) return -1;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const int64_t b = row_b[r];
        const int32_t* sel = idx_rows + r * k;
        double* s = (double*)malloc((size_t)k * sizeof(double));
        int ok = s != NULL && b >= 0 && b < B;
        for (int64_t j = 0; ok && j < k; ++j)
            if (sel[j] >= T) ok = 0;
        if (!ok) {
#pragma omp atomic write
            failed = 1;
            free(s);
            continue;
        }
        for (int h = 0; h < H; ++h) {
            const uint16_t* qh = q_rows + (r * H + h) * D;
            double* oh = out + (r * H + h) * DV;
            double* ah = absw ? absw + (r * H + h) * DV : NULL;
            for (int e = 0; e < DV; ++e) {
                oh[e] = 0.0;
                if (ah) ah[e] = 0.0;
            }
            /* scores of the selected keys */
            double smax = -INFINITY;
            int64_t n = 0;
            for (int64_t j = 0; j < k; ++j) {
                if (sel[j] < 0) continue;
                const uint16_t* kj = kcache + (b * T + sel[j]) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(kj[d]);
                s[j] = scale * dot;
                if (s[j] > smax) smax = s[j];
                ++n;
            }
            if (n == 0) {
                lse[r * H + h] = -INFINITY;
                continue;
            }
            double z = 0.0;
            for (int64_t j = 0; j < k; ++j)
                if (sel[j] >= 0) z += exp(s[j] - smax);
            for (int64_t j = 0; j < k; ++j) {
                if (sel[j] < 0) continue;
                const double p = exp(s[j] - smax) / z;
                const uint16_t* vj = vcache + (b * T + sel[j]) * DV;
                for (int e = 0; e < DV; ++e) {
                    const double v = bf16_to_double(vj[e]);
                    oh[e] += p * v;
                    if (ah) ah[e] += p * fabs(v);
                }
            }
            lse[r * H + h] = smax + log(z);
        }
        free(s);
    }
    return failed ? -1 : 0;
}
