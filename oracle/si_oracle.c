/*
 * si_oracle.c -- plain fp64 CPU oracle for the CSA indexer step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes (StreamIndex: Memory-Bounded Compressed Sparse Attention
 * via Streaming Top-k, arXiv 2605.02568v1, Abstract): the lightning indexer
 * scores every compressed key for each query, and the k best keys per query
 * are kept.  The Abstract gives no formula for the score (only that it is
 * learned and taken over the compressed keys); this library fixes it as
 *
 *     score[b,t,s] = sum_h  w[b,t,h] * max(0, sum_d q[b,t,h,d] * kc[b,s,d])
 *
 * with key s visible to query t iff (s+1)*m <= t+1 (and s < T), the top-k
 * ordered by score descending and then by key index ascending (so equal
 * scores go to the lower index), and rows with fewer than k visible keys
 * padded with index -1 and score -infinity.
 *
 * The method's top-k is exact (it only avoids materialising the score
 * tensor, Abstract), so this oracle is the plain definition written out:
 * score every visible key of a row in fp64 from the exact bf16 input values,
 * sort all (score, index) pairs by the total order above, keep the first k.
 * No blocking, fusion or streaming.  Rows run in parallel with OpenMP.
 *
 * Parity pins (tests/test_oracle_pins.py): hand-computed cases, the H=1
 * non-negative special case (a causal top-k of a matrix product computed with
 * numpy's matmul and argsort), the closed form of the visible count, tie and
 * planted-key structure, invariants and scaling laws.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper half of an IEEE fp32; widening to fp64 is exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    double score;
    int64_t idx;
} scored_key;

/* Total order of the selection: higher score first, then lower index. */
static int by_score_desc_idx_asc(const void* pa, const void* pb) {
    const scored_key* a = (const scored_key*)pa;
    const scored_key* b = (const scored_key*)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    if (a->idx < b->idx) return -1;
    if (a->idx > b->idx) return 1;
    return 0;
}

/* Visibility of compressed key s to query t with compression ratio m. */
static int key_visible(int64_t s, int64_t t, int64_t T, int64_t m) {
    return s < T && (s + 1) * m <= t + 1;
}

/* Indexer score of query row (q_row [H,D], w_row [H]) against key kc_row [D]. */
static double indexer_score(const uint16_t* q_row, const float* w_row,
                            const uint16_t* kc_row, int H, int D) {
    double score = 0.0;
    for (int h = 0; h < H; ++h) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_bits_to_double(q_row[(int64_t)h * D + d]) *
                   bf16_bits_to_double(kc_row[d]);
        double relu = dot > 0.0 ? dot : 0.0;
        score += (double)w_row[h] * relu;
    }
    return score;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Top-k of R query rows.
 *
 *   q_rows   bf16 bits [R, H, D]   the q vectors of the checked rows
 *   w_rows   fp32      [R, H]      their head weights
 *   row_b    int64     [R]         batch of each row
 *   row_t    int64     [R]         query position of each row (0 <= t < S)
 *   kc       bf16 bits [B, T, D]   compressed keys of every batch
 *   out_idx   int32    [R, k]      selected key indices, -1 = padding
 *   out_score fp64     [R, k]      their scores, -inf = padding
 *   out_meta  fp64     [R, 4]      per row: max |score| over visible keys
 *                                  (0 if none), score at rank k, score at
 *                                  rank k+1 (NaN when that rank does not
 *                                  exist), number of visible keys
 *   all_scores fp64    [R, T] or NULL: every visible key's score, NaN for
 *                                  keys the row cannot see
 *
 * Returns 0, or -1 on a bad argument or a failed allocation.
 */
int oracle_topk_rows(const uint16_t* q_rows, const float* w_rows,
                     const int64_t* row_b, const int64_t* row_t, int64_t R,
                     const uint16_t* kc, int64_t B, int64_t T, int H, int D,
                     int64_t m, int64_t k, int32_t* out_idx, double* out_score,
                     double* out_meta, double* all_scores) {
    if (R < 0 || B < 1 || T < 0 || H < 1 || D < 1 || m < 1 || k < 1) return -1;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const int64_t b = row_b[r], t = row_t[r];
        const uint16_t* q_row = q_rows + r * H * D;
        const float* w_row = w_rows + r * H;
        const uint16_t* kc_b = kc + b * T * D;
        scored_key* keys = (scored_key*)malloc((size_t)(T > 0 ? T : 1) * sizeof(scored_key));
        if (!keys || b < 0 || b >= B || t < 0) {
#pragma omp atomic write
            failed = 1;
            free(keys);
            continue;
        }
        int64_t nvis = 0;
        double rowmax = 0.0;
        for (int64_t s = 0; s < T; ++s) {
            double sc = NAN;
            if (key_visible(s, t, T, m)) {
                sc = indexer_score(q_row, w_row, kc_b + s * D, H, D);
                keys[nvis].score = sc;
                keys[nvis].idx = s;
                ++nvis;
                if (fabs(sc) > rowmax) rowmax = fabs(sc);
            }
            if (all_scores) all_scores[r * T + s] = sc;
        }
        qsort(keys, (size_t)nvis, sizeof(scored_key), by_score_desc_idx_asc);
        for (int64_t j = 0; j < k; ++j) {
            if (j < nvis) {
                out_idx[r * k + j] = (int32_t)keys[j].idx;
                out_score[r * k + j] = keys[j].score;
            } else {
                out_idx[r * k + j] = -1;
                out_score[r * k + j] = -INFINITY;
            }
        }
        out_meta[r * 4 + 0] = rowmax;
        out_meta[r * 4 + 1] = (k - 1 < nvis) ? keys[k - 1].score : NAN;
        out_meta[r * 4 + 2] = (k < nvis) ? keys[k].score : NAN;
        out_meta[r * 4 + 3] = (double)nvis;
        free(keys);
    }
    return failed ? -1 : 0;
}
