/*
 * Plain fp64 CPU oracle for the multi-LoRA delta.  TEST INFRASTRUCTURE ONLY:
 * the tests, the smoke check and the benchmark's CPU-baseline leg may call it;
 * the product path never does.  It shares no code with the CUDA library.
 *
 * What it computes is the definition itself, written out as loops:
 *
 *   y_t = W x_t + B_{a(t)} A_{a(t)} x_t        for every token t of the batch
 *
 * ("Multi-LoRA serving: the single translator with a thousand glossaries ...",
 * blog.lo0.es, section "SGMV: the kernel that holds it all up", per-token
 * equation), evaluated in the two phases that section lists:
 *
 *   phase 1, shrink : v_t = A_{a(t)} x_t         (d_in -> r)
 *   phase 2, expand : y_t = y_t + scale * B_{a(t)} v_t   (r -> d_out)
 *
 * with A in R^{r x d_in} and B in R^{d_out x r} as in section "The bare
 * mechanism" (equation y = W x + B(Ax)).  The input y already holds W x.
 * The pages give no LoRA scaling.  Reading taken: the delta of a token is
 * multiplied by `scale` (one real number per call, 1.0 in every workload)
 * times the multiplier of its segment's adapter, seg_scale[s] (LoRA's alpha/r
 * of that adapter; all 1.0 when seg_scale is NULL):
 *
 *   y_t = y_t + (scale * seg_scale[s]) * B_s v_t,   t in segment s
 *
 * Tokens are visited segment by segment (one segment per adapter, "groups
 * the batch's tokens by adapter"), but every token's result depends only on
 * its own x row and its own adapter, so the visiting order does not change
 * any value.  Reductions run in ascending index order in double precision,
 * with no fused multiply-add (build with -ffp-contract=off).
 */
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Returns 0 on success, a negative number on a malformed argument. */
int oracle_lora_delta(int64_t T, int64_t d_in, int64_t d_out,
                      const double* x, int64_t ldx,         /* [T][ldx]          */
                      const double* y_in, int64_t ldy,      /* [T][ldy]  (= W x) */
                      int64_t S,
                      const int64_t* seg_offsets,           /* [S+1] rows of each segment */
                      const int64_t* seg_rank,              /* [S]                         */
                      const double* const* A,               /* [S] -> [r_s][d_in]          */
                      const double* const* B,               /* [S] -> [d_out][r_s]         */
                      const int64_t* token_idx,             /* [rows] row -> token, NULL = identity */
                      double scale,
                      const double* seg_scale,              /* [S] per-segment multiplier, NULL = 1 */
                      double* v, int64_t ldv,               /* [rows][ldv] out             */
                      double* y_out,                        /* [T][ldy] out                */
                      int threads)
{
    if (T < 0 || d_in < 0 || d_out < 0 || S < 0) return -1;
    if (S > 0 && seg_offsets[0] != 0) return -2;
    for (int64_t s = 0; s < S; ++s) {
        if (seg_offsets[s + 1] < seg_offsets[s]) return -3;
        if (seg_rank[s] < 0 || seg_rank[s] > ldv) return -4;
    }
    const int64_t rows = S > 0 ? seg_offsets[S] : 0;

    /* tokens that belong to no segment keep y_in unchanged */
    for (int64_t t = 0; t < T; ++t)
        memcpy(y_out + t * ldy, y_in + t * ldy, (size_t)d_out * sizeof(double));

    /* row -> segment map, so that rows can be processed independently */
    int64_t s_of_row_ok = 1;
    for (int64_t i = 0; i < rows; ++i) {
        int64_t t = token_idx ? token_idx[i] : i;
        if (t < 0 || t >= T) s_of_row_ok = 0;
    }
    if (!s_of_row_ok) return -5;

#ifdef _OPENMP
    if (threads < 1) threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads)
#endif
    for (int64_t i = 0; i < rows; ++i) {
        /* find the segment of row i (linear scan keeps the oracle obvious) */
        int64_t s = 0;
        while (!(seg_offsets[s] <= i && i < seg_offsets[s + 1])) ++s;
        const int64_t r = seg_rank[s];
        const double* As = A[s];
        const double* Bs = B[s];
        const int64_t t = token_idx ? token_idx[i] : i;
        const double* xt = x + t * ldx;
        double* vi = v + i * ldv;

        /* phase 1, shrink: v = A x */
        for (int64_t k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t c = 0; c < d_in; ++c) acc += As[k * d_in + c] * xt[c];
            vi[k] = acc;
        }
        /* phase 2, expand: y = y + (scale * seg_scale[s]) * B v */
        const double sc = seg_scale ? scale * seg_scale[s] : scale;
        for (int64_t j = 0; j < d_out; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < r; ++k) acc += Bs[j * r + k] * vi[k];
            y_out[t * ldy + j] = y_in[t * ldy + j] + sc * acc;
        }
    }
    return 0;
}

/* Number of OpenMP threads a call with `threads` would actually use. */
int oracle_threads(int threads)
{
#ifdef _OPENMP
    int n = 0;
    if (threads < 1) threads = 1;
#pragma omp parallel num_threads(threads)
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
#else
    (void)threads;
    return 1;
#endif
}
