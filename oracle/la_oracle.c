/*
 * la_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, float64 CPU statement of causal linear attention over a
 * recurrent state, written as the literal token-by-token recurrence of the
 * slides "Chunking, causality, and parallel prefill" (sections "Naive
 * recurrence" and "Incoming and outgoing state"):
 *
 *     S_t = S_{t-1} + k_t v_t^T          (S[i][j] += k_t[i] * v_t[j])
 *     o_t = q_t^T S_t                    (o_t[j]  = sum_i q_t[i] * S_t[i][j])
 *
 * The state S is d_k x d_v, rows indexed by the key dimension, stored
 * row-major (the worked example prints S_4 = K_1^T V_1 = [[3,4],[5,5]]:
 * row 0 collects v of the tokens whose key is e_0).  The output of token t
 * reads the state AFTER its own update, so the diagonal of the causal
 * triangle is included (o_1 = v_1 in the worked example).
 *
 * Decode of one token is the same loop body run once (the slide "Prefill and
 * decode": with one token the triangle is 1x1 and only the state read plus
 * the local term remains).
 *
 * No blocking, no reordering: one token at a time, one unit at a time.
 * Units (one sequence of one head) are independent, so they are spread over
 * OpenMP threads; the arithmetic inside a unit is strictly sequential.
 *
 * Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load this file's library.  The CUDA library shares no code,
 * header or constant with it.
 */
#include <stdint.h>

/* Per-unit recurrence.  Unit u owns rows row_start[u] .. row_start[u] +
 * row_len[u] - 1 of q, k (row width dk) and of v, o (row width dv).
 * state: [n_units][dk][dv] float64, holds S_0 on entry and S_T on return.
 * A unit with row_len 0 leaves its state untouched.  Returns 0, or -1 on a
 * bad argument. */
int la_oracle_recurrent(const double* q, const double* k, const double* v,
                        double* o, double* state, int64_t n_units,
                        const int64_t* row_start, const int64_t* row_len,
                        int dk, int dv)
{
    if (n_units < 0 || dk <= 0 || dv <= 0) return -1;
    if (n_units == 0) return 0;
    if (!state || !row_start || !row_len) return -1;

    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < n_units; ++u) {
        double* S = state + u * (int64_t)dk * dv;
        for (int64_t t = 0; t < row_len[u]; ++t) {
            const int64_t r = row_start[u] + t;
            const double* qt = q + r * dk;
            const double* kt = k + r * dk;
            const double* vt = v + r * dv;
            double* ot = o + r * dv;
            /* S_t = S_{t-1} + k_t v_t^T */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[i * dv + j] += kt[i] * vt[j];
            /* o_t = q_t^T S_t */
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    ot[j] += qt[i] * S[i * dv + j];
        }
    }
    return 0;
}

/* Number of OpenMP threads a parallel region of this library would use
 * (reported beside the CPU-baseline timing). */
int la_oracle_max_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
