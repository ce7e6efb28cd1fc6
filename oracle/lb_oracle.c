/*
 * lb_oracle.c - fp64 CPU oracle for the LittleBit factored linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent reference that the
 * CUDA library is checked against.  Only the test suite, the smoke check and
 * the CPU-baseline leg of the benchmark load it.  It shares no code, header,
 * table or helper with the CUDA path, and it never calls it.
 *
 * What it computes (sesamedisk.com, "Samsung LittleBit 13B Model", section
 * "What the method actually computes", Proposition 1; the same page, section
 * "How low-rank binarization works", for the roles of h, g and l):
 *
 *     Y = ((((X (.) g) V_sign) (.) l) U_sign^T) (.) h
 *
 * for every path p (one path, or two when residual compensation is on; the
 * second path is an independent term with its own factors and scales that is
 * added to the first: sesamedisk.com, "How low-rank binarization works",
 * last paragraph; littlebitllm.com, "Pipeline", step 04).
 *
 * Data:
 *   x   [tokens x n_in]  fp64 (callers widen bf16 exactly)
 *   sv  [n_in  x rank]   int8, every entry +1 or -1   (V_sign)
 *   su  [n_out x rank]   int8, every entry +1 or -1   (U_sign)
 *   g   [n_in]           column scale (callers widen fp16 exactly)
 *   l   [rank]           latent scale
 *   h   [n_out]          row scale
 *   y   [tokens x n_out] fp64 output
 *
 * The steps are taken in the proposition's order, one token at a time:
 *   1. t_i = g_i * x_{m,i}
 *   2. c_k = sum_i sv[i][k] * t_i          (i ascending)
 *   3. z_k = l_k * c_k
 *   4. e_o = sum_k su[o][k] * z_k          (k ascending)
 *   5. y_{m,o} = sum_p h_{p,o} * e_{p,o}   (paths in order)
 * No blocking, fusion or reordering of the sums beyond this.  OpenMP only
 * splits independent outputs (the k of step 2, the o of step 4) across threads,
 * so the result does not depend on the thread count.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t rank;
    const int8_t *su; /* [n_out x rank] */
    const int8_t *sv; /* [n_in x rank]  */
    const double *h;  /* [n_out] */
    const double *g;  /* [n_in]  */
    const double *l;  /* [rank]  */
} oracle_path;

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Returns 0 on success, -1 on a bad argument, -2 when out of memory. */
int oracle_forward(const double *x, int64_t tokens, int64_t n_in, int64_t n_out,
                   const oracle_path *paths, int npaths, double *y)
{
    if (tokens < 0 || n_in <= 0 || n_out <= 0 || npaths < 1 || !paths)
        return -1;
    if (tokens == 0)
        return 0;
    if (!x || !y)
        return -1;
    int64_t max_rank = 0;
    for (int p = 0; p < npaths; ++p) {
        const oracle_path *P = &paths[p];
        if (P->rank <= 0 || !P->su || !P->sv || !P->h || !P->g || !P->l)
            return -1;
        if (P->rank > max_rank)
            max_rank = P->rank;
    }
    double *t = (double *)malloc(sizeof(double) * (size_t)n_in);
    double *c = (double *)malloc(sizeof(double) * (size_t)max_rank);
    double *z = (double *)malloc(sizeof(double) * (size_t)max_rank);
    if (!t || !c || !z) {
        free(t); free(c); free(z);
        return -2;
    }

    for (int64_t m = 0; m < tokens; ++m) {
        const double *xm = x + m * n_in;
        double *ym = y + m * n_out;
        for (int64_t o = 0; o < n_out; ++o)
            ym[o] = 0.0;

        for (int p = 0; p < npaths; ++p) {
            const oracle_path *P = &paths[p];
            const int64_t r = P->rank;

            /* step 1: input scale */
            for (int64_t i = 0; i < n_in; ++i)
                t[i] = P->g[i] * xm[i];

            /* step 2: c_k = sum_i sv[i][k] t_i, i ascending for every k.
             * Each thread owns a block of k and walks i in order. */
#pragma omp parallel
            {
                int nth = 1, tid = 0;
#ifdef _OPENMP
                nth = omp_get_num_threads();
                tid = omp_get_thread_num();
#endif
                int64_t k0 = r * tid / nth, k1 = r * (tid + 1) / nth;
                for (int64_t k = k0; k < k1; ++k)
                    c[k] = 0.0;
                for (int64_t i = 0; i < n_in; ++i) {
                    const int8_t *row = P->sv + i * r;
                    const double ti = t[i];
                    for (int64_t k = k0; k < k1; ++k)
                        c[k] += (double)row[k] * ti;
                }
            }

            /* step 3: latent scale */
            for (int64_t k = 0; k < r; ++k)
                z[k] = P->l[k] * c[k];

            /* steps 4 and 5: e_o = sum_k su[o][k] z_k, then y += h_o e_o */
#pragma omp parallel for schedule(static)
            for (int64_t o = 0; o < n_out; ++o) {
                const int8_t *row = P->su + o * r;
                double e = 0.0;
                for (int64_t k = 0; k < r; ++k)
                    e += (double)row[k] * z[k];
                ym[o] += P->h[o] * e;
            }
        }
    }
    free(t); free(c); free(z);
    return 0;
}

/* The first half of the forward pass alone (steps 1 to 3): the latent
 *   z[m][off_p + k] = l_k * sum_i sv[i][k] * g_i * x[m][i]
 * for every path p, paths side by side (off_p = sum of the ranks before p),
 * z [tokens x sum_p rank_p].  Same steps and order as oracle_forward.
 * Returns 0 on success, -1 on a bad argument, -2 when out of memory. */
int oracle_latent(const double *x, int64_t tokens, int64_t n_in, const oracle_path *paths, int npaths,
                  double *z)
{
    if (tokens < 0 || n_in <= 0 || npaths < 1 || !paths)
        return -1;
    if (tokens == 0)
        return 0;
    if (!x || !z)
        return -1;
    int64_t R = 0;
    for (int p = 0; p < npaths; ++p) {
        if (paths[p].rank <= 0 || !paths[p].sv || !paths[p].g || !paths[p].l)
            return -1;
        R += paths[p].rank;
    }
    double *t = (double *)malloc(sizeof(double) * (size_t)n_in);
    if (!t)
        return -2;
    for (int64_t m = 0; m < tokens; ++m) {
        const double *xm = x + m * n_in;
        int64_t off = 0;
        for (int p = 0; p < npaths; ++p) {
            const oracle_path *P = &paths[p];
            const int64_t r = P->rank;
            double *zm = z + m * R + off;
            for (int64_t i = 0; i < n_in; ++i)      /* step 1 */
                t[i] = P->g[i] * xm[i];
#pragma omp parallel
            {
                int nth = 1, tid = 0;
#ifdef _OPENMP
                nth = omp_get_num_threads();
                tid = omp_get_thread_num();
#endif
                int64_t k0 = r * tid / nth, k1 = r * (tid + 1) / nth;
                for (int64_t k = k0; k < k1; ++k)
                    zm[k] = 0.0;
                for (int64_t i = 0; i < n_in; ++i) { /* step 2, i ascending */
                    const int8_t *row = P->sv + i * r;
                    const double ti = t[i];
                    for (int64_t k = k0; k < k1; ++k)
                        zm[k] += (double)row[k] * ti;
                }
            }
            for (int64_t k = 0; k < r; ++k)         /* step 3 */
                zm[k] = P->l[k] * zm[k];
            off += r;
        }
    }
    free(t);
    return 0;
}

/* The second half alone (steps 4 and 5): from a latent z laid out as
 * oracle_latent writes it,
 *   y[m][o] = sum_p h_{p,o} * sum_k su[o][k] * z[m][off_p + k]
 * (k ascending, paths in order; y [tokens x n_out]).  Same steps and order
 * as oracle_forward, so oracle_expand(oracle_latent(x)) equals
 * oracle_forward(x) exactly. */
int oracle_expand(const double *z, int64_t tokens, int64_t n_out, const oracle_path *paths, int npaths,
                  double *y)
{
    if (tokens < 0 || n_out <= 0 || npaths < 1 || !paths)
        return -1;
    if (tokens == 0)
        return 0;
    if (!z || !y)
        return -1;
    int64_t R = 0;
    for (int p = 0; p < npaths; ++p) {
        if (paths[p].rank <= 0 || !paths[p].su || !paths[p].h)
            return -1;
        R += paths[p].rank;
    }
    for (int64_t m = 0; m < tokens; ++m) {
        double *ym = y + m * n_out;
        for (int64_t o = 0; o < n_out; ++o)
            ym[o] = 0.0;
        int64_t off = 0;
        for (int p = 0; p < npaths; ++p) {
            const oracle_path *P = &paths[p];
            const int64_t r = P->rank;
            const double *zm = z + m * R + off;
#pragma omp parallel for schedule(static)
            for (int64_t o = 0; o < n_out; ++o) {
                const int8_t *row = P->su + o * r;
                double e = 0.0;
                for (int64_t k = 0; k < r; ++k)
                    e += (double)row[k] * zm[k];
                ym[o] += P->h[o] * e;
            }
            off += r;
        }
    }
    return 0;
}
