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
 * No blocking, fusion or reordering of the sums beyond this.  oracle_backward
 * (at the end) gives the gradients of the same steps by the chain rule.  OpenMP only
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

/* The backward pass of the layer: given the gradient dy = dL/dy of a loss L
 * with respect to the output, the gradients with respect to the input x and
 * to every path's scale vectors h, g and l.  The pages give the forward pass
 * (Proposition 1, steps 1-5 above) and say that training runs through it with
 * a smooth surrogate for the gradient of sign() (littlebitllm.com, "Pipeline";
 * trove.briskstack.com, "How it works"); the gradients here are those of the
 * five steps, by the chain rule, taken in reverse order for each token:
 *   5'. y_{m,o} = sum_p h_{p,o} e_{p,o}:  dh_{p,o} += dy_{m,o} e_{p,o};
 *       de_o = h_{p,o} dy_{m,o}
 *   4'. e_o = sum_k su[o][k] z_k:         dz_k = sum_o su[o][k] de_o  (o ascending)
 *   3'. z_k = l_k c_k:                    dl_{p,k} += dz_k c_k;  dc_k = l_k dz_k
 *   2'. c_k = sum_i sv[i][k] t_i:         dt_i = sum_k sv[i][k] dc_k  (k ascending)
 *   1'. t_i = g_i x_{m,i}:                dg_{p,i} += dt_i x_{m,i};  dx_{m,i} += g_{p,i} dt_i
 * The forward quantities (t, c, z, e) are recomputed per token by the steps of
 * oracle_forward.  Sums over tokens run in token order, over paths in path
 * order.  The gradient with respect to sign(U) and sign(V) themselves, and
 * through sign() to the real-valued factors, is not computed (the pages give
 * no formula for the surrogate).
 * Layout: dx [tokens x n_in]; dh [npaths x n_out], dg [npaths x n_in] and
 * dl [sum of ranks], each path's block after the previous one's.
 * Returns 0 on success, -1 on a bad argument, -2 when out of memory. */
int oracle_backward(const double *x, const double *dy, int64_t tokens, int64_t n_in, int64_t n_out,
                    const oracle_path *paths, int npaths, double *dx, double *dh, double *dg, double *dl)
{
    if (tokens < 0 || n_in <= 0 || n_out <= 0 || npaths < 1 || !paths)
        return -1;
    if (!dh || !dg || !dl)
        return -1;
    int64_t max_rank = 0, R = 0;
    for (int p = 0; p < npaths; ++p) {
        const oracle_path *P = &paths[p];
        if (P->rank <= 0 || !P->su || !P->sv || !P->h || !P->g || !P->l)
            return -1;
        if (P->rank > max_rank)
            max_rank = P->rank;
        R += P->rank;
    }
    for (int64_t j = 0; j < npaths * n_out; ++j)
        dh[j] = 0.0;
    for (int64_t j = 0; j < npaths * n_in; ++j)
        dg[j] = 0.0;
    for (int64_t j = 0; j < R; ++j)
        dl[j] = 0.0;
    if (tokens == 0)
        return 0;
    if (!x || !dy || !dx)
        return -1;
    double *t = (double *)malloc(sizeof(double) * (size_t)n_in);
    double *dt = (double *)malloc(sizeof(double) * (size_t)n_in);
    double *c = (double *)malloc(sizeof(double) * (size_t)max_rank);
    double *z = (double *)malloc(sizeof(double) * (size_t)max_rank);
    double *dz = (double *)malloc(sizeof(double) * (size_t)max_rank);
    double *dc = (double *)malloc(sizeof(double) * (size_t)max_rank);
    double *e = (double *)malloc(sizeof(double) * (size_t)n_out);
    double *de = (double *)malloc(sizeof(double) * (size_t)n_out);
    if (!t || !dt || !c || !z || !dz || !dc || !e || !de) {
        free(t); free(dt); free(c); free(z); free(dz); free(dc); free(e); free(de);
        return -2;
    }
    for (int64_t m = 0; m < tokens; ++m) {
        const double *xm = x + m * n_in;
        const double *dym = dy + m * n_out;
        double *dxm = dx + m * n_in;
        for (int64_t i = 0; i < n_in; ++i)
            dxm[i] = 0.0;
        int64_t off = 0;
        for (int p = 0; p < npaths; ++p) {
            const oracle_path *P = &paths[p];
            const int64_t r = P->rank;
            double *dhp = dh + p * n_out, *dgp = dg + p * n_in, *dlp = dl + off;

            /* forward steps 1-4 of this token and path */
            for (int64_t i = 0; i < n_in; ++i)
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
                    c[k] = 0.0;
                for (int64_t i = 0; i < n_in; ++i) {
                    const int8_t *row = P->sv + i * r;
                    const double ti = t[i];
                    for (int64_t k = k0; k < k1; ++k)
                        c[k] += (double)row[k] * ti;
                }
            }
            for (int64_t k = 0; k < r; ++k)
                z[k] = P->l[k] * c[k];
#pragma omp parallel for schedule(static)
            for (int64_t o = 0; o < n_out; ++o) {
                const int8_t *row = P->su + o * r;
                double s = 0.0;
                for (int64_t k = 0; k < r; ++k)
                    s += (double)row[k] * z[k];
                e[o] = s;
            }

            /* step 5': the row scale */
            for (int64_t o = 0; o < n_out; ++o) {
                dhp[o] += dym[o] * e[o];
                de[o] = P->h[o] * dym[o];
            }
            /* step 4': dz_k = sum_o su[o][k] de_o, o ascending for every k */
#pragma omp parallel
            {
                int nth = 1, tid = 0;
#ifdef _OPENMP
                nth = omp_get_num_threads();
                tid = omp_get_thread_num();
#endif
                int64_t k0 = r * tid / nth, k1 = r * (tid + 1) / nth;
                for (int64_t k = k0; k < k1; ++k)
                    dz[k] = 0.0;
                for (int64_t o = 0; o < n_out; ++o) {
                    const int8_t *row = P->su + o * r;
                    const double d = de[o];
                    for (int64_t k = k0; k < k1; ++k)
                        dz[k] += (double)row[k] * d;
                }
            }
            /* step 3': the latent scale */
            for (int64_t k = 0; k < r; ++k) {
                dlp[k] += dz[k] * c[k];
                dc[k] = P->l[k] * dz[k];
            }
            /* step 2': dt_i = sum_k sv[i][k] dc_k, k ascending */
#pragma omp parallel for schedule(static)
            for (int64_t i = 0; i < n_in; ++i) {
                const int8_t *row = P->sv + i * r;
                double s = 0.0;
                for (int64_t k = 0; k < r; ++k)
                    s += (double)row[k] * dc[k];
                dt[i] = s;
            }
            /* step 1': the column scale and the input */
            for (int64_t i = 0; i < n_in; ++i) {
                dgp[i] += dt[i] * xm[i];
                dxm[i] += P->g[i] * dt[i];
            }
            off += r;
        }
    }
    free(t); free(dt); free(c); free(z); free(dz); free(dc); free(e); free(de);
    return 0;
}
