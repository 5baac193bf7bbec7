/*
 * recall_oracle.c -- CPU oracle for one attention step under a fixed-recall
 * ("cumulative energy") skip predicate.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Source: "Training-free sparse attention based on cumulative energy
 * filtering" (abstract).  The page casts token filtering as keeping accuracy
 * while maximising sparsity, says that holding a fixed recall rate is enough
 * for accuracy while a fixed threshold wastes work, proposes a dynamic
 * threshold for that, and integrates it into the FlashAttention pass with no
 * separate masking stage.  It gives no formula.  The reading written out here:
 *
 *   recall of a query row = (softmax mass of the keys it keeps) /
 *                           (softmax mass of all keys it was offered),
 *   and a row must keep recall >= p.
 *
 *   Inside the FlashAttention pass (key tiles in ascending order, running row
 *   max m, running kept mass l = sum of exp(s - m) over kept keys), each row
 *   also carries z = an upper bound on the mass of the keys it skipped, in the
 *   same frame as l.  A key tile j with w valid keys and row maxima m_loc can
 *   carry at most w * exp(m_loc - m) of mass for row r.  The tile is skipped for
 *   the query tile when every valid row can afford it:
 *
 *       z_r + w * exp(m_loc_r - m_r)  <=  c * l_r,      c = (1 - p) / p,
 *
 *   i.e. when the tile's max-logit gap lies below the row's dynamic threshold
 *   ln((c * l_r - z_r) / w).  A skipped tile adds its bound to z; a kept tile
 *   updates (m, l, acc) as in FlashAttention and rescales z with l.  Since z only
 *   over-counts and l never shrinks, every row ends with kept / (kept + skipped)
 *   >= l / (l + z) >= p.  The first tile a row processes is always kept
 *   (m = -inf, so nothing can be afforded yet); p = 1 skips nothing.
 *
 *   The step is otherwise the LiteAttention step of lite_oracle.c: tiles dead in
 *   mask_in are not offered at all (they count neither as kept nor as skipped),
 *   a skipped tile gets no softmax and no P V, and mask_out = mask_in without
 *   the skipped tiles.
 *
 * Everything is plain fp64; inputs are bf16 bit patterns converted exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double rc_bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int rc_ceil_div(int a, int b) { return (a + b - 1) / b; }

/*
 * lo_step_recall: run the recall-predicate oracle on n_items work items.
 *
 *   p          : recall target, 0 < p <= 1.
 *   q, k, v, items, mask_in, force, o, mask_out, m_fin, l_fin : as lo_step.
 *   E          : optional out [n_items][Tk], the decision statistic of each tested
 *                tile: max over valid rows of (z_r + w exp(m_loc_r - m_r)) / (c l_r) - 1
 *                (+inf while a row has nothing kept or when p = 1); the tile is
 *                skipped iff E <= 0.  NaN for tiles not tested.
 *   z_fin      : optional out [n_items][Br], each row's final skipped-mass bound in
 *                the frame of m_fin (so recall >= l_fin / (l_fin + z_fin)).
 *
 * Returns 0, or -1 for an invalid argument.
 */
int lo_step_recall(int B, int H, int N, int d, int Br, int Bc, double p,
                   const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   const int64_t *items, int64_t n_items,
                   const uint32_t *mask_in, const int8_t *force,
                   double *o, uint32_t *mask_out, double *E,
                   double *m_fin, double *l_fin, double *z_fin, int n_threads)
{
    if (B < 1 || H < 1 || N < 1 || d < 1 || Br < 1 || Bc < 1) return -1;
    if (!q || !k || !v || !items || !mask_in || !o || !mask_out) return -1;
    if (!(p > 0.0 && p <= 1.0)) return -1;
    const int Tq = rc_ceil_div(N, Br);
    const int Tk = rc_ceil_div(N, Bc);
    const int W = rc_ceil_div(Tk, 32);
    const double scale = 1.0 / sqrt((double)d);
    const double c = (1.0 - p) / p;       /* affordable skipped mass per unit of kept mass */
    for (int64_t it = 0; it < n_items; ++it)
        if (items[it] < 0 || items[it] >= (int64_t)B * H * Tq) return -1;

#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif

#pragma omp parallel
    {
        double *qt   = (double *)malloc(sizeof(double) * (size_t)Br * d);
        double *kt   = (double *)malloc(sizeof(double) * (size_t)Bc * d);
        double *vt   = (double *)malloc(sizeof(double) * (size_t)Bc * d);
        double *s    = (double *)malloc(sizeof(double) * (size_t)Br * Bc);
        double *mrun = (double *)malloc(sizeof(double) * (size_t)Br);
        double *mloc = (double *)malloc(sizeof(double) * (size_t)Br);
        double *l    = (double *)malloc(sizeof(double) * (size_t)Br);
        double *z    = (double *)malloc(sizeof(double) * (size_t)Br);
        double *acc  = (double *)malloc(sizeof(double) * (size_t)Br * d);

#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_items; ++it) {
            const int64_t item = items[it];
            const int64_t bh = item / Tq;
            const int i = (int)(item % Tq);
            const size_t head_off = (size_t)bh * (size_t)N * (size_t)d;
            const int r0 = i * Br;
            const int nr = (N - r0 < Br) ? (N - r0) : Br;   /* valid query rows */
            const uint32_t *min_row = mask_in + (size_t)it * W;
            uint32_t *mout_row = mask_out + (size_t)it * W;
            double *o_item = o + (size_t)it * Br * d;
            double *E_item = E ? E + (size_t)it * Tk : NULL;
            const int8_t *f_item = force ? force + (size_t)it * Tk : NULL;

            for (int r = 0; r < nr; ++r) {
                for (int e = 0; e < d; ++e)
                    qt[r * d + e] = rc_bf16_to_double(q[head_off + (size_t)(r0 + r) * d + e]);
                mrun[r] = -INFINITY;
                l[r] = 0.0;
                z[r] = 0.0;
                for (int e = 0; e < d; ++e) acc[r * d + e] = 0.0;
            }
            for (int w = 0; w < W; ++w) mout_row[w] = 0u;
            if (E_item) for (int j = 0; j < Tk; ++j) E_item[j] = NAN;

            for (int j = 0; j < Tk; ++j) {
                if (!((min_row[j >> 5] >> (j & 31)) & 1u)) continue;   /* not offered in this step */
                const int c0 = j * Bc;
                const int nc = (N - c0 < Bc) ? (N - c0) : Bc;          /* valid keys of the tile */
                for (int cc = 0; cc < nc; ++cc)
                    for (int e = 0; e < d; ++e) {
                        kt[cc * d + e] = rc_bf16_to_double(k[head_off + (size_t)(c0 + cc) * d + e]);
                        vt[cc * d + e] = rc_bf16_to_double(v[head_off + (size_t)(c0 + cc) * d + e]);
                    }
                for (int r = 0; r < nr; ++r) {
                    double mx = -INFINITY;
                    for (int cc = 0; cc < nc; ++cc) {
                        double dot = 0.0;
                        for (int e = 0; e < d; ++e) dot += qt[r * d + e] * kt[cc * d + e];
                        s[r * Bc + cc] = scale * dot;
                        if (s[r * Bc + cc] > mx) mx = s[r * Bc + cc];
                    }
                    mloc[r] = mx;
                }
                /* can every valid row afford to skip this tile? */
                double Ej = -INFINITY;
                for (int r = 0; r < nr; ++r) {
                    double g;
                    if (mrun[r] == -INFINITY || c == 0.0)
                        g = INFINITY;
                    else
                        g = (z[r] + (double)nc * exp(mloc[r] - mrun[r])) / (c * l[r]) - 1.0;
                    if (g > Ej) Ej = g;
                }
                if (E_item) E_item[j] = Ej;
                int skip = (Ej <= 0.0);
                if (f_item && f_item[j] >= 0) skip = (f_item[j] == 0);
                if (skip) {
                    /* the tile's mass bound joins the skipped mass of every valid row */
                    for (int r = 0; r < nr; ++r)
                        if (mrun[r] != -INFINITY) z[r] += (double)nc * exp(mloc[r] - mrun[r]);
                    continue;
                }
                mout_row[j >> 5] |= (1u << (j & 31));
                for (int r = 0; r < nr; ++r) {
                    const double mnew = (mloc[r] > mrun[r]) ? mloc[r] : mrun[r];
                    const double alpha = (mrun[r] == -INFINITY) ? 0.0 : exp(mrun[r] - mnew);
                    double lsum = 0.0;
                    for (int e = 0; e < d; ++e) acc[r * d + e] *= alpha;
                    for (int cc = 0; cc < nc; ++cc) {
                        const double pw = exp(s[r * Bc + cc] - mnew);
                        lsum += pw;
                        for (int e = 0; e < d; ++e) acc[r * d + e] += pw * vt[cc * d + e];
                    }
                    l[r] = l[r] * alpha + lsum;
                    z[r] = z[r] * alpha;
                    mrun[r] = mnew;
                }
            }
            for (int r = 0; r < Br; ++r)
                for (int e = 0; e < d; ++e)
                    o_item[r * d + e] = (r < nr && l[r] > 0.0) ? acc[r * d + e] / l[r] : 0.0;
            if (m_fin)
                for (int r = 0; r < Br; ++r) m_fin[it * Br + r] = (r < nr) ? mrun[r] : NAN;
            if (l_fin)
                for (int r = 0; r < Br; ++r) l_fin[it * Br + r] = (r < nr) ? l[r] : NAN;
            if (z_fin)
                for (int r = 0; r < Br; ++r) z_fin[it * Br + r] = (r < nr) ? z[r] : NAN;
        }
        free(qt); free(kt); free(vt); free(s);
        free(mrun); free(mloc); free(l); free(z); free(acc);
    }
    return 0;
}
