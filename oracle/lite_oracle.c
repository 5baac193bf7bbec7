/*
 * lite_oracle.c -- CPU oracle for one LiteAttention denoising step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * What it computes (sources: "LiteAttention: Temporal Sparse Attention for
 * Diffusion Transformers" skill page, sections "Core Concept" and
 * "Architecture Overview" -- QK-Skip, Skip-Mask, Persistent Propagation,
 * FlashAttention softmax integration; "LiteAttention: A Temporal Sparse
 * Attention for Diffusion Transformers" abstract -- skip decisions are
 * propagated forward across denoising steps):
 *
 *   For one work item (batch b, head h, query tile i) and one step with
 *   threshold tau (natural-log domain, tau <= 0 or -inf):
 *     s[r][c] = (1/sqrt(d)) * sum_e q[r][e] k[c][e]            (fp64)
 *     for key tiles j = 0 .. Tk-1 in ascending order:
 *       not live in mask_in      -> out bit 0, tile ignored entirely
 *       m_loc[r] = max over valid columns of tile j of s[r][c]
 *       D_j      = max over valid rows r of (m_loc[r] - m_run[r])
 *                  (m_run = -inf before the first processed tile, so D = +inf)
 *       D_j < tau (strict)       -> dead: out bit 0, no softmax / PV work
 *       otherwise                -> out bit 1, online-softmax update of
 *                                   (m_run, l, acc) with tile j
 *     o[r] = acc[r] / l[r]  (0 when no tile was processed)
 *
 * The readings of the pages that this encodes (log-domain threshold, the
 * running max over processed tiles, a tile dies only when every valid row
 * agrees, fresh-dead tiles skip their PV in the current step, ties stay live,
 * partial tiles exclude out-of-range rows and columns, an empty live set
 * gives a zero output row) are listed with their reasons in the design notes.
 *
 * Everything is plain fp64 with no blocking or reordering beyond the tile
 * loop the method itself defines.  Inputs are bf16 bit patterns, converted
 * exactly to fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the top half of an IEEE binary32; the conversion is exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

/*
 * lo_step: run the oracle on n_items work items.
 *
 *   q, k, v    : bf16 bit patterns, layout [B][H][N][d] row-major.
 *   items      : work-item ids, item = (b*H + h)*Tq + i.
 *   mask_in    : [n_items][W] live bits of each item's mask_in row
 *                (word j>>5, bit j&31, 1 = live), W = ceil(Tk/32).
 *   force      : optional [n_items][Tk]; -1 = take the oracle's own decision,
 *                0 = force dead, 1 = force live (used to re-run a tile whose
 *                decision sits within rounding distance of tau).
 *   o          : out [n_items][Br][d]; rows past N are left at 0.
 *   mask_out   : out [n_items][W].
 *   D          : optional out [n_items][Tk]; NaN for tiles not tested.
 *   m_fin,l_fin: optional out [n_items][Br]; final running max (logit units)
 *                and denominator per row.
 *
 * Returns 0, or -1 for an invalid argument.
 */
int lo_step(int B, int H, int N, int d, int Br, int Bc, double tau,
            const uint16_t *q, const uint16_t *k, const uint16_t *v,
            const int64_t *items, int64_t n_items,
            const uint32_t *mask_in, const int8_t *force,
            double *o, uint32_t *mask_out, double *D,
            double *m_fin, double *l_fin, int n_threads)
{
    if (B < 1 || H < 1 || N < 1 || d < 1 || Br < 1 || Bc < 1) return -1;
    if (!q || !k || !v || !items || !mask_in || !o || !mask_out) return -1;
    if (isnan(tau) || tau > 0.0) return -1;
    const int Tq = ceil_div(N, Br);
    const int Tk = ceil_div(N, Bc);
    const int W = ceil_div(Tk, 32);
    const double scale = 1.0 / sqrt((double)d);
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
            double *D_item = D ? D + (size_t)it * Tk : NULL;
            const int8_t *f_item = force ? force + (size_t)it * Tk : NULL;

            for (int r = 0; r < nr; ++r) {
                for (int e = 0; e < d; ++e)
                    qt[r * d + e] = bf16_bits_to_double(q[head_off + (size_t)(r0 + r) * d + e]);
                mrun[r] = -INFINITY;
                l[r] = 0.0;
                for (int e = 0; e < d; ++e) acc[r * d + e] = 0.0;
            }
            for (int w = 0; w < W; ++w) mout_row[w] = 0u;
            if (D_item) for (int j = 0; j < Tk; ++j) D_item[j] = NAN;

            for (int j = 0; j < Tk; ++j) {
                if (!((min_row[j >> 5] >> (j & 31)) & 1u)) continue;   /* dead on entry */
                const int c0 = j * Bc;
                const int nc = (N - c0 < Bc) ? (N - c0) : Bc;          /* valid key columns */
                for (int c = 0; c < nc; ++c)
                    for (int e = 0; e < d; ++e) {
                        kt[c * d + e] = bf16_bits_to_double(k[head_off + (size_t)(c0 + c) * d + e]);
                        vt[c * d + e] = bf16_bits_to_double(v[head_off + (size_t)(c0 + c) * d + e]);
                    }
                /* logits and per-row tile maxima */
                for (int r = 0; r < nr; ++r) {
                    double mx = -INFINITY;
                    for (int c = 0; c < nc; ++c) {
                        double dot = 0.0;
                        for (int e = 0; e < d; ++e) dot += qt[r * d + e] * kt[c * d + e];
                        s[r * Bc + c] = scale * dot;
                        if (s[r * Bc + c] > mx) mx = s[r * Bc + c];
                    }
                    mloc[r] = mx;
                }
                /* QK-Skip statistic: largest rise of any row's max over its running max */
                double Dj = -INFINITY;
                for (int r = 0; r < nr; ++r) {
                    double rise = (mrun[r] == -INFINITY) ? INFINITY : mloc[r] - mrun[r];
                    if (rise > Dj) Dj = rise;
                }
                if (D_item) D_item[j] = Dj;
                int dead = (Dj < tau);
                if (f_item && f_item[j] >= 0) dead = (f_item[j] == 0);
                if (dead) continue;
                mout_row[j >> 5] |= (1u << (j & 31));
                /* online-softmax update with tile j */
                for (int r = 0; r < nr; ++r) {
                    const double mnew = (mloc[r] > mrun[r]) ? mloc[r] : mrun[r];
                    const double alpha = (mrun[r] == -INFINITY) ? 0.0 : exp(mrun[r] - mnew);
                    double lsum = 0.0;
                    for (int e = 0; e < d; ++e) acc[r * d + e] *= alpha;
                    for (int c = 0; c < nc; ++c) {
                        const double p = exp(s[r * Bc + c] - mnew);
                        lsum += p;
                        for (int e = 0; e < d; ++e) acc[r * d + e] += p * vt[c * d + e];
                    }
                    l[r] = l[r] * alpha + lsum;
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
        }
        free(qt); free(kt); free(vt); free(s);
        free(mrun); free(mloc); free(l); free(acc);
    }
    return 0;
}

/* Number of OpenMP threads the oracle will use (for reporting). */
int lo_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
