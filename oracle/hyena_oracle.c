/*
 * hyena_oracle.c -- plain fp64 CPU oracle for the gated modal long convolution.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * path.
 *
 * What it computes (all arithmetic in IEEE double, complex numbers written out
 * as (re, im) pairs, no blocking, no FFT, no reordering beyond the definitions):
 *
 *   Operator (order-2 Hyena block: a long convolution between two element-wise
 *   gates -- "Hyena processes long sequences 100x faster than FlashAttention"
 *   (lequren.com), sections "Hyena層次結構" / "Hyena塊"):
 *       u_t = k_t * v_t,   z_t = sum_{j<=t} h_{t-j} u_j,   y_t = q_t * z_t
 *
 *   Filter, one per head and shared by all channels of that head (weight tying:
 *   Laughing Hyena Distillery, nubint.ai review, "Proposed method" and the
 *   abstract), in the modal (diagonal complex-pole) state-space form that the
 *   distillation produces:
 *       h_0 = Dskip,   h_j = Re sum_{n<d} R_n lambda_n^(j-1)   (j >= 1)
 *
 *   Recurrent form with O(d) state per channel (Laughing Hyena Distillery
 *   review, "Main findings": O(d) memory and O(dK) time for K tokens):
 *       y_t = q_t (Dskip u_t + Re sum_n R_n s_n)    -- emitted from the state
 *       s_n <- lambda_n s_n + u_t                   -- then the state advances
 *   and the state that a length-L prompt leaves behind:
 *       s_n = sum_{j<L} lambda_n^(L-1-j) u_j
 *
 * Readings taken where the pages are silent:
 *   - channel c belongs to head c / (Dch / H) (contiguous heads);
 *   - decode emits y_t from the state *before* the update, then updates: the
 *     only order under which prompt state + decode equals the full convolution;
 *   - lambda^0 = 1 also for lambda = 0, so lambda = 0 gives the 2-tap filter
 *     [Dskip, Re sum R];
 *   - activations given in bf16 are widened exactly to double by the caller.
 *
 * Layouts (all row-major, complex interleaved re,im):
 *   lam, R : [H][d][2]       Dskip : [H]
 *   q,k,v,y: [B][L][Dch]     (channel innermost)
 *   h      : [H][L]
 *   state  : [B][d][Dch][2]  (mode-major, channel innermost)
 *   spec   : [H][N/2+1][2]
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC hyena_oracle.c -o libhyena_oracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of OpenMP threads the oracle's parallel loops use. */
int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------
 * Filter materialisation: h_0 = Dskip, h_j = Re sum_n R_n lambda_n^(j-1).
 * Powers by repeated multiplication p <- p * lambda starting from p = 1, so
 * lambda = 0 gives p = 1 at j = 1 and 0 afterwards.
 * ------------------------------------------------------------------------- */
void oracle_filter(const double *lam, const double *R, const double *Dskip,
                   int H, int d, int L, double *h)
{
    for (int hd = 0; hd < H; ++hd) {
        double *hh = h + (size_t)hd * L;
        if (L <= 0) continue;
        hh[0] = Dskip[hd];
        for (int j = 1; j < L; ++j) hh[j] = 0.0;
        for (int n = 0; n < d; ++n) {
            const double lr = lam[((size_t)hd * d + n) * 2 + 0];
            const double li = lam[((size_t)hd * d + n) * 2 + 1];
            const double rr = R[((size_t)hd * d + n) * 2 + 0];
            const double ri = R[((size_t)hd * d + n) * 2 + 1];
            double pr = 1.0, pi = 0.0;               /* lambda^(j-1) */
            for (int j = 1; j < L; ++j) {
                /* Re(R * p) */
                hh[j] += rr * pr - ri * pi;
                /* p <- p * lambda */
                const double nr = pr * lr - pi * li;
                const double ni = pr * li + pi * lr;
                pr = nr; pi = ni;
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * Spectrum of the zero-padded filter, by the DFT definition:
 *   spec[hd][f] = sum_{j<L} h[hd][j] exp(-2 pi i j f / N),  f = 0..N/2.
 * The angle index (j*f) mod N is reduced exactly in integers first.
 * nbins/bins: evaluate only the listed bins (bins == NULL -> all N/2+1),
 * output spec[hd][i] for i < nbins.
 * ------------------------------------------------------------------------- */
void oracle_spectrum(const double *h, int H, int L, int N,
                     const int *bins, int nbins, double *spec)
{
    const double two_pi = 6.283185307179586476925286766559;
    const int nb = bins ? nbins : (N / 2 + 1);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int hd = 0; hd < H; ++hd) {
        for (int i = 0; i < nb; ++i) {
            const int64_t f = bins ? bins[i] : i;
            double sr = 0.0, si = 0.0;
            for (int j = 0; j < L; ++j) {
                const int64_t m = ((int64_t)j * f) % N;
                const double ang = -two_pi * (double)m / (double)N;
                sr += h[(size_t)hd * L + j] * cos(ang);
                si += h[(size_t)hd * L + j] * sin(ang);
            }
            spec[((size_t)hd * nb + i) * 2 + 0] = sr;
            spec[((size_t)hd * nb + i) * 2 + 1] = si;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Direct causal convolution, O(L^2) per channel (the definition):
 *   y[b][t][c] = q[b][t][c] * sum_{j<=t} h[head(c)][t-j] * k[b][j][c] * v[b][j][c]
 * ------------------------------------------------------------------------- */
void oracle_conv_direct(const double *q, const double *k, const double *v,
                        int B, int L, int Dch, int H, const double *h, double *y)
{
    const int ch = Dch / H;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < Dch; ++c) {
            const double *hh = h + (size_t)(c / ch) * L;
            for (int t = 0; t < L; ++t) {
                double z = 0.0;
                for (int j = 0; j <= t; ++j) {
                    const size_t ij = ((size_t)b * L + j) * Dch + c;
                    z += hh[t - j] * (k[ij] * v[ij]);
                }
                const size_t it = ((size_t)b * L + t) * Dch + c;
                y[it] = q[it] * z;
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * State left by a length-L prompt, by its definition:
 *   s[b][n][c] = sum_{j<L} lambda_n^(L-1-j) * u[b][j][c]
 * Walking j downwards from L-1, the power starts at 1 and is multiplied by
 * lambda once per step.
 * ------------------------------------------------------------------------- */
void oracle_prompt_state(const double *k, const double *v,
                         int B, int L, int Dch, int H, int d,
                         const double *lam, double *s)
{
    const int ch = Dch / H;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < Dch; ++c) {
            const int hd = c / ch;
            for (int n = 0; n < d; ++n) {
                const double lr = lam[((size_t)hd * d + n) * 2 + 0];
                const double li = lam[((size_t)hd * d + n) * 2 + 1];
                double pr = 1.0, pi = 0.0;      /* lambda^(L-1-j) */
                double sr = 0.0, si = 0.0;
                for (int j = L - 1; j >= 0; --j) {
                    const size_t ij = ((size_t)b * L + j) * Dch + c;
                    const double u = k[ij] * v[ij];
                    sr += pr * u;
                    si += pi * u;
                    const double nr = pr * lr - pi * li;
                    const double ni = pr * li + pi * lr;
                    pr = nr; pi = ni;
                }
                s[(((size_t)b * d + n) * Dch + c) * 2 + 0] = sr;
                s[(((size_t)b * d + n) * Dch + c) * 2 + 1] = si;
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * Recurrent evaluation over T tokens per sequence (one decode step per token):
 *   for t: u = k*v;  y_t = q_t (Dskip u + Re sum_n R_n s_n);  s_n <- lambda_n s_n + u
 * q,k,v,y: [B][T][Dch]; s: [B][d][Dch][2], read as the initial state and
 * overwritten with the final one.  T = 1 is a single decode step; T = L from a
 * zero state is the prefill evaluated as a recurrence.
 * ------------------------------------------------------------------------- */
void oracle_recurrent(const double *q, const double *k, const double *v,
                      int B, int T, int Dch, int H, int d,
                      const double *lam, const double *R, const double *Dskip,
                      double *s, double *y)
{
    const int ch = Dch / H;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < Dch; ++c) {
            const int hd = c / ch;
            for (int t = 0; t < T; ++t) {
                const size_t it = ((size_t)b * T + t) * Dch + c;
                const double u = k[it] * v[it];
                double acc = Dskip[hd] * u;
                for (int n = 0; n < d; ++n) {
                    const double rr = R[((size_t)hd * d + n) * 2 + 0];
                    const double ri = R[((size_t)hd * d + n) * 2 + 1];
                    const size_t is = (((size_t)b * d + n) * Dch + c) * 2;
                    acc += rr * s[is + 0] - ri * s[is + 1];        /* Re(R s) */
                }
                y[it] = q[it] * acc;
                for (int n = 0; n < d; ++n) {
                    const double lr = lam[((size_t)hd * d + n) * 2 + 0];
                    const double li = lam[((size_t)hd * d + n) * 2 + 1];
                    const size_t is = (((size_t)b * d + n) * Dch + c) * 2;
                    const double sr = s[is + 0], si = s[is + 1];
                    s[is + 0] = lr * sr - li * si + u;               /* lambda s + u */
                    s[is + 1] = lr * si + li * sr;
                }
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * Modal truncation (model-order reduction of the modal SSM: "Laughing Hyena
 * Distillery", nubint.ai review, "Proposed method", balanced and modal
 * truncation).  Each mode's share of the filter taps j >= 1 is
 * Re(R_n lambda_n^(j-1)), whose l1 norm is at most
 *     score_n = |R_n| / (1 - |lambda_n|)      (+inf when |lambda_n| >= 1).
 * The k modes with the largest scores are kept, ties going to the lower
 * index: mode n is kept iff fewer than k modes m have score_m > score_n or
 * (score_m == score_n and m < n).  Kept modes are written in index order.
 * Outputs per head: kept[k] (indices), lam_out/R_out [k][2], bound = sum of
 * the dropped scores, and, by direct summation over taps j = 1..J of the
 * dropped modes' filter dh_j = Re sum_{n dropped} R_n lambda_n^(j-1) (powers by
 * repeated multiplication), err_l1 = sum |dh_j| and err_l2 = sqrt(sum dh_j^2).
 * ------------------------------------------------------------------------- */
void oracle_modal_truncate(const double *lam, const double *R, int H, int d, int k, int J,
                           int *kept, double *lam_out, double *R_out,
                           double *bound, double *err_l1, double *err_l2)
{
    for (int hd = 0; hd < H; ++hd) {
        const double *lh = lam + (size_t)hd * d * 2, *rh = R + (size_t)hd * d * 2;
        double score[256];
        int keep[256];
        for (int n = 0; n < d; ++n) {
            const double a = sqrt(lh[2 * n] * lh[2 * n] + lh[2 * n + 1] * lh[2 * n + 1]);
            const double r = sqrt(rh[2 * n] * rh[2 * n] + rh[2 * n + 1] * rh[2 * n + 1]);
            score[n] = a < 1.0 ? r / (1.0 - a) : INFINITY;
        }
        int out = 0;
        double b = 0.0;
        for (int n = 0; n < d; ++n) {
            int ahead = 0;
            for (int m = 0; m < d; ++m)
                if (score[m] > score[n] || (score[m] == score[n] && m < n)) ++ahead;
            keep[n] = ahead < k;
            if (keep[n]) {
                kept[(size_t)hd * k + out] = n;
                lam_out[((size_t)hd * k + out) * 2 + 0] = lh[2 * n];
                lam_out[((size_t)hd * k + out) * 2 + 1] = lh[2 * n + 1];
                R_out[((size_t)hd * k + out) * 2 + 0] = rh[2 * n];
                R_out[((size_t)hd * k + out) * 2 + 1] = rh[2 * n + 1];
                ++out;
            } else {
                b += score[n];
            }
        }
        bound[hd] = b;
        double l1 = 0.0, l2 = 0.0;
        double pr[256], pi[256];
        for (int n = 0; n < d; ++n) { pr[n] = 1.0; pi[n] = 0.0; }
        for (int j = 1; j <= J; ++j) {
            double dh = 0.0;
            for (int n = 0; n < d; ++n) {
                if (keep[n]) continue;
                dh += rh[2 * n] * pr[n] - rh[2 * n + 1] * pi[n];
                const double nr = pr[n] * lh[2 * n] - pi[n] * lh[2 * n + 1];
                const double ni = pr[n] * lh[2 * n + 1] + pi[n] * lh[2 * n];
                pr[n] = nr; pi[n] = ni;
            }
            l1 += fabs(dh);
            l2 += dh * dh;
        }
        err_l1[hd] = l1;
        err_l2[hd] = sqrt(l2);
    }
}
