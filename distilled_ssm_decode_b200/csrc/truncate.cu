// truncate.cu -- modal truncation of the distilled SSM (model-order reduction).
//
// The distillation reduces each head's SSM by balanced or modal truncation
// ("Laughing Hyena Distillery", nubint.ai review, "Proposed method").  In the
// modal (diagonal) form, mode n contributes Re(R_n lambda_n^(j-1)) to tap j, and
// the l1 norm of that contribution is at most
//     score_n = |R_n| / (1 - |lambda_n|).
// Modal truncation keeps the k modes with the largest scores (ties to the lower
// index), so the filter error in l1 is at most the sum of the dropped scores,
// which bounds max|dy| / max|u| of the convolution.  The exact l2 error of the
// dropped part dh_j = Re sum_{n in D} c_n mu_n^(j-1) (c = R, mu = lambda) follows
// from geometric series over pairs of modes (Gramian-type sums):
//     sum_{j>=1} dh_j^2 = 1/2 Re sum_{n,m in D} c_n c_m / (1 - mu_n mu_m)
//                       + 1/2 Re sum_{n,m in D} c_n conj(c_m) / (1 - mu_n conj(mu_m)),
// using Re(z)^2 = (z^2 + 2|z|^2 + conj(z)^2) / 4.
//
// One block per head, one thread per mode; scores, ranks and sums in fp64, sums
// over modes in index order (deterministic).  Per-head work is O(d^2) with d <= 64.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace hyena {

namespace {

__device__ __forceinline__ cd cd_div(cd a, cd b) {   // a / b
    const double den = b.x * b.x + b.y * b.y;
    return cd{(a.x * b.x + a.y * b.y) / den, (a.y * b.x - a.x * b.y) / den};
}

__global__ void __launch_bounds__(HYENA_MAX_MODES)
truncate_kernel(const float2 *__restrict__ lam, const float2 *__restrict__ R, int d, int k,
                int *__restrict__ kept, float2 *__restrict__ lam_out, float2 *__restrict__ R_out,
                double *__restrict__ bound, double *__restrict__ err_l2) {
    __shared__ double score[HYENA_MAX_MODES], row[HYENA_MAX_MODES];
    __shared__ int keep[HYENA_MAX_MODES];
    __shared__ cd c[HYENA_MAX_MODES], mu[HYENA_MAX_MODES];
    const int hd = blockIdx.x, n = threadIdx.x, H = gridDim.x;
    (void)H;
    if (n < d) {
        const float2 l = lam[HB_IDX((size_t)hd * d + n, (long long)H * d)], r = R[HB_IDX((size_t)hd * d + n, (long long)H * d)];
        mu[n] = cd{l.x, l.y};
        c[n] = cd{r.x, r.y};
        const double a = sqrt((double)l.x * l.x + (double)l.y * l.y);
        const double m = sqrt((double)r.x * r.x + (double)r.y * r.y);
        score[n] = a < 1.0 ? m / (1.0 - a) : INFINITY;
    }
    __syncthreads();
    if (n < d) {
        int ahead = 0;
        for (int m = 0; m < d; ++m) ahead += (score[m] > score[n] || (score[m] == score[n] && m < n));
        keep[n] = ahead < k;
    }
    __syncthreads();
    if (n < d) {
        if (keep[n]) {
            int pos = 0;
            for (int m = 0; m < n; ++m) pos += keep[m];
            const size_t o = (size_t)hd * k + pos;
            if (HB_OK(o, (long long)H * k)) {
                kept[o] = n;
                lam_out[o] = lam[HB_IDX((size_t)hd * d + n, (long long)H * d)];
                R_out[o] = R[HB_IDX((size_t)hd * d + n, (long long)H * d)];
            }
            row[n] = 0.0;
        } else {
            // row n of the pair sums over the dropped modes m
            double s = 0.0;
            for (int m = 0; m < d; ++m) {
                if (keep[m]) continue;
                const cd cc = cdmul(c[n], c[m]);
                const cd mm = cdmul(mu[n], mu[m]);
                const cd cb = cdmul(c[n], cd{c[m].x, -c[m].y});
                const cd mb = cdmul(mu[n], cd{mu[m].x, -mu[m].y});
                s += cd_div(cc, cd{1.0 - mm.x, -mm.y}).x + cd_div(cb, cd{1.0 - mb.x, -mb.y}).x;
            }
            row[n] = 0.5 * s;
        }
    }
    __syncthreads();
    if (n == 0) {
        double b = 0.0, e = 0.0;
        bool inf = false;
        for (int m = 0; m < d; ++m) {
            if (keep[m]) continue;
            b += score[m];
            inf |= isinf(score[m]);
            e += row[m];
        }
        if (HB_OK(hd, H)) {
            bound[hd] = b;
            err_l2[hd] = inf ? INFINITY : sqrt(fmax(e, 0.0));
        }
    }
}

}  // namespace

HYENA_BOUNDS_READER(truncate)

cudaError_t launch_modal_truncate(const float2 *lam, const float2 *R, int H, int d, int k, int *kept,
                                  float2 *lam_out, float2 *R_out, double *bound, double *err_l2, cudaStream_t s) {
    if (H == 0) return cudaSuccess;
    truncate_kernel<<<H, HYENA_MAX_MODES, 0, s>>>(lam, R, d, k, kept, lam_out, R_out, bound, err_l2);
    return cudaGetLastError();
}

}  // namespace hyena
