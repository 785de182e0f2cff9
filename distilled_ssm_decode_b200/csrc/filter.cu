// filter.cu -- modal filter materialisation (Vandermonde evaluation).
//
// h_0 = Dskip, h_j = Re sum_n R_n lambda_n^(j-1): the impulse response of the
// low-order modal state-space model distilled from each long convolution
// ("Laughing Hyena Distillery", nubint.ai review, "Proposed method"), one
// filter per head (weight tying across the head's channels).
//
// Each thread produces a run of kRun consecutive taps.  The first power of the
// run comes from fp64 binary powering of lambda (exact to a few fp64 ulps even
// for j ~ 1e5), the rest of the run from fp64 multiplications, and the sum over
// modes is accumulated in fp64 before one rounding to fp32.
#include "common.cuh"
#include "kernels.h"

namespace hyena {

namespace {
constexpr int kRun = 16;

__global__ void __launch_bounds__(128)
filter_kernel(const float2 *__restrict__ lam, const float2 *__restrict__ R,
              const float *__restrict__ Dskip, int d, int L, float *__restrict__ h, int *clear) {
    const int hd = blockIdx.y, H = gridDim.y;
    if (clear && hd == 0 && blockIdx.x == 0 && threadIdx.x == 0) *clear = 0;
    (void)H;
    const long long j0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * kRun;
    if (j0 >= L) return;
    double acc[kRun];
#pragma unroll
    for (int r = 0; r < kRun; ++r) acc[r] = 0.0;
    // tap j >= 1 uses lambda^(j-1); the run starts at power max(j0-1, 0)
    const long long p0 = j0 > 0 ? j0 - 1 : 0;
    for (int n = 0; n < d; ++n) {
        const float2 lf = __ldg(&lam[HB_IDX((size_t)hd * d + n, (long long)H * d)]);
        const float2 rf = __ldg(&R[HB_IDX((size_t)hd * d + n, (long long)H * d)]);
        const cd l{lf.x, lf.y};
        cd p = cdpow(l, p0);
#pragma unroll
        for (int r = 0; r < kRun; ++r) {
            const long long j = j0 + r;
            if (j >= 1) {
                acc[r] += (double)rf.x * p.x - (double)rf.y * p.y;   // Re(R p)
                p = cdmul(p, l);
            }
        }
    }
    float *out = h + (size_t)hd * L;
#pragma unroll
    for (int r = 0; r < kRun; ++r) {
        const long long j = j0 + r;
        if (j < L && HB_OK((long long)hd * L + j, (long long)H * L)) out[j] = (j == 0) ? Dskip[HB_IDX(hd, H)] : (float)acc[r];
    }
}
}  // namespace

HYENA_BOUNDS_READER(filter)

cudaError_t launch_filter(const float2 *lam, const float2 *R, const float *Dskip,
                          int H, int d, int L, float *h, cudaStream_t s, int *clear) {
    if (H == 0 || L == 0) return cudaSuccess;
    const int threads = 128;
    const long long runs = (L + kRun - 1) / kRun;
    dim3 grid((unsigned)((runs + threads - 1) / threads), (unsigned)H);
    filter_kernel<<<grid, threads, 0, s>>>(lam, R, Dskip, d, L, h, clear);
    return cudaGetLastError();
}

}  // namespace hyena
