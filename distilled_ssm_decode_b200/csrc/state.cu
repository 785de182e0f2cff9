// state.cu -- prompt -> recurrent-state reduction (Vandermonde contraction).
//
// s[b][n][c] = sum_{j<L} lambda_n^(L-1-j) u[b][j][c],  u = k * v:
// the O(d)-per-channel state that lets generation continue in O(1) per token
// after a prompt ("Laughing Hyena Distillery", nubint.ai review, "Main
// findings"; the recurrence is the modal SSM of "Proposed method").
//
// Only the last W tokens of the prompt are summed, W chosen per head so that
// the older ones weigh at most 2^-40 max|u| (state_window in common.cuh).
// Kernel 1: one thread per (batch, channel, segment of that window) runs Horner's
// rule over its segment for every mode (acc <- acc * lambda + u), then scales by
// lambda^(L - segment end) (fp64 binary powering) and writes a partial state.
// Kernel 2 adds the partials of each (b, n, c) in segment order, so the result
// does not depend on scheduling.  Consecutive threads take consecutive
// channels, so every token row is read coalesced.
#include "common.cuh"
#include "kernels.h"

namespace hyena {

namespace {

constexpr int kThreads = 128;
constexpr int kModeChunk = 16;

int choose_nseg(int B, int L, int Dch) {
    const long long want = 148LL * 1024;   // threads to cover the GPU
    long long cols = (long long)B * Dch;
    long long nseg = (want + cols - 1) / cols;
    long long maxseg = (L + 63) / 64;      // keep segments >= 64 tokens
    if (nseg > maxseg) nseg = maxseg;
    if (nseg < 1) nseg = 1;
    return (int)nseg;
}

template <class Act>
__global__ void __launch_bounds__(kThreads)
state_partial_kernel(const typename Act::T *__restrict__ k, const typename Act::T *__restrict__ v,
                     int L, int Dch, int ch, int d, const float2 *__restrict__ lam,
                     float2 *__restrict__ part /* [B][nseg][d][Dch] */) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= Dch) return;
    const int g = blockIdx.y, b = blockIdx.z, nseg = gridDim.y;
    const int hd = c / ch, H = Dch / ch;
    const long long n_act = (long long)gridDim.z * L * Dch, n_part = (long long)gridDim.z * nseg * d * Dch;
    (void)H; (void)n_act; (void)n_part;
    // the nseg segments cover this head's window [L - W, L)
    const int W = state_window(lam + (size_t)hd * d, d, L);
    const int jstart = L - W;
    const int segw = (W + nseg - 1) / nseg;
    const int j0 = jstart + g * segw, j1 = min(L, j0 + segw);
    for (int n0 = 0; n0 < d; n0 += kModeChunk) {
        float2 l[kModeChunk], a[kModeChunk];
#pragma unroll
        for (int i = 0; i < kModeChunk; ++i) {
            l[i] = (n0 + i < d) ? __ldg(&lam[HB_IDX((size_t)hd * d + n0 + i, (long long)H * d)]) : make_float2(0.f, 0.f);
            a[i] = make_float2(0.f, 0.f);
        }
        for (int j = j0; j < j1; ++j) {
            const size_t o = HB_IDX(((size_t)b * L + j) * Dch + c, n_act);
            const float u = Act::ld(k + o) * Act::ld(v + o);
#pragma unroll
            for (int i = 0; i < kModeChunk; ++i)
                a[i] = make_float2(fmaf(a[i].x, l[i].x, fmaf(-a[i].y, l[i].y, u)),
                                   fmaf(a[i].x, l[i].y, a[i].y * l[i].x));
        }
#pragma unroll
        for (int i = 0; i < kModeChunk; ++i) {
            const int n = n0 + i;
            if (n >= d) break;
            float2 r = make_float2(0.f, 0.f);
            if (j1 > j0) {
                const cd pw = cdpow(cd{l[i].x, l[i].y}, (long long)(L - j1));
                r = cmul(a[i], make_float2((float)pw.x, (float)pw.y));
            }
            const size_t pi = (((size_t)b * nseg + g) * d + n) * Dch + c;
            if (HB_OK(pi, n_part)) part[pi] = r;
        }
    }
}

__global__ void state_sum_kernel(const float2 *__restrict__ part, int nseg, int d, int Dch,
                                 float2 *__restrict__ state) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= Dch) return;
    const int n = blockIdx.y, b = blockIdx.z;
    const long long n_part = (long long)gridDim.z * nseg * d * Dch, n_state = (long long)gridDim.z * d * Dch;
    (void)n_part; (void)n_state;
    float2 s = make_float2(0.f, 0.f);
    for (int g = 0; g < nseg; ++g) s = cadd(s, part[HB_IDX((((size_t)b * nseg + g) * d + n) * Dch + c, n_part)]);
    if (HB_OK(((size_t)b * d + n) * Dch + c, n_state)) state[((size_t)b * d + n) * Dch + c] = s;
}

}  // namespace

HYENA_BOUNDS_READER(state)

size_t state_ws_bytes(int B, int L, int Dch, int d) {
    if (L <= 0) return 0;
    return (size_t)B * choose_nseg(B, L, Dch) * d * Dch * sizeof(float2);
}

cudaError_t launch_prompt_state(const void *k, const void *v, int dtype, int B, int L, int Dch,
                                int H, int d, const float2 *lam, float *state_out, void *scratch,
                                cudaStream_t s) {
    if (B == 0 || Dch == 0) return cudaSuccess;
    if (L == 0) return cudaMemsetAsync(state_out, 0, (size_t)B * d * Dch * 2 * sizeof(float), s);
    const int ch = Dch / H;
    const int nseg = choose_nseg(B, L, Dch);
    float2 *part = static_cast<float2 *>(scratch);
    dim3 grid((Dch + kThreads - 1) / kThreads, nseg, B);
    if (dtype == HYENA_BF16)
        state_partial_kernel<ActBF16><<<grid, kThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), L, Dch, ch,
            d, lam, part);
    else
        state_partial_kernel<ActF32><<<grid, kThreads, 0, s>>>(
            static_cast<const float *>(k), static_cast<const float *>(v), L, Dch, ch, d, lam, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2((Dch + 255) / 256, d, B);
    state_sum_kernel<<<g2, 256, 0, s>>>(part, nseg, d, Dch, reinterpret_cast<float2 *>(state_out));
    return cudaGetLastError();
}

}  // namespace hyena
