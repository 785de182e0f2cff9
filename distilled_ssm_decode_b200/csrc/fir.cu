// fir.cu -- the undistilled decode baseline: cached-activation long convolution.
//
// Without the distilled recurrence, generating token t means convolving the
// whole history with the long filter:
//
//   y_t = q_t * sum_{j<=t} h_{t-j} u_j,    u_j = k_j v_j
//
// which costs O(t) time and keeps O(t) activations per channel, against the O(d)
// state and O(d) time per token of the distilled modal recurrence ("Laughing
// Hyena Distillery", nubint.ai review, "Main findings": generation in O(d)
// memory and O(dK) time for K tokens, against O(K) and O(K^2) without it).  This
// file is that comparison point on the same hardware: the filter is the same
// modal filter, materialised to the longest length needed.
//
// The history u is cached in fp32 (u = k v is exact in fp32 for bf16 inputs).
// The step kernel is memory-bound: it streams the history [B][t][Dch] once per
// token.  A block covers 32 consecutive channels of one sequence with S warps
// (8, or 32 when there are too few blocks to keep enough loads in flight); warp
// w sums the history rows j = w, w + S, ... (each row read as one 128-byte line
// per warp, 8 rows in flight), then the S partial sums meet in shared memory in
// a fixed order, so the result does not depend on scheduling.
#include "common.cuh"
#include "kernels.h"

namespace hyena {

namespace {

constexpr int kUnroll = 8;      // history rows in flight per warp

template <class Act>
__global__ void __launch_bounds__(256)
fir_fill_kernel(const typename Act::T *__restrict__ k, const typename Act::T *__restrict__ v, int B, int L,
                int Dch, int t_max, float *__restrict__ u_cache) {
    const long long n = (long long)B * L * Dch, row = (long long)L * Dch;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const long long b = e / row, r = e - b * row;
        if (HB_OK(b * t_max * Dch + r, (long long)B * t_max * Dch))
            u_cache[b * t_max * Dch + r] = Act::ld(k + HB_IDX(e, n)) * Act::ld(v + HB_IDX(e, n));
    }
}

template <class Act, int kSlices>
__global__ void __launch_bounds__(32 * kSlices)
fir_step_kernel(const typename Act::T *__restrict__ q, const typename Act::T *__restrict__ k,
                const typename Act::T *__restrict__ v, int Dch, int ch, int t, int t_max,
                const float *__restrict__ h, float *__restrict__ u_cache, typename Act::T *__restrict__ y) {
    __shared__ float part[kSlices][32];
    const int lane = threadIdx.x & 31, slice = threadIdx.x >> 5;
    const int b = blockIdx.y, c = blockIdx.x * 32 + lane;
    const bool valid = c < Dch;
    const int hd = valid ? c / ch : 0;
    const float *hh = h + (size_t)hd * t_max;            // taps of this channel's head
    float *uc = u_cache + (size_t)b * t_max * Dch + c;
    // extents (bounds-checked build), relative to hh and uc
    const long long n_h = (long long)(Dch / ch) * t_max - (long long)hd * t_max;
    const long long n_u = (long long)gridDim.y * t_max * Dch - ((long long)b * t_max * Dch + c);
    (void)n_h; (void)n_u;
    float acc = 0.f;
    if (valid) {
        // rows j < t come from the cache; row t (this token) is added below from registers
        int j = slice;
        for (; j + (kUnroll - 1) * kSlices < t; j += kUnroll * kSlices) {
            float u[kUnroll], w[kUnroll];
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) {
                u[i] = __ldcs(uc + HB_IDX((size_t)(j + i * kSlices) * Dch, n_u));
                w[i] = __ldg(hh + HB_IDX(t - j - i * kSlices, n_h));
            }
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) acc = fmaf(w[i], u[i], acc);
        }
        for (; j < t; j += kSlices) acc = fmaf(__ldg(hh + HB_IDX(t - j, n_h)), __ldcs(uc + HB_IDX((size_t)j * Dch, n_u)), acc);
    }
    part[slice][lane] = acc;
    __syncthreads();
    if (slice == 0 && valid) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kSlices; ++w) s += part[w][lane];
        const size_t o = HB_IDX((size_t)b * Dch + c, (long long)gridDim.y * Dch);
        const float u = Act::ld(k + o) * Act::ld(v + o);
        if (HB_OK((size_t)t * Dch, n_u)) uc[(size_t)t * Dch] = u;     // append this token to the history
        if (HB_OK((size_t)b * Dch + c, (long long)gridDim.y * Dch))
            Act::st(y + o, Act::ld(q + o) * fmaf(__ldg(hh + HB_IDX(0, n_h)), u, s));
    }
}

}  // namespace

HYENA_BOUNDS_READER(fir)

cudaError_t launch_fir_fill(const void *k, const void *v, int dtype, int B, int L, int Dch, int t_max,
                            float *u_cache, cudaStream_t s) {
    const long long n = (long long)B * L * Dch;
    if (n == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
    if (dtype == HYENA_BF16)
        fir_fill_kernel<ActBF16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(k),
                                                        static_cast<const __nv_bfloat16 *>(v), B, L, Dch, t_max,
                                                        u_cache);
    else
        fir_fill_kernel<ActF32><<<blocks, 256, 0, s>>>(static_cast<const float *>(k), static_cast<const float *>(v),
                                                       B, L, Dch, t_max, u_cache);
    return cudaGetLastError();
}

cudaError_t launch_fir_step(const void *q, const void *k, const void *v, int dtype, int B, int Dch, int H, int t,
                            int t_max, const float *h, float *u_cache, void *y, cudaStream_t s) {
    if (B == 0 || Dch == 0) return cudaSuccess;
    const dim3 grid((unsigned)((Dch + 31) / 32), (unsigned)B);
    const int ch = Dch / H;
    // 8 warps per block once there are enough blocks for ~8 MB of history loads in flight
    // (blocks x 8 warps x 8 rows x 128 B); fewer blocks take 32 warps each
    const bool wide = (long long)grid.x * grid.y < 1024;
    using BF = __nv_bfloat16;
    if (dtype == HYENA_BF16) {
        const BF *qq = static_cast<const BF *>(q), *kk = static_cast<const BF *>(k), *vv = static_cast<const BF *>(v);
        if (wide)
            fir_step_kernel<ActBF16, 32><<<grid, 1024, 0, s>>>(qq, kk, vv, Dch, ch, t, t_max, h, u_cache, static_cast<BF *>(y));
        else
            fir_step_kernel<ActBF16, 8><<<grid, 256, 0, s>>>(qq, kk, vv, Dch, ch, t, t_max, h, u_cache, static_cast<BF *>(y));
    } else {
        const float *qq = static_cast<const float *>(q), *kk = static_cast<const float *>(k),
                    *vv = static_cast<const float *>(v);
        if (wide)
            fir_step_kernel<ActF32, 32><<<grid, 1024, 0, s>>>(qq, kk, vv, Dch, ch, t, t_max, h, u_cache, static_cast<float *>(y));
        else
            fir_step_kernel<ActF32, 8><<<grid, 256, 0, s>>>(qq, kk, vv, Dch, ch, t, t_max, h, u_cache, static_cast<float *>(y));
    }
    return cudaGetLastError();
}

}  // namespace hyena
