// prefill_fft.cu -- FFT long convolution + gating + prompt->state reduction.
//
// Order-2 Hyena operator y = q * (h conv (k * v)) evaluated by zero-padded FFT
// ("Hyena processes long sequences 100x faster than FlashAttention",
// lequren.com: long convolution and element-wise gating in section
// "Hyena層次結構"; fast convolution without forming the full matrix), with the
// weight-tied per-head filter of "Laughing Hyena Distillery" (nubint.ai review,
// "Proposed method") and the prompt -> recurrent-state reduction
// s_n = sum_j lambda_n^(L-1-j) u_j that hands the prompt over to O(1) decode.
//
// Two channels of one head are packed into one complex sequence
// x = u_a + i u_b; because the filter is real, the inverse transform of
// X * H returns (h conv u_a) + i (h conv u_b).  The upper half of the padded
// input is zero (fft_len >= 2L-1 implies L <= fft_len/2), so the first forward
// pass reads only half its inputs, and the last inverse pass stores only the
// first L outputs.
//
// Fused route (N <= 16384): one CTA per (batch, channel pair) keeps the whole
// padded sequence in shared memory: load + gate-in -> state reduction from the
// on-chip u -> forward FFT -> multiply by the head's spectrum -> inverse FFT ->
// gate-out -> store.  Four-step route (N > 16384): N = N1 * 8192; the radix-N1
// step across the long stride and the inner 8192-point transforms go through
// the workspace, and the state comes from the standalone reduction kernel.
#include "common.cuh"
#include "fft.cuh"
#include "kernels.h"

namespace hyena {

using fft::pad;
using fft::padded_len;

namespace {

constexpr int kFusedThreads = 256;
constexpr int kFusedMinBlocks = 2;   // two CTAs per SM: one loads while the other computes; the
                                      // 128-register cap keeps the radix-16 passes' loads in flight

int fused_threads(int N) {
    int t = N / 32;
    if (t < 64) t = 64;
    if (t > kFusedThreads) t = kFusedThreads;
    return t;
}

// ------------------------------------------------------------------ spectrum
// One CTA per head: forward transform of the zero-padded filter, times scale,
// stored in the transform's digit-reversed order (mon_r3 == 0), or, for the
// tensor-core route, at frequency k = k1 + 64 k2 + 4096 k3 in the order its lanes read it
// (mon_r3 = N / 4096): with c = k1 % 2 and f8 = (k1 / 2) R3 + k3, the float2 index is
// ((((f8 / 8) * 4 + (f8 % 8) / 2) * 64 + k2) * 2 + c) * 2 + f8 % 2, so that the 32 lanes of a
// warp (16 values of k2, two of c) read one contiguous 512-byte run per 16-byte load.
__global__ void __launch_bounds__(kFusedThreads)
spectrum_fused_kernel(const float *__restrict__ h, int L, int N, float scale,
                      float2 *__restrict__ spec_perm, int mon_r3) {
    extern __shared__ float2 buf[];
    const int hd = blockIdx.x, H = gridDim.x;
    (void)H;
    const float *hh = h + (size_t)hd * L;
    const bool half_zero = (L <= N / 2);
    const int fill = half_zero ? N / 2 : N;
    for (int t = threadIdx.x; t < fill; t += blockDim.x)
        buf[pad(t)] = make_float2(t < L ? hh[HB_IDX(t, (long long)(H - hd) * L)] : 0.f, 0.f);
    __syncthreads();
    fft::forward(buf, N, half_zero);
    float2 *out = spec_perm + (size_t)hd * N;
    for (int p = threadIdx.x; p < N; p += blockDim.x) {
        int o = p;
        if (mon_r3) {
            const int f = fft::freq_of_pos(p, N);
            const int k1 = f & 63, k2 = (f >> 6) & 63, f8 = (k1 >> 1) * mon_r3 + (f >> 12);
            o = (((((f8 >> 3) * 4 + ((f8 & 7) >> 1)) * 64 + k2) * 2 + (k1 & 1)) * 2) + (f8 & 1);
        }
        if (HB_OK((long long)hd * N + o, (long long)H * N)) out[o] = cscale(buf[pad(p)], scale);
    }
}

// natural-order bins 0..N/2 from the digit-reversed layout
__global__ void spectrum_natural_kernel(const float2 *__restrict__ spec_perm, int N, int N2,
                                        float2 *__restrict__ out) {
    const int hd = blockIdx.y;
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= N) return;
    int f;
    if (N2 == 0) {
        f = fft::freq_of_pos(p, N);
    } else {
        const int N1 = N / N2;
        f = (p / N2) + N1 * fft::freq_of_pos(p % N2, N2);
    }
    if (f <= N / 2 && HB_OK((long long)hd * (N / 2 + 1) + f, (long long)gridDim.y * (N / 2 + 1)))
        out[(size_t)hd * (N / 2 + 1) + f] = spec_perm[HB_IDX((size_t)hd * N + p, (long long)gridDim.y * N)];
}

// ------------------------------------------------------------------ fused prefill
// grid (slots, B); slot = channel pair (paired) or single channel.
template <class Act>
__global__ void __launch_bounds__(kFusedThreads, kFusedMinBlocks)
prefill_fused_kernel(const typename Act::T *__restrict__ q, const typename Act::T *__restrict__ k,
                     const typename Act::T *__restrict__ v, int L, int Dch, int ch, int d, int N,
                     int paired, const float2 *__restrict__ spec_perm,
                     const float2 *__restrict__ lam, typename Act::T *__restrict__ y,
                     float *__restrict__ state_out) {
    extern __shared__ float2 smem[];
    float2 *buf = smem;
    float4 *part = reinterpret_cast<float4 *>(smem + padded_len(N) + 1);  // [d][nseg] (s_a, s_b)

    const int tid = threadIdx.x, nthr = blockDim.x;
    const int b = blockIdx.y;
    const int c0 = paired ? 2 * blockIdx.x : blockIdx.x;
    const int hd = c0 / ch;
    const typename Act::T *kb = k + (size_t)b * L * Dch + c0;
    const typename Act::T *vb = v + (size_t)b * L * Dch + c0;
    // extents (bounds-checked build): activations from kb, state, spectra, poles
    const long long n_act = (long long)gridDim.y * L * Dch - ((long long)b * L * Dch + c0);
    const long long H = Dch / ch;
    (void)n_act; (void)H;

    // 1. gate-in: x_t = (k_a v_a, k_b v_b), zero padding up to N/2; four rows per
    //    thread are loaded before any is used so that their latencies overlap
    constexpr int U = 4;
    for (int t0 = tid; t0 < N / 2; t0 += U * nthr) {
        float2 kk[U], vv[U];
#pragma unroll
        for (int r = 0; r < U; ++r) {
            const int t = t0 + r * nthr;
            kk[r] = vv[r] = make_float2(0.f, 0.f);
            if (t < L && HB_OK((long long)t * Dch + paired, n_act)) {
                const size_t o = (size_t)t * Dch;
                if (paired) { kk[r] = Act::ld2(kb + o); vv[r] = Act::ld2(vb + o); }
                else { kk[r].x = Act::ld(kb + o); vv[r].x = Act::ld(vb + o); }
            }
        }
#pragma unroll
        for (int r = 0; r < U; ++r) {
            const int t = t0 + r * nthr;
            if (t < N / 2) buf[pad(t)] = make_float2(kk[r].x * vv[r].x, kk[r].y * vv[r].y);
        }
    }
    __syncthreads();

    // 2. prompt -> state: s_n = sum_j lambda_n^(L-1-j) x_j over the last W tokens
    //    (older ones weigh < 2^-40 max|u|), by segments: Horner inside a segment,
    //    then scaled by lambda^(L - segment end) (fp64 power), segments summed in order.
    const float2 *lh = lam + (size_t)HB_IDX(hd, H) * d;
    const int jstart = L - state_window(lh, d, L);
    const int nseg = max(1, nthr / d);
    const int seglen = (L - jstart + nseg - 1) / nseg;
    for (int w = tid; w < d * nseg; w += nthr) {
        const int n = w % d, g = w / d;
        const float2 l = __ldg(&lh[n]);
        const int j0 = jstart + g * seglen;
        const int j1 = min(L, j0 + seglen);
        float2 aa = make_float2(0.f, 0.f), ab = make_float2(0.f, 0.f);
        for (int j = j0; j < j1; ++j) {
            const float2 x = buf[pad(j)];
            aa = make_float2(fmaf(aa.x, l.x, fmaf(-aa.y, l.y, x.x)), fmaf(aa.x, l.y, aa.y * l.x));
            ab = make_float2(fmaf(ab.x, l.x, fmaf(-ab.y, l.y, x.y)), fmaf(ab.x, l.y, ab.y * l.x));
        }
        if (j1 > j0) {
            const cd pw = cdpow(cd{l.x, l.y}, (long long)(L - j1));
            const float2 p = make_float2((float)pw.x, (float)pw.y);
            aa = cmul(aa, p);
            ab = cmul(ab, p);
        }
        part[n * nseg + g] = make_float4(aa.x, aa.y, ab.x, ab.y);
    }
    __syncthreads();
    for (int n = tid; n < d; n += nthr) {
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int g = 0; g < nseg; ++g) {
            const float4 p = part[n * nseg + g];
            s.x += p.x; s.y += p.y; s.z += p.z; s.w += p.w;
        }
        float *so = state_out + (((size_t)b * d + n) * Dch + c0) * 2;
        const long long si = (((long long)b * d + n) * Dch + c0) * 2, n_state = (long long)gridDim.y * d * Dch * 2;
        (void)si; (void)n_state;
        if (HB_OK(si + 1, n_state)) *reinterpret_cast<float2 *>(so) = make_float2(s.x, s.y);   // state is 8-byte aligned
        if (paired && HB_OK(si + 3, n_state)) *reinterpret_cast<float2 *>(so + 2) = make_float2(s.z, s.w);
    }

    // 3. forward transform, product with the head's spectrum (scaled by 1/N), inverse
    fft::forward(buf, N, true);
    const float2 *hs = spec_perm + (size_t)hd * N;
    for (int p = tid; p < N; p += nthr) buf[pad(p)] = cmul(buf[pad(p)], __ldg(&hs[HB_IDX(p, (H - hd) * N)]));
    __syncthreads();
    fft::inverse(buf, N, L);

    // 4. gate-out and store the first L outputs
    const typename Act::T *qb = q + (size_t)b * L * Dch + c0;
    typename Act::T *yb = y + (size_t)b * L * Dch + c0;
    for (int t0 = tid; t0 < L; t0 += U * nthr) {
        float2 qq[U];
#pragma unroll
        for (int r = 0; r < U; ++r) {
            const int t = t0 + r * nthr;
            qq[r] = make_float2(0.f, 0.f);
            if (t < L && HB_OK((long long)t * Dch + paired, n_act)) {
                if (paired) qq[r] = Act::ld2(qb + (size_t)t * Dch);
                else qq[r].x = Act::ld(qb + (size_t)t * Dch);
            }
        }
#pragma unroll
        for (int r = 0; r < U; ++r) {
            const int t = t0 + r * nthr;
            if (t < L && HB_OK((long long)t * Dch + paired, n_act)) {
                const float2 z = buf[pad(t)];
                if (paired) Act::st2(yb + (size_t)t * Dch, qq[r].x * z.x, qq[r].y * z.y);
                else Act::st(yb + (size_t)t * Dch, qq[r].x * z.x);
            }
        }
    }
}

// ------------------------------------------------------------------ four-step route
// x = h row (real) for the filter spectrum
struct FilterSrc {
    const float *h;
    int L;
    __device__ __forceinline__ float2 operator()(int col, long long t) const {
        return make_float2(t < L ? h[(size_t)col * L + t] : 0.f, 0.f);
    }
};

template <class Act>
struct ActSrc {
    const typename Act::T *k, *v;
    int L, Dch, nslots, paired;
    __device__ __forceinline__ float2 operator()(int col, long long t) const {
        if (t >= L) return make_float2(0.f, 0.f);
        const int b = col / nslots, slot = col % nslots;
        const int c0 = paired ? 2 * slot : slot;
        const size_t o = ((size_t)b * L + t) * Dch + c0;
        if (paired) {
            const float2 kk = Act::ld2(k + o), vv = Act::ld2(v + o);
            return make_float2(kk.x * vv.x, kk.y * vv.y);
        }
        return make_float2(Act::ld(k + o) * Act::ld(v + o), 0.f);
    }
};

// Thread -> (column, n2) of the outer steps.  COLS8: a block takes 8 adjacent columns x 32 values
// of n2, the column fastest, so that 8 lanes read (or write) one 32-byte piece of an activation row
// (8 channel pairs) instead of 8 separate 4-byte pieces; else a block takes 256 values of n2 of one
// column.
template <bool COLS8>
__device__ __forceinline__ void outer_index(int &col, int &n2) {
    if constexpr (COLS8) {
        col = blockIdx.y * 8 + (threadIdx.x & 7);
        n2 = blockIdx.x * 32 + (threadIdx.x >> 3);
    } else {
        col = blockIdx.y;
        n2 = blockIdx.x * blockDim.x + threadIdx.x;
    }
}

// step 1: Y[col][k1][n2] = w_N^(n2 k1) * DFT_N1 over n1 of x[N2 n1 + n2]
template <int N1, class Src, bool COLS8>
__global__ void __launch_bounds__(256)
fourstep_fwd1_kernel(Src src, int N2, float2 *__restrict__ Y, int ncols) {
    int col, n2;
    outer_index<COLS8>(col, n2);
    if (n2 >= N2 || col >= ncols) return;
    const long long N = (long long)N1 * N2;
    float2 x[N1];
#pragma unroll
    for (int n1 = 0; n1 < N1; ++n1) x[n1] = src(col, (long long)N2 * n1 + n2);
    fft::dftR<N1, false>(x);
    float2 *out = Y + (size_t)col * N + n2;
    // twiddles w_N^(n2 k1) as powers of one exactly reduced w_N^(n2) (at most 15 products)
    const float2 w1 = fft::expi_neg(n2, (int)N);
    float2 w = w1;
#pragma unroll
    for (int k1 = 0; k1 < N1; ++k1) {
        if (HB_OK((long long)col * N + (long long)k1 * N2 + n2, (long long)ncols * N))
            out[(size_t)k1 * N2] = k1 ? cmul(x[k1], w) : x[k1];
        if (k1) w = cmul(w, w1);
    }
}

// step 2: per (col, k1) an N2-point transform in shared memory.
//   mode 0 (spectrum): forward, times scale, stored in place
//   mode 1 (convolution): forward, times spec[head][k1*N2 + p], inverse, stored in place
__global__ void __launch_bounds__(kFusedThreads)
fourstep_inner_kernel(float2 *__restrict__ Y, int N1, int N2, int mode, float scale,
                      const float2 *__restrict__ spec_perm, int nslots, int paired, int ch) {
    extern __shared__ float2 buf[];
    const int col = blockIdx.y, k1 = blockIdx.x;
    const long long N = (long long)N1 * N2;
    float2 *row = Y + (size_t)col * N + (size_t)k1 * N2;
    const long long n_row = (long long)gridDim.y * N - ((long long)col * N + (long long)k1 * N2);
    (void)n_row;
    for (int t = threadIdx.x; t < N2; t += blockDim.x) buf[pad(t)] = row[HB_IDX(t, n_row)];
    __syncthreads();
    fft::forward(buf, N2, false);
    if (mode == 0) {
        for (int p = threadIdx.x; p < N2; p += blockDim.x)
            if (HB_OK(p, n_row)) row[p] = cscale(buf[pad(p)], scale);
        return;
    }
    const int slot = col % nslots;
    const int hd = (paired ? 2 * slot : slot) / ch;
    const float2 *hs = spec_perm + (size_t)hd * N + (size_t)k1 * N2;
    for (int p = threadIdx.x; p < N2; p += blockDim.x) buf[pad(p)] = cmul(buf[pad(p)], __ldg(&hs[p]));
    __syncthreads();
    fft::inverse(buf, N2, -1);
    for (int t = threadIdx.x; t < N2; t += blockDim.x)
        if (HB_OK(t, n_row)) row[t] = buf[pad(t)];
}

// The four-step spectrum rows (row k1 of a head: the spectrum at k1 + N1 f2, f2 in the inner
// transform's digit-reversed order) reordered for the tensor-core inner kernel: inner frequency
// f2 = a1 + 64 a2 + 4096 a3 goes where its lanes read it (the order of spectrum_fused_kernel's
// tensor-core layout at 8192 points).
__global__ void fourstep_spec_tc_kernel(const float2 *__restrict__ spec_perm, int N1, int N2,
                                        float2 *__restrict__ out) {
    const int k1 = blockIdx.x, hd = blockIdx.y;
    const long long N = (long long)N1 * N2;
    const long long n_all = (long long)gridDim.y * N;
    (void)n_all;
    for (int p = threadIdx.x; p < N2; p += blockDim.x) {
        const int f = fft::freq_of_pos(p, N2);
        const int a1 = f & 63, a2 = (f >> 6) & 63, f8 = (a1 >> 1) * 2 + (f >> 12);
        const int o = (((((f8 >> 3) * 4 + ((f8 & 7) >> 1)) * 64 + a2) * 2 + (a1 & 1)) * 2) + (f8 & 1);
        const long long dst = ((long long)hd * N1 + k1) * N2 + o;
        if (HB_OK(dst, n_all))
            out[dst] = spec_perm[HB_IDX((long long)hd * N + (long long)k1 * N2 + p, n_all)];
    }
}

// step 3: inverse across the long stride, gate-out, store the first L outputs
template <int N1, class Act, bool COLS8>
__global__ void __launch_bounds__(256)
fourstep_inv1_kernel(const float2 *__restrict__ Y, int N2, int L, int Dch, int nslots, int paired,
                     const typename Act::T *__restrict__ q, typename Act::T *__restrict__ y, int ncols) {
    int col, n2;
    outer_index<COLS8>(col, n2);
    if (n2 >= N2 || col >= ncols) return;
    const long long N = (long long)N1 * N2;
    const float2 *in = Y + (size_t)col * N + n2;
    const long long n_in = (long long)ncols * N - ((long long)col * N + n2);
    (void)n_in;
    float2 x[N1];
    const float2 w1 = fft::expi_neg(n2, (int)N);
    float2 w = w1;
#pragma unroll
    for (int k1 = 0; k1 < N1; ++k1) {
        x[k1] = k1 ? cmulc(in[HB_IDX((long long)k1 * N2, n_in)], w) : in[0];
        if (k1) w = cmul(w, w1);
    }
    fft::dftR<N1, true>(x);
    const int b = col / nslots, slot = col % nslots;
    const int c0 = paired ? 2 * slot : slot;
#pragma unroll
    for (int n1 = 0; n1 < N1; ++n1) {
        const long long t = (long long)N2 * n1 + n2;
        if (t < L && HB_OK(((long long)b * L + t) * Dch + c0 + paired, (long long)(ncols / nslots) * L * Dch)) {
            const size_t o = ((size_t)b * L + t) * Dch + c0;
            if (paired) {
                const float2 qq = Act::ld2(q + o);
                Act::st2(y + o, qq.x * x[n1].x, qq.y * x[n1].y);
            } else {
                Act::st(y + o, Act::ld(q + o) * x[n1].x);
            }
        }
    }
}

template <class Src, bool COLS8>
cudaError_t launch_fwd1_t(int N1, Src src, int N2, int ncols, float2 *Y, cudaStream_t s) {
    const dim3 grid = COLS8 ? dim3((N2 + 31) / 32, (ncols + 7) / 8) : dim3((N2 + 255) / 256, ncols);
    switch (N1) {
        case 2: fourstep_fwd1_kernel<2, Src, COLS8><<<grid, 256, 0, s>>>(src, N2, Y, ncols); break;
        case 4: fourstep_fwd1_kernel<4, Src, COLS8><<<grid, 256, 0, s>>>(src, N2, Y, ncols); break;
        case 8: fourstep_fwd1_kernel<8, Src, COLS8><<<grid, 256, 0, s>>>(src, N2, Y, ncols); break;
        case 16: fourstep_fwd1_kernel<16, Src, COLS8><<<grid, 256, 0, s>>>(src, N2, Y, ncols); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}
// activation columns (channel pairs or channels) take the 8-column blocks; the filter's do not
template <class Src>
cudaError_t launch_fwd1(int N1, Src src, int N2, int ncols, float2 *Y, cudaStream_t s, bool cols8 = false) {
    return cols8 ? launch_fwd1_t<Src, true>(N1, src, N2, ncols, Y, s) : launch_fwd1_t<Src, false>(N1, src, N2, ncols, Y, s);
}

template <class Act>
cudaError_t launch_inv1(int N1, const float2 *Y, int N2, int L, int Dch, int nslots, int paired,
                        int ncols, const void *q, void *y, cudaStream_t s) {
    const dim3 grid((N2 + 31) / 32, (ncols + 7) / 8);          // 8-column blocks
    using T = typename Act::T;
    const T *qq = static_cast<const T *>(q);
    T *yy = static_cast<T *>(y);
    switch (N1) {
        case 2: fourstep_inv1_kernel<2, Act, true><<<grid, 256, 0, s>>>(Y, N2, L, Dch, nslots, paired, qq, yy, ncols); break;
        case 4: fourstep_inv1_kernel<4, Act, true><<<grid, 256, 0, s>>>(Y, N2, L, Dch, nslots, paired, qq, yy, ncols); break;
        case 8: fourstep_inv1_kernel<8, Act, true><<<grid, 256, 0, s>>>(Y, N2, L, Dch, nslots, paired, qq, yy, ncols); break;
        case 16: fourstep_inv1_kernel<16, Act, true><<<grid, 256, 0, s>>>(Y, N2, L, Dch, nslots, paired, qq, yy, ncols); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

size_t inner_smem_bytes(int N) { return (size_t)padded_len(N) * sizeof(float2); }

cudaError_t set_smem(const void *fn, size_t bytes) {
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <class Act>
cudaError_t prefill_fused(const void *q, const void *k, const void *v, int B, int L, int Dch,
                          int ch, int d, int N, int paired, const float2 *spec_perm,
                          const float2 *lam, void *y, float *state_out, cudaStream_t s) {
    using T = typename Act::T;
    const int nthr = fused_threads(N);
    const int nseg = nthr / d > 0 ? nthr / d : 1;
    const size_t smem = (size_t)(padded_len(N) + 2) * sizeof(float2) + (size_t)d * nseg * sizeof(float4);
    cudaError_t e = set_smem((const void *)prefill_fused_kernel<Act>, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(paired ? Dch / 2 : Dch, B);
    prefill_fused_kernel<Act><<<grid, nthr, smem, s>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), L, Dch, ch,
        d, N, paired, spec_perm, lam, static_cast<T *>(y), state_out);
    return cudaGetLastError();
}

template <class Act>
cudaError_t prefill_fourstep(const void *q, const void *k, const void *v, int B, int L, int Dch,
                             int H, int ch, int d, int N, int paired, const float2 *spec_perm,
                             const float2 *lam, void *y, float *state_out, void *scratch,
                             int *err, cudaStream_t s) {
    using T = typename Act::T;
    const int N2 = kFourStepN2, N1 = N / N2;
    const int nslots = paired ? Dch / 2 : Dch;
    const int ncols = B * nslots;
    float2 *Y = static_cast<float2 *>(scratch);
    char *after = static_cast<char *>(scratch) + (size_t)ncols * N * sizeof(float2);
    ActSrc<Act> src{static_cast<const T *>(k), static_cast<const T *>(v), L, Dch, nslots, paired};
    cudaError_t e = launch_fwd1(N1, src, N2, ncols, Y, s, true);
    if (e != cudaSuccess) return e;
    if (Act::bytes == 2 && fourstep_tc_enabled()) {
        // bf16 activations: the inner transforms on the tensor cores, with the spectrum rows in the
        // order that kernel reads them (after the state partials in the scratch)
        float2 *specm = reinterpret_cast<float2 *>(after + ((state_ws_bytes(B, L, Dch, d) + 255) & ~size_t(255)));
        fourstep_spec_tc_kernel<<<dim3(N1, H), 256, 0, s>>>(spec_perm, N1, N2, specm);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = launch_fourstep_inner_tc(Y, N1, ncols, nslots, paired, ch, H, specm, err, s);
    } else {
        const size_t smem = inner_smem_bytes(N2);
        e = set_smem((const void *)fourstep_inner_kernel, smem);
        if (e != cudaSuccess) return e;
        fourstep_inner_kernel<<<dim3(N1, ncols), kFusedThreads, smem, s>>>(Y, N1, N2, 1, 1.f, spec_perm,
                                                                          nslots, paired, ch);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    e = launch_inv1<Act>(N1, Y, N2, L, Dch, nslots, paired, ncols, q, y, s);
    if (e != cudaSuccess) return e;
    // the state comes from the standalone reduction (u is never whole in one CTA here)
    return launch_prompt_state(k, v, Act::bytes == 2 ? HYENA_BF16 : HYENA_F32, B, L, Dch, H, d,
                               lam, state_out, after, s);
}

}  // namespace

HYENA_BOUNDS_READER(prefill_fft)

size_t spectrum_ws_bytes(int H, int N) { return (size_t)H * N * sizeof(float2); }

cudaError_t launch_spectrum_perm(const float *h, int H, int L, int N, float2 *spec_perm,
                                 float scale, cudaStream_t s) {
    if (H == 0) return cudaSuccess;
    if (N <= kFusedMaxN) {
        const size_t smem = inner_smem_bytes(N);
        cudaError_t e = set_smem((const void *)spectrum_fused_kernel, smem);
        if (e != cudaSuccess) return e;
        spectrum_fused_kernel<<<H, fused_threads(N), smem, s>>>(h, L, N, scale, spec_perm, 0);
        return cudaGetLastError();
    }
    const int N2 = kFourStepN2, N1 = N / N2;
    cudaError_t e = launch_fwd1(N1, FilterSrc{h, L}, N2, H, spec_perm, s);
    if (e != cudaSuccess) return e;
    const size_t smem = inner_smem_bytes(N2);
    e = set_smem((const void *)fourstep_inner_kernel, smem);
    if (e != cudaSuccess) return e;
    fourstep_inner_kernel<<<dim3(N1, H), kFusedThreads, smem, s>>>(spec_perm, N1, N2, 0, scale,
                                                                  nullptr, 1, 0, 1);
    return cudaGetLastError();
}

cudaError_t launch_spectrum_monarch(const float *h, int H, int L, int N, float2 *spec, float scale,
                                    cudaStream_t s) {
    if (H == 0) return cudaSuccess;
    if (N != 4096 && N != 8192 && N != 16384) return cudaErrorInvalidValue;
    const size_t smem = inner_smem_bytes(N);
    cudaError_t e = set_smem((const void *)spectrum_fused_kernel, smem);
    if (e != cudaSuccess) return e;
    spectrum_fused_kernel<<<H, fused_threads(N), smem, s>>>(h, L, N, scale, spec, N / 4096);
    return cudaGetLastError();
}

cudaError_t launch_spectrum_natural(const float2 *spec_perm, int H, int N, float2 *out,
                                    cudaStream_t s) {
    if (H == 0) return cudaSuccess;
    dim3 grid((N + 255) / 256, H);
    spectrum_natural_kernel<<<grid, 256, 0, s>>>(spec_perm, N, N <= kFusedMaxN ? 0 : kFourStepN2, out);
    return cudaGetLastError();
}

size_t fourstep_ws_bytes(int B, int Dch, int ch, int N) {
    if (N <= kFusedMaxN) return 0;
    const int nslots = (ch % 2 == 0) ? Dch / 2 : Dch;
    return (size_t)B * nslots * N * sizeof(float2);
}

cudaError_t launch_prefill_fft(const void *q, const void *k, const void *v, int dtype,
                               int B, int L, int Dch, int H, int d, int N,
                               const float2 *spec_perm, const float2 *lam,
                               void *y, float *state_out, void *scratch, size_t scratch_bytes,
                               int *err, cudaStream_t s) {
    (void)scratch_bytes;
    const int ch = Dch / H;
    const int paired = (ch % 2 == 0) ? 1 : 0;
    if (N <= kFusedMaxN) {
        return dtype == HYENA_BF16
                   ? prefill_fused<ActBF16>(q, k, v, B, L, Dch, ch, d, N, paired, spec_perm, lam, y, state_out, s)
                   : prefill_fused<ActF32>(q, k, v, B, L, Dch, ch, d, N, paired, spec_perm, lam, y, state_out, s);
    }
    return dtype == HYENA_BF16
               ? prefill_fourstep<ActBF16>(q, k, v, B, L, Dch, H, ch, d, N, paired, spec_perm, lam, y, state_out, scratch, err, s)
               : prefill_fourstep<ActF32>(q, k, v, B, L, Dch, H, ch, d, N, paired, spec_perm, lam, y, state_out, scratch, err, s);
}

}  // namespace hyena
