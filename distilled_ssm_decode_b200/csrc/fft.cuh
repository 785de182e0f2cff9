// fft.cuh -- shared-memory complex FFT for the long-convolution prefill.
//
// The long convolution is evaluated by zero-padded FFTs, the "fast
// convolution" route by which the Hyena operator avoids forming its full
// Toeplitz matrix ("Hyena processes long sequences 100x faster than
// FlashAttention", lequren.com, section "Hyena層次結構").
//
// Layout and algorithm (written for this library):
//  * One complex sequence of length N = 2^m lives in shared memory as float2,
//    with one float2 of padding after every 16 (index i lives at i + i/16) so
//    that the strided accesses of the late passes do not all hit one bank.
//  * Forward transform = decimation-in-frequency passes of radix 16 (and one
//    final pass of radix 2, 4 or 8 for the leftover bits).  A pass over
//    sub-transforms of size M with span s = M/R takes, for each (block g,
//    offset i < s), the R values at g*M + i + k*s, applies an R-point DFT in
//    registers, multiplies output k' by w_M^(i k'), and writes it back to the
//    same R slots.  The result is the DFT in digit-reversed order.
//  * The inverse runs the mirrored passes in reverse order (conjugate
//    twiddles, inverse small DFTs, decimation in time) and so takes the
//    digit-reversed spectrum back to natural order; it is unnormalised
//    (factor N), which the caller folds into the filter spectrum.
//  * Filter spectra are produced by the same forward transform, so the
//    pointwise product needs no reordering.
//  * Twiddles come from sincospif of an exactly reduced rational angle (two
//    calls per radix-16 group) and short products of those.
#pragma once

#include "common.cuh"

namespace hyena {
namespace fft {

__device__ __forceinline__ int pad(int i) { return i + (i >> 4); }
__host__ __device__ __forceinline__ int padded_len(int n) { return n + (n >> 4) + 1; }

// exp(-2 pi i * num / den) for 0 <= num < den (den a power of two), fp32.
// The argument -2 num/den is exact in fp32 for den <= 2^24.
__device__ __forceinline__ float2 expi_neg(int num, int den) {
    float s, c;
    sincospif(-2.0f * (float)num / (float)den, &s, &c);
    return make_float2(c, s);
}

// ------------------------------------------------------------------ small DFTs
// In-place R-point DFT in natural order: X[k] = sum_n x[n] w_R^(sgn * n k),
// w_R = exp(-2 pi i / R); INV selects sgn = -1 (i.e. exp(+2 pi i n k / R)).
template <bool INV>
__device__ __forceinline__ void dft2(float2 &a, float2 &b) {
    float2 t = a;
    a = cadd(t, b);
    b = csub(t, b);
}

// multiply by -i (forward) or +i (inverse)
template <bool INV>
__device__ __forceinline__ float2 mul_mi(float2 a) {
    return INV ? make_float2(-a.y, a.x) : make_float2(a.y, -a.x);
}

template <bool INV>
__device__ __forceinline__ void dft4(float2 &x0, float2 &x1, float2 &x2, float2 &x3) {
    float2 a0 = cadd(x0, x2), a1 = csub(x0, x2);
    float2 b0 = cadd(x1, x3), b1 = mul_mi<INV>(csub(x1, x3));
    x0 = cadd(a0, b0);
    x2 = csub(a0, b0);
    x1 = cadd(a1, b1);
    x3 = csub(a1, b1);
}

template <bool INV>
__device__ __forceinline__ void dft8(float2 *x) {
    // x[n], n = 0..7 ; split n = n1 + 2 n2 ... use 2 x radix-4 then radix-2 combine
    float2 e0 = x[0], e1 = x[2], e2 = x[4], e3 = x[6];
    float2 o0 = x[1], o1 = x[3], o2 = x[5], o3 = x[7];
    dft4<INV>(e0, e1, e2, e3);
    dft4<INV>(o0, o1, o2, o3);
    const float r = 0.70710678118654752440f;
    // twiddles w_8^k (forward exp(-i pi k/4)), k = 0..3
    float2 t1 = INV ? make_float2(r * (o1.x - o1.y), r * (o1.x + o1.y))
                    : make_float2(r * (o1.x + o1.y), r * (o1.y - o1.x));
    float2 t2 = mul_mi<INV>(o2);
    float2 t3 = INV ? make_float2(-r * (o3.x + o3.y), r * (o3.x - o3.y))
                    : make_float2(r * (o3.y - o3.x), -r * (o3.x + o3.y));
    x[0] = cadd(e0, o0); x[4] = csub(e0, o0);
    x[1] = cadd(e1, t1); x[5] = csub(e1, t1);
    x[2] = cadd(e2, t2); x[6] = csub(e2, t2);
    x[3] = cadd(e3, t3); x[7] = csub(e3, t3);
}

template <bool INV>
__device__ __forceinline__ void dft16(float2 *x) {
    // n = n1 + 4 n2 (n1, n2 in 0..3); k = k2 + 4 k1.
    // step 1: for each n1, 4-point DFT over n2 -> A[n1][k2]
    float2 a[4][4];
#pragma unroll
    for (int n1 = 0; n1 < 4; ++n1) {
        a[n1][0] = x[n1]; a[n1][1] = x[n1 + 4]; a[n1][2] = x[n1 + 8]; a[n1][3] = x[n1 + 12];
        dft4<INV>(a[n1][0], a[n1][1], a[n1][2], a[n1][3]);
    }
    // step 2: twiddle A[n1][k2] *= w_16^(n1 k2)
    const float c1 = 0.92387953251128675613f, s1 = 0.38268343236508977173f;
    const float r = 0.70710678118654752440f;
    const float2 w[10] = {
        make_float2(1.f, 0.f),
        make_float2(c1, INV ? s1 : -s1),      // w^1
        make_float2(r, INV ? r : -r),         // w^2
        make_float2(s1, INV ? c1 : -c1),      // w^3
        make_float2(0.f, INV ? 1.f : -1.f),   // w^4
        make_float2(-s1, INV ? c1 : -c1),     // w^5
        make_float2(-r, INV ? r : -r),        // w^6
        make_float2(-c1, INV ? s1 : -s1),     // w^7
        make_float2(-1.f, 0.f),               // w^8
        make_float2(-c1, INV ? -s1 : s1),     // w^9
    };
#pragma unroll
    for (int n1 = 1; n1 < 4; ++n1)
#pragma unroll
        for (int k2 = 1; k2 < 4; ++k2) a[n1][k2] = cmul(a[n1][k2], w[n1 * k2]);
    // step 3: for each k2, 4-point DFT over n1 -> X[k2 + 4 k1]
#pragma unroll
    for (int k2 = 0; k2 < 4; ++k2) {
        float2 b0 = a[0][k2], b1 = a[1][k2], b2 = a[2][k2], b3 = a[3][k2];
        dft4<INV>(b0, b1, b2, b3);
        x[k2] = b0; x[k2 + 4] = b1; x[k2 + 8] = b2; x[k2 + 12] = b3;
    }
}

template <int R, bool INV>
__device__ __forceinline__ void dftR(float2 *x) {
    if constexpr (R == 2) dft2<INV>(x[0], x[1]);
    else if constexpr (R == 4) dft4<INV>(x[0], x[1], x[2], x[3]);
    else if constexpr (R == 8) dft8<INV>(x);
    else dft16<INV>(x);
}

// w^k for k = 0..R-1 given the group's base angle num/den (w = exp(-2 pi i num/den)),
// conjugated for the inverse.  Two accurate evaluations (w, w^4), the rest by products.
template <int R, bool INV>
__device__ __forceinline__ void twiddles(float2 *tw, int num, int den) {
    float2 w1 = expi_neg(num, den);
    tw[0] = make_float2(1.f, 0.f);
    if constexpr (R >= 2) tw[1] = w1;
    if constexpr (R >= 4) {
        float2 w2 = cmul(w1, w1);
        tw[2] = w2;
        tw[3] = cmul(w2, w1);
    }
    if constexpr (R >= 8) {
        float2 w4 = expi_neg(num * 4, den);     // num < den / R, so 4 num < den
#pragma unroll
        for (int k = 4; k < R; ++k) {
            float2 base = (k >= 12) ? cmul(cmul(w4, w4), w4) : (k >= 8 ? cmul(w4, w4) : w4);
            tw[k] = (k & 3) ? cmul(base, tw[k & 3]) : base;
        }
    }
    if constexpr (INV) {
#pragma unroll
        for (int k = 0; k < R; ++k) tw[k].y = -tw[k].y;
    }
}

// ------------------------------------------------------------------ passes
// One DIF pass of radix R on sub-transforms of size M over buffer buf (padded
// indexing).  Block-wide: groups distributed over threads [tid0, tid0+nthr).
// If HALF_IN, inputs at k >= R/2 are known zero (only valid for M == N with
// the upper half zero).
template <int R, bool HALF_IN>
__device__ __forceinline__ void fwd_pass(float2 *buf, int N, int M, int tid, int nthr) {
    const int s = M / R;               // powers of two: index math by shifts and masks
    const int lgs = __ffs(s) - 1;
    const int groups = N / R;
    for (int gi = tid; gi < groups; gi += nthr) {
        const int i = gi & (s - 1);
        const int base = ((gi >> lgs) * M) + i;
        float2 x[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            if (HALF_IN && k >= R / 2) x[k] = make_float2(0.f, 0.f);
            else x[k] = buf[pad(base + k * s)];
        }
        dftR<R, false>(x);
        if (s > 1) {
            float2 tw[R];
            twiddles<R, false>(tw, i, M);
#pragma unroll
            for (int k = 1; k < R; ++k) x[k] = cmul(x[k], tw[k]);
        }
#pragma unroll
        for (int k = 0; k < R; ++k) buf[pad(base + k * s)] = x[k];
    }
}

// Mirror of fwd_pass: conjugate twiddles first, then the inverse R-point DFT.
// If OUT_LIMIT >= 0, only outputs at positions < out_limit are stored (used on
// the final pass, M == N, when only the first L outputs are needed).
template <int R>
__device__ __forceinline__ void inv_pass(float2 *buf, int N, int M, int tid, int nthr, int out_limit) {
    const int s = M / R;
    const int lgs = __ffs(s) - 1;
    const int groups = N / R;
    for (int gi = tid; gi < groups; gi += nthr) {
        const int i = gi & (s - 1);
        const int base = ((gi >> lgs) * M) + i;
        float2 x[R];
#pragma unroll
        for (int k = 0; k < R; ++k) x[k] = buf[pad(base + k * s)];
        if (s > 1) {
            float2 tw[R];
            twiddles<R, true>(tw, i, M);
#pragma unroll
            for (int k = 1; k < R; ++k) x[k] = cmul(x[k], tw[k]);
        }
        dftR<R, true>(x);
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int p = base + k * s;
            if (out_limit < 0 || p < out_limit) buf[pad(p)] = x[k];
        }
    }
}

// Radix plan: log2N = 4*a + r -> a passes of radix 16, then one pass of 2^r (r > 0).
__host__ __device__ __forceinline__ int ilog2(int n) {
    int l = 0;
    while ((1 << l) < n) ++l;
    return l;
}

// Full forward transform (block-wide, includes the __syncthreads between passes).
// upper_half_zero: the input's positions >= N/2 are zero and need not be read.
__device__ __forceinline__ void forward(float2 *buf, int N, bool upper_half_zero) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int lg = ilog2(N);
    const int a = lg / 4, r = lg % 4;
    int M = N;
    bool first = true;
    for (int p = 0; p < a; ++p) {
        if (first && upper_half_zero) fwd_pass<16, true>(buf, N, M, tid, nthr);
        else fwd_pass<16, false>(buf, N, M, tid, nthr);
        first = false;
        M /= 16;
        __syncthreads();
    }
    if (r > 0) {
        const bool hz = first && upper_half_zero;
        if (r == 1) { if (hz) fwd_pass<2, true>(buf, N, M, tid, nthr); else fwd_pass<2, false>(buf, N, M, tid, nthr); }
        if (r == 2) { if (hz) fwd_pass<4, true>(buf, N, M, tid, nthr); else fwd_pass<4, false>(buf, N, M, tid, nthr); }
        if (r == 3) { if (hz) fwd_pass<8, true>(buf, N, M, tid, nthr); else fwd_pass<8, false>(buf, N, M, tid, nthr); }
        __syncthreads();
    }
}

// Full inverse transform (unnormalised).  Only positions < out_limit of the
// result are guaranteed written (out_limit = -1: all).
__device__ __forceinline__ void inverse(float2 *buf, int N, int out_limit) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int lg = ilog2(N);
    const int a = lg / 4, r = lg % 4;
    int M = 1 << r;
    if (r > 0) {
        const int lim = (a == 0) ? out_limit : -1;
        if (r == 1) inv_pass<2>(buf, N, M, tid, nthr, lim);
        if (r == 2) inv_pass<4>(buf, N, M, tid, nthr, lim);
        if (r == 3) inv_pass<8>(buf, N, M, tid, nthr, lim);
        __syncthreads();
    }
    for (int p = 0; p < a; ++p) {
        M *= 16;
        inv_pass<16>(buf, N, M, tid, nthr, (p == a - 1) ? out_limit : -1);
        __syncthreads();
    }
}

// Frequency index held at position p of the forward transform's output.
__host__ __device__ __forceinline__ int freq_of_pos(int p, int N) {
    const int lg = ilog2(N);
    const int a = lg / 4, r = lg % 4;
    // forward radices in order: 16 (a times) then 2^r
    int f = 0, mult = 1, M = N;
    for (int q = 0; q < a + (r > 0 ? 1 : 0); ++q) {
        const int R = (q < a) ? 16 : (1 << r);
        const int s = M / R;
        const int k = p / s;    // digit of this pass
        p = p % s;
        f += k * mult;
        mult *= R;
        M = s;
    }
    return f;
}

}  // namespace fft
}  // namespace hyena
