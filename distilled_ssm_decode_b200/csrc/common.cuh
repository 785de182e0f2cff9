// common.cuh -- small device helpers shared by the libhyena_b200 kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hyena.h"   // from include/ (on the -I path)

namespace hyena {

// ---------------------------------------------------------------- bounds-checked build
// Built with -DHYENA_DEBUG_BOUNDS (libhyena_b200_dbg.so), the kernels check the index of each
// global load and store against the extent their arguments give that buffer.  The first index
// out of range is recorded in a device record of the source file (source line, index, extent)
// and the access is skipped: a store is dropped, a load reads element 0 instead.  There is no
// trap and no fault; the host reads and clears the records with hyena_debug_bounds_check().
// In the release build both macros are the plain index (no code).
#ifdef HYENA_DEBUG_BOUNDS
static __device__ unsigned long long g_hb_rec[4];   // one record per source file (internal linkage)
__device__ __forceinline__ bool hb_ok(long long i, long long n, int line) {
    if (i >= 0 && i < n) return true;
    if (atomicCAS(&g_hb_rec[0], 0ull, 1ull) == 0ull) {
        g_hb_rec[1] = (unsigned long long)line;
        g_hb_rec[2] = (unsigned long long)i;
        g_hb_rec[3] = (unsigned long long)n;
    }
    return false;
}
#define HB_OK(i, n) (::hyena::hb_ok((long long)(i), (long long)(n), __LINE__))
#define HB_IDX(i, n) (HB_OK(i, n) ? (i) : 0)
// reads and clears this file's record: 1 and rec = {1, line, index, extent} if an access was
// out of range, 0 if none, -1 if the record could not be read
#define HYENA_BOUNDS_READER(NAME)                                                              \
    int bounds_read_##NAME(long long *rec) {                                                   \
        unsigned long long r[4] = {0, 0, 0, 0}, z[4] = {0, 0, 0, 0};                           \
        if (cudaMemcpyFromSymbol(r, g_hb_rec, sizeof(r)) != cudaSuccess) return -1;            \
        if (cudaMemcpyToSymbol(g_hb_rec, z, sizeof(z)) != cudaSuccess) return -1;              \
        for (int i = 0; i < 4; ++i) rec[i] = (long long)r[i];                                  \
        return r[0] != 0;                                                                      \
    }
#else
#define HB_OK(i, n) true
#define HB_IDX(i, n) (i)
#define HYENA_BOUNDS_READER(NAME)                                                              \
    int bounds_read_##NAME(long long *rec) {                                                   \
        for (int i = 0; i < 4; ++i) rec[i] = 0;                                                \
        return 0;                                                                              \
    }
#endif
#ifdef HYENA_DEBUG_BOUNDS
constexpr bool kBoundsChecked = true;
#else
constexpr bool kBoundsChecked = false;
#endif

// ---------------------------------------------------------------- activations
// Activation element types.  Loads widen to fp32; stores round to nearest-even.
struct ActF32 {
    using T = float;
    static constexpr int bytes = 4;
    __device__ __forceinline__ static float ld(const T *p) { return __ldg(p); }
    __device__ __forceinline__ static void st(T *p, float x) { *p = x; }
    // two consecutive channels
    __device__ __forceinline__ static float2 ld2(const T *p) {
        return __ldg(reinterpret_cast<const float2 *>(p));
    }
    __device__ __forceinline__ static void st2(T *p, float a, float b) {
        *reinterpret_cast<float2 *>(p) = make_float2(a, b);
    }
};

struct ActBF16 {
    using T = __nv_bfloat16;
    static constexpr int bytes = 2;
    __device__ __forceinline__ static float ld(const T *p) { return __bfloat162float(*p); }
    __device__ __forceinline__ static void st(T *p, float x) { *p = __float2bfloat16_rn(x); }
    __device__ __forceinline__ static float2 ld2(const T *p) {
        unsigned int w = __ldg(reinterpret_cast<const unsigned int *>(p));
        // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    __device__ __forceinline__ static void st2(T *p, float a, float b) {
        __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        *reinterpret_cast<__nv_bfloat162 *>(p) = v;
    }
};

// ---------------------------------------------------------------- complex fp32
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
__device__ __forceinline__ float2 cmulc(float2 a, float2 b) {  // a * conj(b)
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cscale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }

// ---------------------------------------------------------------- complex fp64
struct cd { double x, y; };
__device__ __forceinline__ cd cdmul(cd a, cd b) {
    return cd{fma(a.x, b.x, -a.y * b.y), fma(a.x, b.y, a.y * b.x)};
}
// lambda^m by binary powering in fp64 (m >= 0; lambda^0 = 1 also for lambda = 0).
__device__ __forceinline__ cd cdpow(cd lam, long long m) {
    cd r{1.0, 0.0};
    cd b = lam;
    while (m > 0) {
        if (m & 1) r = cdmul(r, b);
        b = cdmul(b, b);
        m >>= 1;
    }
    return r;
}

// Number of trailing prompt tokens that the prompt -> state reduction needs:
// with r = max_n |lambda_n| < 1, the tokens older than M contribute at most
// max|u| * r^M / (1 - r) <= 2^-40 max|u| to any state entry (a geometric tail
// far below fp32 resolution), so only the last M tokens are summed.
// r == 0 gives M = 1 (lambda^0 = 1 is the only nonzero power); r >= 1 (outside
// the stated |lambda| < 1 precondition) keeps the whole prompt.
__device__ __forceinline__ int state_window(const float2 *lam_head, int d, int L) {
    float r2 = 0.f;
    for (int n = 0; n < d; ++n) {
        const float2 l = lam_head[n];
        r2 = fmaxf(r2, l.x * l.x + l.y * l.y);
    }
    if (r2 == 0.f) return L < 1 ? L : 1;
    if (r2 >= 1.f) return L;
    const double r = sqrt((double)r2);
    const double m = (-40.0 * 0.69314718055994530942 + log1p(-r)) / log(r);
    if (!(m < (double)L)) return L;
    return (int)ceil(m) + 1;
}

}  // namespace hyena
