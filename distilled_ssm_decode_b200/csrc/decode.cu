// decode.cu -- O(1)-per-token recurrent decode step.
//
//   y[b][c] = q (Dskip u + Re sum_n R_n s_n),   u = k v
//   s_n    <- lambda_n s_n + u
//
// The constant-time, O(d)-memory generation step of the distilled modal SSM
// ("Laughing Hyena Distillery", nubint.ai review, "Main findings": O(d) memory
// and O(dK) time for K tokens).  The output is taken from the state before the
// update, which makes prompt state + decode equal to the full convolution.
//
// Memory-bound: per (b, c) the step reads q, k, v (3 activations), reads and
// writes d complex64 state entries, and writes y.  The vector kernel gives each
// thread two adjacent channels, so one mode of the pair is one 16-byte load;
// consecutive threads take consecutive pairs, so each mode row is read as
// contiguous 128-byte lines.  A thread's modes (up to 8 at a time) are loaded
// before any arithmetic so that they are all in flight together.  When B * Dch is
// very small, NG threads share one pair (each takes every NG-th mode) and combine
// their partial outputs with warp shuffles, so that the few pairs still put
// enough loads in flight to cover memory latency.
#include "common.cuh"
#include "kernels.h"

namespace hyena {

namespace {

constexpr int kThreads = 256;

// MPT: modes held in registers per thread per iteration (all loaded before use).
template <class Act, int MPT>
__global__ void __launch_bounds__(kThreads)
decode_vec_kernel(const typename Act::T *__restrict__ q, const typename Act::T *__restrict__ k,
                  const typename Act::T *__restrict__ v, int B, int Dch, int ch, int d, int lg_ng,
                  const float2 *__restrict__ lam, const float2 *__restrict__ R,
                  const float *__restrict__ Dskip, float4 *__restrict__ state,
                  typename Act::T *__restrict__ y) {
    // launched with programmatic stream serialisation: wait until the previous kernel in the
    // stream (e.g. the previous decode step, which wrote this state) has completed, then let
    // the next one start its launch while this one runs
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int NG = 1 << lg_ng;
    const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long pair_id = gtid >> lg_ng;
    const int g = (int)(gtid & (NG - 1));
    const int pairs = Dch >> 1;
    const bool valid = pair_id < (long long)B * pairs;
    const int b = valid ? (int)(pair_id / pairs) : 0;
    const int c = valid ? 2 * (int)(pair_id % pairs) : 0;
    const int hd = c / ch;

    const size_t srow = (size_t)Dch >> 1;                    // float4 per mode row
    float4 *sp = state + (size_t)b * d * srow + (c >> 1);
    const float2 *lh = lam + (size_t)hd * d;
    const float2 *rh = R + (size_t)hd * d;

    float ua = 0.f, ub = 0.f;
    float2 qq = make_float2(0.f, 0.f);
    float acc_a = 0.f, acc_b = 0.f;
    for (int n0 = g; n0 < d; n0 += NG * MPT) {
        float4 s[MPT];
#pragma unroll
        for (int i = 0; i < MPT; ++i) {
            const int n = n0 + i * NG;
            if (valid && n < d) s[i] = sp[(size_t)n * srow];
        }
        if (n0 == g && valid) {   // activations: issued after the first state loads
            const size_t o = (size_t)b * Dch + c;
            const float2 kk = Act::ld2(k + o), vv = Act::ld2(v + o);
            qq = Act::ld2(q + o);
            ua = kk.x * vv.x;
            ub = kk.y * vv.y;
        }
#pragma unroll
        for (int i = 0; i < MPT; ++i) {
            const int n = n0 + i * NG;
            if (valid && n < d) {
                const float2 r = __ldg(&rh[n]);
                const float2 l = __ldg(&lh[n]);
                acc_a = fmaf(r.x, s[i].x, fmaf(-r.y, s[i].y, acc_a));
                acc_b = fmaf(r.x, s[i].z, fmaf(-r.y, s[i].w, acc_b));
                float4 t;
                t.x = fmaf(l.x, s[i].x, fmaf(-l.y, s[i].y, ua));
                t.y = fmaf(l.x, s[i].y, l.y * s[i].x);
                t.z = fmaf(l.x, s[i].z, fmaf(-l.y, s[i].w, ub));
                t.w = fmaf(l.x, s[i].w, l.y * s[i].z);
                sp[(size_t)n * srow] = t;
            }
        }
    }
    for (int off = NG >> 1; off > 0; off >>= 1) {
        acc_a += __shfl_xor_sync(0xffffffffu, acc_a, off);
        acc_b += __shfl_xor_sync(0xffffffffu, acc_b, off);
    }
    if (valid && g == 0) {
        const float D = __ldg(&Dskip[hd]);
        Act::st2(y + (size_t)b * Dch + c, qq.x * fmaf(D, ua, acc_a), qq.y * fmaf(D, ub, acc_b));
    }
}

// General layout (odd channels per head / odd Dch / 8-byte aligned state): one thread per channel.
template <class Act>
__global__ void __launch_bounds__(kThreads)
decode_scalar_kernel(const typename Act::T *__restrict__ q, const typename Act::T *__restrict__ k,
                     const typename Act::T *__restrict__ v, int B, int Dch, int ch, int d,
                     const float2 *__restrict__ lam, const float2 *__restrict__ R,
                     const float *__restrict__ Dskip, float2 *__restrict__ state,
                     typename Act::T *__restrict__ y) {
    const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gtid >= (long long)B * Dch) return;
    const int b = (int)(gtid / Dch), c = (int)(gtid % Dch);
    const int hd = c / ch;
    const size_t o = (size_t)b * Dch + c;
    const float u = Act::ld(k + o) * Act::ld(v + o);
    float acc = 0.f;
    float2 *sp = state + (size_t)b * d * Dch + c;
    for (int n = 0; n < d; ++n) {
        const float2 s = sp[(size_t)n * Dch];
        const float2 r = __ldg(&R[(size_t)hd * d + n]);
        const float2 l = __ldg(&lam[(size_t)hd * d + n]);
        acc = fmaf(r.x, s.x, fmaf(-r.y, s.y, acc));
        sp[(size_t)n * Dch] = make_float2(fmaf(l.x, s.x, fmaf(-l.y, s.y, u)), fmaf(l.x, s.y, l.y * s.x));
    }
    Act::st(y + o, Act::ld(q + o) * fmaf(__ldg(&Dskip[hd]), u, acc));
}

// Lanes per channel pair (NG = 2^lg) and modes per thread (MPT), from a sweep on B200 of
// one-token steps replayed from a CUDA graph (d = 16):
//   4096 pairs:  NG = 8..16, MPT = 1 best (2.3 us); one lane per pair is 2.8x slower
//   32768 pairs: NG = 1, MPT = 4 best (3.6 us); NG = 16 is 2.3x slower
//   >= 65536:    NG = 1, MPT = 8 best (5.4 us at 65536 pairs, 44.5 us at 524288)
// Splitting a pair's modes across lanes only pays when there are too few pairs to cover
// the SMs at all.
void choose_split(long long pairs, int d, int *lg_ng, int *mpt) {
    int lg = 0, m = 8;
    if (pairs < 8192) {
        while ((1 << (lg + 1)) <= 16 && (1 << (lg + 1)) <= d) ++lg;   // up to 16 lanes, one mode each
        m = 1;
    } else if (pairs < 65536) {
        m = 4;
    }
    while (m > 1 && m / 2 >= (d + (1 << lg) - 1) >> lg) m >>= 1;     // no more slots than modes
    *lg_ng = lg;
    *mpt = m;
}

// Launch with programmatic dependent launch: in a stream (or a graph captured from one) of
// back-to-back decode steps, each step's grid is scheduled while the previous step runs; the
// kernel's griddepcontrol.wait keeps the data ordering of an ordinary stream launch.
template <class Act, int MPT>
void launch_vec(unsigned blocks, cudaStream_t s, const typename Act::T *q, const typename Act::T *k,
                const typename Act::T *v, int B, int Dch, int ch, int d, int lg, const float2 *lam,
                const float2 *R, const float *Dskip, float *state, typename Act::T *y) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, decode_vec_kernel<Act, MPT>, q, k, v, B, Dch, ch, d, lg, lam, R, Dskip,
                       reinterpret_cast<float4 *>(state), y);
}

template <class Act>
cudaError_t decode_launch(const void *q, const void *k, const void *v, int B, int Dch, int ch, int d,
                          const float2 *lam, const float2 *R, const float *Dskip, float *state,
                          void *y, cudaStream_t s) {
    using T = typename Act::T;
    const T *qq = static_cast<const T *>(q), *kk = static_cast<const T *>(k), *vv = static_cast<const T *>(v);
    T *yy = static_cast<T *>(y);
    const bool vec = (ch % 2 == 0) && (Dch % 2 == 0) &&
                     ((reinterpret_cast<uintptr_t>(state) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(y)) % (2 * Act::bytes) == 0);
    if (vec) {
        const long long pairs = (long long)B * (Dch / 2);
        int lg, mpt;
        choose_split(pairs, d, &lg, &mpt);
        const long long threads = pairs << lg;
        const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
        switch (mpt) {
            case 1: launch_vec<Act, 1>(blocks, s, qq, kk, vv, B, Dch, ch, d, lg, lam, R, Dskip, state, yy); break;
            case 2: launch_vec<Act, 2>(blocks, s, qq, kk, vv, B, Dch, ch, d, lg, lam, R, Dskip, state, yy); break;
            case 4: launch_vec<Act, 4>(blocks, s, qq, kk, vv, B, Dch, ch, d, lg, lam, R, Dskip, state, yy); break;
            default: launch_vec<Act, 8>(blocks, s, qq, kk, vv, B, Dch, ch, d, lg, lam, R, Dskip, state, yy); break;
        }
    } else {
        const long long threads = (long long)B * Dch;
        const long long blocks = (threads + kThreads - 1) / kThreads;
        decode_scalar_kernel<Act><<<(unsigned)blocks, kThreads, 0, s>>>(
            qq, kk, vv, B, Dch, ch, d, lam, R, Dskip, reinterpret_cast<float2 *>(state), yy);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_step(const void *q, const void *k, const void *v, int dtype,
                               int B, int Dch, int H, int d, const float2 *lam, const float2 *R,
                               const float *Dskip, float *state, void *y, cudaStream_t s) {
    if (B == 0 || Dch == 0) return cudaSuccess;
    const int ch = Dch / H;
    return dtype == HYENA_BF16
               ? decode_launch<ActBF16>(q, k, v, B, Dch, ch, d, lam, R, Dskip, state, y, s)
               : decode_launch<ActF32>(q, k, v, B, Dch, ch, d, lam, R, Dskip, state, y, s);
}

}  // namespace hyena
