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
// writes d complex64 state entries, and writes y.  Each thread takes two
// adjacent channels (a "pair"), so one mode of the pair is one 16-byte load.
// NG = 2^lg lanes of a warp share a pair, each taking every NG-th mode, and
// combine their partial outputs with warp shuffles; the warp's 32/NG pairs are
// consecutive, so lanes that hold the same mode read 32/NG consecutive 16-byte
// entries of one mode row (whole 128-byte lines for NG <= 4).  A thread's modes
// (up to MPT at a time) are loaded before any arithmetic so that they are all
// in flight together.  Few pairs need many lanes per pair to put enough loads
// in flight; many pairs need none.
#include "common.cuh"
#include "kernels.h"

namespace hyena {

namespace {

constexpr int kThreads = 256;      // scalar kernel
constexpr int kMaxLayers = HYENA_MAX_LAYERS;

// One decode step for the channel pairs of one layer: the thread's pair and mode slot follow
// from gtid (its index in the layer's grid).  MPT: modes held in registers per thread per
// iteration (all loaded before use).  kEarly: the mode parameters and Dskip are loaded in the
// same batch as the state instead of at their first use.  That shortens the dependent chain of a
// latency-bound step (few pairs, state in L2; measured 2.03 -> 1.78 us at 4096 pairs, 3.81 -> 3.60
// us at 32768) but costs registers that the bandwidth-bound shapes need (3-6% slower there), so
// only the launches of at most 32768 pairs use it.
template <class Act, int MPT, bool kEarly>
__device__ __forceinline__ void decode_pairs(const typename Act::T *__restrict__ q, const typename Act::T *__restrict__ k,
                                             const typename Act::T *__restrict__ v, int B, int Dch, int ch, int d,
                                             int lg_ng, const float2 *__restrict__ lam, const float2 *__restrict__ R,
                                             const float *__restrict__ Dskip, float4 *__restrict__ state,
                                             typename Act::T *__restrict__ y, long long gtid) {
    const int NG = 1 << lg_ng;
    // warp w holds pairs w * ppw .. w * ppw + ppw - 1; lane = g * ppw + (pair offset)
    const int lane = threadIdx.x & 31, ppw = 32 >> lg_ng;
    const long long pair_id = (gtid >> 5) * ppw + (lane & (ppw - 1));
    const int g = lane >> (5 - lg_ng);
    const int pairs = Dch >> 1;
    const bool valid = pair_id < (long long)B * pairs;
    const int b = valid ? (int)(pair_id / pairs) : 0;
    const int c = valid ? 2 * (int)(pair_id % pairs) : 0;
    const int hd = c / ch;

    const size_t srow = (size_t)Dch >> 1;                    // float4 per mode row
    const size_t sbase = (size_t)b * d * srow + (c >> 1);
    float4 *sp = state + sbase;
    const float2 *lh = lam + (size_t)hd * d;
    const float2 *rh = R + (size_t)hd * d;
    // extents for the bounds-checked build: state rows, activations, per-head parameters
    const long long n_state = (long long)B * d * srow, n_act = (long long)B * Dch, n_par = (long long)(Dch / ch) * d;
    (void)n_state; (void)n_act; (void)n_par;

    float ua = 0.f, ub = 0.f;
    float2 qq = make_float2(0.f, 0.f);
    float acc_a = 0.f, acc_b = 0.f;
    float D = 0.f;
    if (kEarly && valid && g == 0) D = __ldg(&Dskip[HB_IDX(hd, Dch / ch)]);
    for (int n0 = g; n0 < d; n0 += NG * MPT) {
        float4 s[MPT];
        float2 re[MPT], le[MPT];
#pragma unroll
        for (int i = 0; i < MPT; ++i) {
            const int n = n0 + i * NG;
            if (valid && n < d) s[i] = sp[HB_IDX((long long)n * srow, n_state - (long long)sbase)];
        }
        if constexpr (kEarly) {
#pragma unroll
            for (int i = 0; i < MPT; ++i) {
                const int n = n0 + i * NG;
                if (valid && n < d) {
                    re[i] = __ldg(&rh[HB_IDX(n, n_par - (long long)hd * d)]);
                    le[i] = __ldg(&lh[HB_IDX(n, n_par - (long long)hd * d)]);
                }
            }
        }
        if (n0 == g && valid) {   // activations: issued after the first state loads
            const size_t o = HB_OK((long long)b * Dch + c + 1, n_act) ? (size_t)b * Dch + c : 0;
            const float2 kk = Act::ld2(k + o), vv = Act::ld2(v + o);
            qq = Act::ld2(q + o);
            ua = kk.x * vv.x;
            ub = kk.y * vv.y;
        }
#pragma unroll
        for (int i = 0; i < MPT; ++i) {
            const int n = n0 + i * NG;
            if (valid && n < d) {
                const float2 r = kEarly ? re[i] : __ldg(&rh[HB_IDX(n, n_par - (long long)hd * d)]);
                const float2 l = kEarly ? le[i] : __ldg(&lh[HB_IDX(n, n_par - (long long)hd * d)]);
                acc_a = fmaf(r.x, s[i].x, fmaf(-r.y, s[i].y, acc_a));
                acc_b = fmaf(r.x, s[i].z, fmaf(-r.y, s[i].w, acc_b));
                float4 t;
                t.x = fmaf(l.x, s[i].x, fmaf(-l.y, s[i].y, ua));
                t.y = fmaf(l.x, s[i].y, l.y * s[i].x);
                t.z = fmaf(l.x, s[i].z, fmaf(-l.y, s[i].w, ub));
                t.w = fmaf(l.x, s[i].w, l.y * s[i].z);
                if (HB_OK((long long)sbase + (long long)n * srow, n_state)) sp[(size_t)n * srow] = t;
            }
        }
    }
    for (int off = 16; off >= ppw; off >>= 1) {     // sum over the NG lanes of the pair
        acc_a += __shfl_xor_sync(0xffffffffu, acc_a, off);
        acc_b += __shfl_xor_sync(0xffffffffu, acc_b, off);
    }
    if (valid && g == 0) {
        if (!kEarly) D = __ldg(&Dskip[HB_IDX(hd, Dch / ch)]);
        if (HB_OK((long long)b * Dch + c + 1, n_act))
            Act::st2(y + (size_t)b * Dch + c, qq.x * fmaf(D, ua, acc_a), qq.y * fmaf(D, ub, acc_b));
    }
}

// Launched with programmatic stream serialisation: wait until the previous kernel in the stream
// (e.g. the previous decode step, which wrote this state) has completed, then let the next one
// start its launch while this one runs.  Before waiting, one lane per 128-byte line of q, k, v
// asks L2 to fetch that line: a prefetch returns no data, so it is safe even while an earlier
// kernel still writes these inputs, and the loads after the wait then find them in L2.
template <class Act>
__device__ __forceinline__ void pdl_enter(const typename Act::T *q, const typename Act::T *k,
                                          const typename Act::T *v, int B, int Dch, int lg_ng, long long gtid) {
    const int lane = threadIdx.x & 31, ppw = 32 >> lg_ng;
    const long long pair_id = (gtid >> 5) * ppw + (lane & (ppw - 1));
    constexpr int kPairsPerLine = 128 / (2 * Act::bytes);
    if ((lane >> (5 - lg_ng)) == 0 && pair_id % kPairsPerLine == 0 && pair_id < (long long)B * (Dch >> 1) &&
        HB_OK(pair_id * 2 + 1, (long long)B * Dch)) {
        const size_t o = (size_t)pair_id * 2;    // element offset of the pair in [B][Dch]
        asm volatile("prefetch.global.L2 [%0];" ::"l"(q + o));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(k + o));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(v + o));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}

// NT: threads per block (128, 256 or 512), fixed at compile time so that register allocation
// and scheduling are made for the block size each launch shape uses.
template <class Act, int MPT, int NT, bool kEarly>
__global__ void __launch_bounds__(NT)
decode_vec_kernel(const typename Act::T *__restrict__ q, const typename Act::T *__restrict__ k,
                  const typename Act::T *__restrict__ v, int B, int Dch, int ch, int d, int lg_ng,
                  const float2 *__restrict__ lam, const float2 *__restrict__ R,
                  const float *__restrict__ Dskip, float4 *__restrict__ state,
                  typename Act::T *__restrict__ y) {
    const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    pdl_enter<Act>(q, k, v, B, Dch, lg_ng, gtid);
    decode_pairs<Act, MPT, kEarly>(q, k, v, B, Dch, ch, d, lg_ng, lam, R, Dskip, state, y, gtid);
}

// Several independent layers in one launch: blockIdx.y selects the layer, whose pointers travel
// by value in the kernel parameter (so a captured graph keeps them).
struct LayerPtrs {
    const void *q, *k, *v;
    void *y;
    float4 *state;
    const float2 *lam, *R;
    const float *Dskip;
};
struct LayerTable {
    LayerPtrs l[kMaxLayers];
};

template <class Act, int MPT, int NT, bool kEarly>
__global__ void __launch_bounds__(NT)
decode_layers_kernel(const __grid_constant__ LayerTable t, int B, int Dch, int ch, int d, int lg_ng) {
    using T = typename Act::T;
    const LayerPtrs &p = t.l[blockIdx.y];
    const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const T *q = static_cast<const T *>(p.q), *k = static_cast<const T *>(p.k), *v = static_cast<const T *>(p.v);
    pdl_enter<Act>(q, k, v, B, Dch, lg_ng, gtid);
    decode_pairs<Act, MPT, kEarly>(q, k, v, B, Dch, ch, d, lg_ng, p.lam, p.R, p.Dskip, p.state, static_cast<T *>(p.y), gtid);
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
    const int hd = c / ch, H = Dch / ch;
    const long long n_act = (long long)B * Dch, n_state = (long long)B * d * Dch, n_par = (long long)H * d;
    (void)n_state; (void)n_par;
    const size_t o = HB_IDX((size_t)b * Dch + c, n_act);
    const float u = Act::ld(k + o) * Act::ld(v + o);
    float acc = 0.f;
    const size_t sbase = (size_t)b * d * Dch + c;
    for (int n = 0; n < d; ++n) {
        const size_t si = HB_IDX(sbase + (size_t)n * Dch, n_state);
        const float2 s = state[si];
        const float2 r = __ldg(&R[HB_IDX((size_t)hd * d + n, n_par)]);
        const float2 l = __ldg(&lam[HB_IDX((size_t)hd * d + n, n_par)]);
        acc = fmaf(r.x, s.x, fmaf(-r.y, s.y, acc));
        if (HB_OK(sbase + (size_t)n * Dch, n_state))
            state[si] = make_float2(fmaf(l.x, s.x, fmaf(-l.y, s.y, u)), fmaf(l.x, s.y, l.y * s.x));
    }
    if (HB_OK(o, n_act)) Act::st(y + o, Act::ld(q + o) * fmaf(__ldg(&Dskip[HB_IDX(hd, H)]), u, acc));
}

// Lanes per pair (NG = 2^lg), modes per thread (MPT) and block size, from a sweep on B200 of
// one-token steps replayed from a CUDA graph (d = 16, bf16, every combination of lg 0..4,
// MPT 1..8 and 128/256/512 threads; best per size, us per step):
//      2048 pairs: NG 16, MPT 1, 256 (1.60)      4096: NG 8, MPT 2, 256 (1.82)
//      8192 pairs: NG 8,  MPT 2      (2.05)     16384: NG 4, MPT 2, 256 (2.65)
//     32768 pairs: NG 2,  MPT 2, 512 (3.35)     65536: NG 2, MPT 2, 512 (4.90)
//    131072 pairs: NG 1,  MPT 2, 512 (8.2)   >=524288: NG 1, MPT 4, 128 (43.5 at 524288,
//                                                       166.8 at 2097152 = 99% of HBM)
// Fewer modes than NG * MPT slots: NG and MPT shrink so that no slot stays empty.
void choose_split(long long pairs, int d, int *lg_ng, int *mpt, int *threads) {
    int lg, m, nt;
    if (pairs <= 2048)        { lg = 4; m = 1; nt = 256; }
    else if (pairs <= 8192)   { lg = 3; m = 2; nt = 256; }
    else if (pairs <= 16384)  { lg = 2; m = 2; nt = 256; }
    else if (pairs <= 65536)  { lg = 1; m = 2; nt = 512; }
    else if (pairs <= 131072) { lg = 0; m = 2; nt = 512; }
    else                      { lg = 0; m = 4; nt = 128; }
    while (lg > 0 && (1 << lg) > d) --lg;
    while (m > 1 && m / 2 >= (d + (1 << lg) - 1) >> lg) m >>= 1;
    *lg_ng = lg;
    *mpt = m;
    *threads = nt;
}

// Launch with programmatic dependent launch: in a stream (or a graph captured from one) of
// back-to-back decode steps, each step's grid is scheduled while the previous step runs; the
// kernel's griddepcontrol.wait keeps the data ordering of an ordinary stream launch.
template <class Act, int MPT>
void launch_vec(unsigned blocks, int threads, cudaStream_t s, const typename Act::T *q, const typename Act::T *k,
                const typename Act::T *v, int B, int Dch, int ch, int d, int lg, const float2 *lam,
                const float2 *R, const float *Dskip, float *state, typename Act::T *y) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // early parameter loads for the latency-bound shapes (at most 32768 pairs)
    const bool early = (long long)blocks * threads <= (32768ll << lg);
    auto kern = (early && threads == 256) ? decode_vec_kernel<Act, MPT, 256, true>
                : (early && threads == 512) ? decode_vec_kernel<Act, MPT, 512, true>
                : threads == 128 ? decode_vec_kernel<Act, MPT, 128, false>
                : threads == 256 ? decode_vec_kernel<Act, MPT, 256, false> : decode_vec_kernel<Act, MPT, 512, false>;
    cudaLaunchKernelEx(&cfg, kern, q, k, v, B, Dch, ch, d, lg, lam, R, Dskip, reinterpret_cast<float4 *>(state), y);
}

template <class Act, int MPT>
cudaError_t launch_layers(dim3 grid, int threads, cudaStream_t s, const LayerTable &t, int B, int Dch, int ch,
                          int d, int lg) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kern = (lg >= 2 && threads == 256) ? decode_layers_kernel<Act, MPT, 256, true>
                : threads == 128 ? decode_layers_kernel<Act, MPT, 128, false>
                : threads == 256 ? decode_layers_kernel<Act, MPT, 256, false> : decode_layers_kernel<Act, MPT, 512, false>;
    return cudaLaunchKernelEx(&cfg, kern, t, B, Dch, ch, d, lg);
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
        int lg, mpt, nt;
        choose_split(pairs, d, &lg, &mpt, &nt);
        const long long threads = pairs << lg;
        const unsigned blocks = (unsigned)((threads + nt - 1) / nt);
        switch (mpt) {
            case 1: launch_vec<Act, 1>(blocks, nt, s, qq, kk, vv, B, Dch, ch, d, lg, lam, R, Dskip, state, yy); break;
            case 2: launch_vec<Act, 2>(blocks, nt, s, qq, kk, vv, B, Dch, ch, d, lg, lam, R, Dskip, state, yy); break;
            default: launch_vec<Act, 4>(blocks, nt, s, qq, kk, vv, B, Dch, ch, d, lg, lam, R, Dskip, state, yy); break;
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

HYENA_BOUNDS_READER(decode)

cudaError_t launch_decode_step(const void *q, const void *k, const void *v, int dtype,
                               int B, int Dch, int H, int d, const float2 *lam, const float2 *R,
                               const float *Dskip, float *state, void *y, cudaStream_t s) {
    if (B == 0 || Dch == 0) return cudaSuccess;
    const int ch = Dch / H;
    return dtype == HYENA_BF16
               ? decode_launch<ActBF16>(q, k, v, B, Dch, ch, d, lam, R, Dskip, state, y, s)
               : decode_launch<ActF32>(q, k, v, B, Dch, ch, d, lam, R, Dskip, state, y, s);
}

bool decode_layers_vec_ok(int Dch, int H) { return Dch % 2 == 0 && (Dch / H) % 2 == 0; }

cudaError_t launch_decode_layers(int layers, const void *const *q, const void *const *k, const void *const *v,
                                 int dtype, int B, int Dch, int H, int d, const float *const *lam,
                                 const float *const *R, const float *const *Dskip, float *const *state,
                                 void *const *y, cudaStream_t s) {
    if (layers == 0 || B == 0 || Dch == 0) return cudaSuccess;
    LayerTable t;
    for (int i = 0; i < layers; ++i)
        t.l[i] = LayerPtrs{q[i], k[i], v[i], y[i], reinterpret_cast<float4 *>(state[i]),
                           reinterpret_cast<const float2 *>(lam[i]), reinterpret_cast<const float2 *>(R[i]), Dskip[i]};
    const long long pairs = (long long)B * (Dch / 2);
    int lg, mpt, nt;
    choose_split(pairs * layers, d, &lg, &mpt, &nt);
    const long long threads = pairs << lg;
    const dim3 grid((unsigned)((threads + nt - 1) / nt), (unsigned)layers);
    const int ch = Dch / H;
    cudaError_t e;
    if (dtype == HYENA_BF16) {
        e = mpt == 1 ? launch_layers<ActBF16, 1>(grid, nt, s, t, B, Dch, ch, d, lg)
            : mpt == 2 ? launch_layers<ActBF16, 2>(grid, nt, s, t, B, Dch, ch, d, lg)
                       : launch_layers<ActBF16, 4>(grid, nt, s, t, B, Dch, ch, d, lg);
    } else {
        e = mpt == 1 ? launch_layers<ActF32, 1>(grid, nt, s, t, B, Dch, ch, d, lg)
            : mpt == 2 ? launch_layers<ActF32, 2>(grid, nt, s, t, B, Dch, ch, d, lg)
                       : launch_layers<ActF32, 4>(grid, nt, s, t, B, Dch, ch, d, lg);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace hyena
