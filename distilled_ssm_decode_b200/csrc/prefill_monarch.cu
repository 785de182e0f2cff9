// prefill_monarch.cu -- the FFT route on the tensor cores, for bf16 activations.
//
// The long convolution y = q * (h conv (k v)) is evaluated by a zero-padded FFT, as the
// Hyena operator does to avoid its full Toeplitz matrix ("Hyena processes long sequences 100x
// faster than FlashAttention", lequren.com, section "Hyena層次結構").  Here every DFT of the
// convolution is cast as a dense matrix product (a Monarch-style factorisation), issued as
// tcgen05 MMAs from shared memory into tensor memory; the twiddles, the spectral product and
// the gates run on the CUDA cores between the products.
//
// Factorisation (written for this library).  N = 4096 R3 = 64 x 64 x R3 with R3 in {1, 2, 4};
// time t = 64 R3 n1 + R3 n2 + n3 and frequency k = k1 + 64 k2 + 4096 k3.  Then
//   w_N^(t k) = w_64^(n1 k1) . w_N^((R3 n2 + n3) k1) . w_64^(n2 k2) . w_(64 R3)^(n3 k2) . w_R3^(n3 k3)
// so the forward transform is
//   stage A  64-point DFTs over n1                  (product, K halved: t < N/2 is the input)
//   T1       twiddle w_N^((R3 n2 + n3) k1)          (registers)
//   stage B  64-point DFTs over n2                  (product)
//   T2       twiddle w_(64R3)^(n3 k2), R3-point DFT over n3, times the filter spectrum, and
//            back: the inverse R3-point DFT and the conjugate twiddle (registers)
// and the inverse transform runs stage B and stage A again, with T3 (twiddle) between them and
// T4 (gate-out staging) after.  The inverse uses conj(F conj(x)), so ONE real matrix serves
// all four products: the 64-point DFT F in real-stacked form, 128 x 128 bf16,
//   [Re y; Im y] = [[Re F, -Im F], [Im F, Re F]] [Re x; Im x],
// and the conjugations fold into the register steps (T2 writes conj(Z); T3 multiplies by
// w_N^(+e), which is conj(conj(W) w_N^(-e)); T4 takes conj of the last product).
//
// Layouts.  A product D[m][col] = sum_kk A[m][kk] B[kk][col] has M = 128 rows (64 outputs x
// {Re, Im}: row 2 k + c, so the two parts of one value sit in adjacent lanes of one warp and
// meet by one shuffle), K = 128 (64 inputs x {Re, Im}: K-row kappa(n, c) = 8 (n/4) + 4 c + n%4,
// which keeps the Re and Im rows written by one warp on different banks) and N = 64 R3 batch
// columns.  A (the DFT matrix) is K-major without swizzle; every B operand is MN-major with the
// 128-byte swizzle (atoms of 64 columns x 8 K-rows) and is written by the threads; D lives in
// tensor memory (lane = row, column = batch column).  Between products each thread owns one
// row: it reads its 64 R3 columns with tcgen05.ld, exchanges the other part with its partner
// lane, applies its step, and writes the next product's B operand (T1, T3: R3 adjacent
// columns of 64 K-rows; T2: its whole K-row with 16-byte stores).
//
// Work split.  One CTA holds P channel pairs (x = u_a + i u_b, both channels of one head),
// one warpgroup per pair; the pairs' G = 2P channels are adjacent, so the gate-in and gate-out
// move G * 2 bytes per token row (16 bytes for P = 4) in a CTA-wide pass.  Each warpgroup
// then runs its pair through the four products on its own barrier, so the products of one
// pair overlap the register steps of the others.  The CTA is persistent over (batch, channel
// group) units.  The prompt -> state reduction s_n = sum_j lambda_n^(L-1-j) u_j (the recurrent
// state the Laughing Hyena decode continues from; "Laughing Hyena Distillery", nubint.ai
// review, "Main findings") runs per warpgroup over the last W tokens (state_window) while its
// first product is in flight: Horner per segment, segments scaled by lambda^(L - end) in fp64
// and summed by a lane-tree.  u is exact fp32 for the last kUWin tokens, bf16 before that
// (terms older than kUWin tokens weigh |lambda|^kUWin or less).
//
// Arithmetic: bf16 operands (u, the DFT matrix, the three intermediate operands), fp32
// accumulation and fp32 register steps; y is rounded to bf16 once.
#include "common.cuh"
#include "fft.cuh"
#include "kernels.h"
#include "tc.cuh"

#include <atomic>

namespace hyena {

namespace {

std::atomic<int> g_tensor_core_fft{1};   // 0: the FFT route stays on the CUDA cores

__host__ __device__ constexpr int kappa(int n, int c) { return 8 * (n >> 2) + 4 * c + (n & 3); }

template <int R3>
struct Mon {
    static constexpr int N = 4096 * R3;
    static constexpr int C = 64 * R3;            // batch columns of every product
    static constexpr int P = (R3 == 4) ? 2 : 4;  // channel pairs per CTA (one warpgroup each)
    static constexpr int G = 2 * P;              // channels per CTA
    static constexpr int kThreads = 128 * P;
    static constexpr int kAtom = 128 * 128;      // 64 columns x 128 K-rows, 128-byte swizzled
    static constexpr int kBop = (C / 64) * kAtom;
    static constexpr int kUWin = 1024;           // trailing tokens whose u is kept in fp32
    static constexpr int kSmA = 0;               // 128 x 128 bf16 DFT matrix (core matrices)
    static constexpr int kSmB = 128 * 128 * 2;   // P B operands (also the gate-out staging)
    static constexpr int kSmU = kSmB + P * kBop; // [G][kUWin] fp32
    static constexpr int kSmBar = kSmU + G * kUWin * 4;
    static constexpr int kSmBytes = kSmBar + 64;   // P barriers, tensor-memory slot, abort, P windows
    static_assert(8 * P + 8 + 4 * P <= 64, "control block");
    static constexpr int kTmemCols = P * C;
    static_assert(kTmemCols == 256 || kTmemCols == 512, "tensor memory allocation");
    static_assert(kSmB % 1024 == 0 && kBop % 1024 == 0, "swizzle atoms are 1024-byte aligned");
};

template <int G> struct Row;
template <> struct Row<8> { using T = uint4; };
template <> struct Row<4> { using T = uint2; };

// channel i of a row of bf16 words, widened exactly to fp32
template <class T>
__device__ __forceinline__ float chan(const T &w, int i) {
    const uint32_t *u = reinterpret_cast<const uint32_t *>(&w);
    const uint32_t x = u[i >> 1];
    return __uint_as_float((i & 1) ? (x & 0xffff0000u) : (x << 16));
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
// byte offset of bf16 element (K-row, column) in a B operand (MN-major, 128-byte swizzle)
__device__ __forceinline__ uint32_t bop_off(int row, int col) {
    return (uint32_t)((col >> 6) * (128 * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
}
// byte offset of bf16 element (row, k) of the 128 x 128 DFT matrix (K-major core matrices)
__device__ __forceinline__ uint32_t amat_off(int row, int k) {
    return (uint32_t)((k >> 3) * 128 + (row >> 3) * 2048 + (row & 7) * 16 + (k & 7) * 2);
}
// byte offset of fp32 staging element (channel c of the pair, token t) in the gate-out staging
// (two planes of N/2 floats; rows of C tokens; 16-byte chunks XOR-ed by ((n1 % 4) * 2 + c))
template <int R3>
__device__ __forceinline__ uint32_t ystage_off(int c, int t) {
    constexpr int C = 64 * R3, N = 4096 * R3;
    const int n1 = t / C, j = t % C;
    const int key = ((n1 & 3) << 1) | c;
    return (uint32_t)(c * (N / 2) * 4 + n1 * C * 4 + ((((j >> 2) ^ key)) << 4) + (j & 3) * 4);
}

template <int R, bool INV>
__device__ __forceinline__ void small_dft(float2 *x) {
    if constexpr (R == 2) fft::dft2<INV>(x[0], x[1]);
    else if constexpr (R == 4) fft::dft4<INV>(x[0], x[1], x[2], x[3]);
}

// Trailing prompt tokens the state needs, from r2 = max_n |lambda_n|^2 of a head (the rule of
// state_window: the older tokens weigh at most 2^-40 max|u|).
__device__ __forceinline__ int window_of(float r2, int L) {
    if (r2 == 0.f) return L < 1 ? L : 1;
    if (r2 >= 1.f) return L;
    const double r = sqrt((double)r2);
    const double m = (-40.0 * 0.69314718055994530942 + log1p(-r)) / log(r);
    if (!(m < (double)L)) return L;
    return (int)ceil(m) + 1;
}

__device__ __forceinline__ void wg_sync(int p) {
    asm volatile("bar.sync %0, 128;" ::"r"(p + 1) : "memory");
}

template <int R3>
__global__ void __launch_bounds__(Mon<R3>::kThreads, 1)
prefill_monarch_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                       const __nv_bfloat16 *__restrict__ v, __nv_bfloat16 *__restrict__ y,
                       int B, int L, int Dch, int ch, int d, const float2 *__restrict__ spec,
                       const float2 *__restrict__ lam, float *__restrict__ state_out, int *err) {
    using M = Mon<R3>;
    constexpr int N = M::N, C = M::C, P = M::P, G = M::G;
    using RowT = typename Row<G>::T;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sp + M::kSmBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sp + M::kSmBar + 8 * P);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sp + M::kSmBar + 8 * P + 4);
    int *wwin = reinterpret_cast<int *>(sp + M::kSmBar + 8 * P + 8);     // [P] state windows
    float *us = reinterpret_cast<float *>(sp + M::kSmU);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p = warp >> 2, qd = warp & 3;      // pair (warpgroup) and tensor-memory lane quadrant
    const int r = 32 * qd + lane;                // this thread's product row = tensor-memory lane
    const int c = r & 1;                         // Re (0) or Im (1) part of the row
    const uint32_t bar_p = tc::smem_u32(&bars[p]);
    uint8_t *bop = sp + M::kSmB + p * M::kBop;
    const uint32_t bop_s = sbase + M::kSmB + p * M::kBop;
    const int H = Dch / ch;
    (void)H;

    if (tid == 0) {
        for (int i = 0; i < P; ++i) tc::mbar_init(tc::smem_u32(&bars[i]), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_u32(tmem_slot), M::kTmemCols);
        tc::tmem_relinquish();
    }
    // the real-stacked 64-point DFT matrix: F = cos - i sin of 2 pi (k n mod 64) / 64
    for (int e = tid; e < 128 * 128; e += blockDim.x) {
        const int row = e >> 7, kk = e & 127;
        const int kf = row >> 1, co = row & 1;
        const int n = 4 * (kk >> 3) + (kk & 3), ci = (kk >> 2) & 1;
        float s, cs;
        sincospif((float)((kf * n) & 63) / 32.0f, &s, &cs);
        const float val = co == 0 ? (ci == 0 ? cs : s) : (ci == 0 ? -s : cs);
        *reinterpret_cast<__nv_bfloat16 *>(sp + M::kSmA + amat_off(row, kk)) = __float2bfloat16_rn(val);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t dcol = tmem + p * C;                         // this pair's product columns
    const uint32_t trow = tmem + ((uint32_t)(32 * qd) << 16) + p * C;
    const bool issuer = (qd == 0 && lane == 0);
    uint32_t ph = 0;
    bool ok = true;

    auto issue = [&](int nks) {
        tc::tc_fence_after();
        if (ok) {
            const uint32_t idesc = tc::idesc_bf16(128, C, true);
#pragma unroll 1
            for (int ks = 0; ks < nks; ++ks) {
                const uint64_t ad = tc::smem_desc(sbase + M::kSmA + ks * 256, 128, 2048);
                const uint64_t bd = tc::smem_desc_sw128(bop_s + ks * 2048, M::kAtom, 1024);
                tc::mma_bf16(dcol, ad, bd, idesc, ks > 0);
            }
            tc::mma_commit(bar_p);
        }
    };
    auto wait_product = [&]() {
        if (ok && !tc::mbar_wait(bar_p, ph, abort_flag)) {
            ok = false;
            *abort_flag = 1;
            atomicCAS(err, 0, 1);
        }
        ph ^= 1;
        tc::tc_fence_after();
    };
    // end of a register step: loads done, operand visible to the tensor core, then the warpgroup
    // barrier, after which the issuer starts the next product
    auto step_done = [&]() {
        tc::tmem_wait_ld();
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        wg_sync(p);
    };

    const int ngc = Dch / G;
    const long long ngroups = (long long)B * ngc;
    const long long n_act = (long long)B * L * Dch;
    (void)n_act;
    const int Wf = L < M::kUWin ? L : M::kUWin;      // tokens [L - Wf, L) keep u in fp32
    for (long long grp = blockIdx.x; grp < ngroups; grp += gridDim.x) {
        const int b = (int)(grp / ngc), c0 = (int)(grp % ngc) * G;

        // ---- 1. gate-in (CTA-wide): u = k v for the G channels, rows of 8 tokens per thread
        //      (each row is G * 2 bytes of a token's channels: loaded through L2 only)
        for (int it = tid; it < N / 16; it += blockDim.x) {
            const int t0 = it * 8;
            RowT kr[8], vr[8];
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const int t = t0 + s;
                const long long o = ((long long)b * L + t) * Dch + c0;
                if (t < L && HB_OK(o + G - 1, n_act)) {
                    kr[s] = __ldcg(reinterpret_cast<const RowT *>(k + o));
                    vr[s] = __ldcg(reinterpret_cast<const RowT *>(v + o));
                } else {
                    kr[s] = RowT{};
                    vr[s] = RowT{};
                }
            }
            const int n1 = t0 / C, j0 = t0 % C;
#pragma unroll
            for (int chl = 0; chl < G; ++chl) {
                float u[8];
#pragma unroll
                for (int s = 0; s < 8; ++s) u[s] = chan(kr[s], chl) * chan(vr[s], chl);
                if (t0 + 8 > L - Wf && t0 < L) {
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const int t = t0 + s;
                        if (t >= L - Wf && t < L) us[chl * M::kUWin + (t - (L - Wf))] = u[s];
                    }
                }
                const int row = kappa(n1, chl & 1);
                uint4 pk = make_uint4(pack2(u[0], u[1]), pack2(u[2], u[3]), pack2(u[4], u[5]), pack2(u[6], u[7]));
                *reinterpret_cast<uint4 *>(sp + M::kSmB + (chl >> 1) * M::kBop + bop_off(row, j0)) = pk;
            }
        }
        // the state window of each pair's head (the rule of state_window), one warp per pair
        if (warp < P) {
            const float2 *lw = lam + (size_t)HB_IDX((c0 + 2 * warp) / ch, H) * d;
            float r2 = 0.f;
            for (int n = lane; n < d; n += 32) {
                const float2 l = __ldg(&lw[n]);
                r2 = fmaxf(r2, l.x * l.x + l.y * l.y);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) r2 = fmaxf(r2, __shfl_xor_sync(0xffffffffu, r2, off));
            if (lane == 0) wwin[warp] = window_of(r2, L);
        }
        tc::fence_proxy_async_smem();
        __syncthreads();

        // ---- 2. this warpgroup's pair through the four products
        const int cp = c0 + 2 * p;                    // first channel of the pair
        const int hd = cp / ch;
        if (issuer) issue(4);                         // stage A: K-rows of n1 < 32 (t < N/2)

        // prompt -> state reduction for the pair while the product runs
        {
            const float2 *lh = lam + (size_t)HB_IDX(hd, H) * d;
            const int W = wwin[p];
            const int jstart = L - W;
            int nseg = 1;
            while (nseg * 2 * 2 * d <= 128 && nseg < 32) nseg *= 2;
            const int wt = tid - 128 * p;
            const int g = wt % nseg, nc = wt / nseg;
            float2 acc = make_float2(0.f, 0.f);
            if (nc < 2 * d) {
                const int n = nc >> 1, cc = nc & 1;
                const float2 l = __ldg(&lh[n]);
                const int seglen = (W + nseg - 1) / nseg;
                const int j0 = jstart + g * seglen;
                const int j1 = min(L, j0 + seglen);
                auto u_at = [&](int t) -> float {
                    if (t >= L - Wf) return us[(2 * p + cc) * M::kUWin + (t - (L - Wf))];
                    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(bop + bop_off(kappa(t / C, cc), t % C)));
                };
                // Horner over blocks of 8 tokens: acc <- acc lambda^8 + sum_i lambda^(7-i) u(t+i)
                float2 lp[8];
                lp[0] = make_float2(1.f, 0.f);
#pragma unroll
                for (int i = 1; i < 8; ++i) lp[i] = cmul(lp[i - 1], l);
                const float2 l8 = cmul(lp[7], l);
                float2 aa = make_float2(0.f, 0.f);
                const int cnt = j1 > j0 ? j1 - j0 : 0;   // the last segments can be empty
                int t = j0;
                for (; t < j0 + (cnt & 7); ++t) {
                    const float x = u_at(t);
                    aa = make_float2(fmaf(aa.x, l.x, fmaf(-aa.y, l.y, x)), fmaf(aa.x, l.y, aa.y * l.x));
                }
                if (t >= L - Wf) {
                    // the whole rest of the segment has fp32 u: straight reads, no per-token test
                    const float *ur = us + (2 * p + cc) * M::kUWin + (t - (L - Wf));
                    for (; t < j0 + cnt; t += 8, ur += 8) {
                        float x[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) x[i] = ur[i];
                        float bx = 0.f, by = 0.f;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            bx = fmaf(lp[7 - i].x, x[i], bx);
                            by = fmaf(lp[7 - i].y, x[i], by);
                        }
                        aa = make_float2(fmaf(aa.x, l8.x, fmaf(-aa.y, l8.y, bx)), fmaf(aa.x, l8.y, fmaf(aa.y, l8.x, by)));
                    }
                }
                for (; t < j0 + cnt; t += 8) {
                    float bx = 0.f, by = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float x = u_at(t + i);
                        bx = fmaf(lp[7 - i].x, x, bx);
                        by = fmaf(lp[7 - i].y, x, by);
                    }
                    aa = make_float2(fmaf(aa.x, l8.x, fmaf(-aa.y, l8.y, bx)), fmaf(aa.x, l8.y, fmaf(aa.y, l8.x, by)));
                }
                if (j1 > j0) {
                    const cd pw = cdpow(cd{l.x, l.y}, (long long)(L - j1));
                    aa = cmul(aa, make_float2((float)pw.x, (float)pw.y));
                }
                acc = aa;
            }
            for (int off = nseg / 2; off > 0; off >>= 1) {
                acc.x += __shfl_down_sync(0xffffffffu, acc.x, off, nseg);
                acc.y += __shfl_down_sync(0xffffffffu, acc.y, off, nseg);
            }
            if (nc < 2 * d && g == 0) {
                const int n = nc >> 1, cc = nc & 1;
                const long long si = (((long long)b * d + n) * Dch + cp + cc) * 2;
                if (HB_OK(si + 1, (long long)B * d * Dch * 2))
                    *reinterpret_cast<float2 *>(state_out + si) = acc;
            }
        }
        wait_product();
        wg_sync(p);                                   // the state's reads of the operand are done

        // T1: rows (k1, c), columns j = R3 n2 + n3: times w_N^(j k1); to K-row kappa(n2, c),
        //     columns R3 k1 + n3.  Lane c forms the complex products of the columns j % 2 == c
        //     (twiddle chain stepping by w_N^(2 k1)); two shuffles per column pair swap the parts.
        {
            const int k1 = r >> 1;
            const float2 st = fft::expi_neg((2 * k1) % N, N);
            const int col = R3 * k1;
#pragma unroll 1
            for (int j0 = 0; j0 < C; j0 += 32) {
                float x[32];
                tc::tmem_ld32(trow + j0, x);
                tc::tmem_wait_ld();
                float2 w = fft::expi_neg(((j0 + c) * k1) % N, N);
                float o[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float rcv = __shfl_xor_sync(0xffffffffu, c ? x[2 * i] : x[2 * i + 1], 1);
                    const float2 V = c ? make_float2(rcv, x[2 * i + 1]) : make_float2(x[2 * i], rcv);
                    const float2 z = cmul(V, w);
                    w = cmul(w, st);
                    const float back = __shfl_xor_sync(0xffffffffu, c ? z.x : z.y, 1);
                    o[2 * i] = c ? back : z.x;
                    o[2 * i + 1] = c ? z.y : back;
                }
#pragma unroll
                for (int gq = 0; gq < 32 / R3; ++gq) {
                    uint8_t *dst = bop + bop_off(kappa(j0 / R3 + gq, c), col);
                    if constexpr (R3 == 1) *reinterpret_cast<__nv_bfloat16 *>(dst) = __float2bfloat16_rn(o[gq]);
                    else if constexpr (R3 == 2) *reinterpret_cast<uint32_t *>(dst) = pack2(o[2 * gq], o[2 * gq + 1]);
                    else *reinterpret_cast<uint2 *>(dst) = make_uint2(pack2(o[4 * gq], o[4 * gq + 1]), pack2(o[4 * gq + 2], o[4 * gq + 3]));
                }
            }
        }
        // the spectrum of this row's first two T2 chunks, loaded while stage B runs: row (k2, c)
        // reads the k1 with k1 % 2 == c, 8 values per 16-column chunk as 4 float4; float4 i of
        // chunk q sits at ((q * 4 + i) * 64 + k2) * 2 + c, so a warp's loads are contiguous
        const float4 *hrow4 = reinterpret_cast<const float4 *>(spec + (size_t)HB_IDX(hd, H) * N) + r;
        float4 ha[4], hb[4];
        step_done();
        if (issuer) issue(8);                         // stage B
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ha[i] = __ldg(&hrow4[i * 128]);
            hb[i] = __ldg(&hrow4[(4 + i) * 128]);
        }
        wait_product();

        // T2: rows (k2, c), columns R3 k1 + n3: twiddle, R3-point DFT, spectrum, inverse
        //     R3-point DFT, conjugate twiddle; conj(Z) to K-row kappa(k2, c), same columns.
        //     The two lanes of a row pair split the work: lane c computes the complex chain of
        //     the k1 with k1 % 2 == c (one shuffle brings in the other part of its inputs, one
        //     more hands back the partner's part of its outputs), and loads only those k1's
        //     spectrum (8 values per 16-column chunk, contiguous across the warp), two chunks ahead.
        {
            constexpr int CW = 16, KPC = CW / R3, OWN = KPC / 2;
            static_assert(OWN * R3 == 8, "eight spectrum values per chunk");
            const int k2 = r >> 1;
            float2 tw[R3];
#pragma unroll
            for (int n3 = 0; n3 < R3; ++n3) tw[n3] = fft::expi_neg(n3 * k2, 64 * R3);
            const int row = kappa(k2, c);
#pragma unroll 1
            for (int m0 = 0; m0 < C; m0 += CW) {
                float4 h4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    h4[i] = ha[i];
                    ha[i] = hb[i];
                }
                if (m0 + 2 * CW < C) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) hb[i] = __ldg(&hrow4[(((m0 + 2 * CW) / CW) * 4 + i) * 128]);
                }
                const float2 *hc = reinterpret_cast<const float2 *>(h4);
                float x[CW];
                tc::tmem_ld16(trow + m0, x);
                tc::tmem_wait_ld();
                float o[CW];
#pragma unroll
                for (int i = 0; i < OWN; ++i) {
                    float2 V[R3];
#pragma unroll
                    for (int n3 = 0; n3 < R3; ++n3) {
                        const int je = (2 * i) * R3 + n3, jo = (2 * i + 1) * R3 + n3;
                        const float rcv = __shfl_xor_sync(0xffffffffu, c ? x[je] : x[jo], 1);
                        V[n3] = c ? make_float2(rcv, x[jo]) : make_float2(x[je], rcv);
                        if (n3) V[n3] = cmul(V[n3], tw[n3]);
                    }
                    small_dft<R3, false>(V);
#pragma unroll
                    for (int k3 = 0; k3 < R3; ++k3) V[k3] = cmul(V[k3], hc[i * R3 + k3]);
                    small_dft<R3, true>(V);
#pragma unroll
                    for (int n3 = 0; n3 < R3; ++n3) {
                        const float2 z = n3 ? cmulc(V[n3], tw[n3]) : V[n3];
                        const int je = (2 * i) * R3 + n3, jo = (2 * i + 1) * R3 + n3;
                        const float rcv = __shfl_xor_sync(0xffffffffu, c ? z.x : -z.y, 1);
                        o[je] = c ? rcv : z.x;
                        o[jo] = c ? -z.y : rcv;
                    }
                }
                uint8_t *drow = bop + (m0 >> 6) * M::kAtom + row * 128;
#pragma unroll
                for (int i = 0; i < CW / 8; ++i) {
                    const int chunk = ((m0 & 63) >> 3) + i;
                    *reinterpret_cast<uint4 *>(drow + ((chunk ^ (row & 7)) << 4)) =
                        make_uint4(pack2(o[8 * i], o[8 * i + 1]), pack2(o[8 * i + 2], o[8 * i + 3]),
                                   pack2(o[8 * i + 4], o[8 * i + 5]), pack2(o[8 * i + 6], o[8 * i + 7]));
                }
            }
        }
        step_done();
        if (issuer) issue(8);                         // stage B, inverse direction
        wait_product();

        // T3: rows (n2, c), columns R3 k1 + n3: times w_N^((R3 n2 + n3) k1); to K-row
        //     kappa(k1, c), columns R3 n2 + n3.  Lane c forms the complex products of the columns
        //     m % 2 == c, as in T1 (chains per n3 residue: one, or two for R3 = 4).
        {
            const int n2 = r >> 1;
            constexpr int NCH = (R3 == 4) ? 2 : 1;
            constexpr int KSTEP = (R3 == 1) ? 2 : 1;       // k1 advance of a chain per use
            float2 st[NCH];
            int ex[NCH];                                    // R3 n2 + n3 of each chain
#pragma unroll
            for (int q2 = 0; q2 < NCH; ++q2) {
                const int n3q = (R3 == 1) ? 0 : c + 2 * q2;
                ex[q2] = R3 * n2 + n3q;
                st[q2] = fft::expi_neg((ex[q2] * KSTEP) % N, N);
            }
            const int col = R3 * n2;
#pragma unroll 1
            for (int m0 = 0; m0 < C; m0 += 32) {
                float x[32];
                tc::tmem_ld32(trow + m0, x);
                tc::tmem_wait_ld();
                const int k10 = m0 / R3;
                const int k1f = (R3 == 1) ? m0 + c : k10;      // first k1 of each chain in the chunk
                float2 w[NCH];
#pragma unroll
                for (int q2 = 0; q2 < NCH; ++q2) w[q2] = fft::expi_neg((ex[q2] * k1f) % N, N);
                float o[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int q2 = (R3 == 4) ? (i & 1) : 0;
                    const float rcv = __shfl_xor_sync(0xffffffffu, c ? x[2 * i] : x[2 * i + 1], 1);
                    const float2 V = c ? make_float2(rcv, x[2 * i + 1]) : make_float2(x[2 * i], rcv);
                    const float2 z = cmul(V, w[q2]);
                    w[q2] = cmul(w[q2], st[q2]);
                    const float back = __shfl_xor_sync(0xffffffffu, c ? z.x : z.y, 1);
                    o[2 * i] = c ? back : z.x;
                    o[2 * i + 1] = c ? z.y : back;
                }
#pragma unroll
                for (int gq = 0; gq < 32 / R3; ++gq) {
                    uint8_t *dst = bop + bop_off(kappa(k10 + gq, c), col);
                    if constexpr (R3 == 1) *reinterpret_cast<__nv_bfloat16 *>(dst) = __float2bfloat16_rn(o[gq]);
                    else if constexpr (R3 == 2) *reinterpret_cast<uint32_t *>(dst) = pack2(o[2 * gq], o[2 * gq + 1]);
                    else *reinterpret_cast<uint2 *>(dst) = make_uint2(pack2(o[4 * gq], o[4 * gq + 1]), pack2(o[4 * gq + 2], o[4 * gq + 3]));
                }
            }
        }
        step_done();
        if (issuer) issue(8);                         // stage A, inverse direction
        wait_product();

        // T4: rows (n1, c), n1 < 32, columns j: y_c(t = C n1 + j) = conj of the product, staged
        //     in fp32 over the (now free) operand
        if (qd < 2) {
            const int n1 = r >> 1;
            const float sg = c ? -1.f : 1.f;
#pragma unroll 1
            for (int j0 = 0; j0 < C; j0 += 32) {
                float x[32];
                tc::tmem_ld32(trow + j0, x);
                tc::tmem_wait_ld();
                if (C * n1 < L) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        *reinterpret_cast<float4 *>(bop + ystage_off<R3>(c, C * n1 + j0 + 4 * i)) =
                            make_float4(sg * x[4 * i], sg * x[4 * i + 1], sg * x[4 * i + 2], sg * x[4 * i + 3]);
                }
            }
        }
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncthreads();

        // ---- 3. gate-out (CTA-wide): y = q * conv for the G channels, rows of 8 tokens per thread
        for (int it = tid; it < N / 16; it += blockDim.x) {
            const int t0 = it * 8;
            if (t0 >= L) continue;
            RowT qr[8];
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const long long o = ((long long)b * L + t0 + s) * Dch + c0;
                qr[s] = (t0 + s < L && HB_OK(o + G - 1, n_act)) ? __ldcg(reinterpret_cast<const RowT *>(q + o)) : RowT{};
            }
            float yv[G][8];
#pragma unroll
            for (int chl = 0; chl < G; ++chl) {
                const uint8_t *pb = sp + M::kSmB + (chl >> 1) * M::kBop;
                const float4 a0 = *reinterpret_cast<const float4 *>(pb + ystage_off<R3>(chl & 1, t0));
                const float4 a1 = *reinterpret_cast<const float4 *>(pb + ystage_off<R3>(chl & 1, t0 + 4));
                const float zz[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                for (int s = 0; s < 8; ++s) yv[chl][s] = chan(qr[s], chl) * zz[s];
            }
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const long long o = ((long long)b * L + t0 + s) * Dch + c0;
                if (t0 + s < L && HB_OK(o + G - 1, n_act)) {
                    RowT w;
                    uint32_t *wp = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                    for (int i = 0; i < G / 2; ++i) wp[i] = pack2(yv[2 * i][s], yv[2 * i + 1][s]);
                    *reinterpret_cast<RowT *>(y + o) = w;
                }
            }
        }
        __syncthreads();
        if (*abort_flag) break;                       // uniform: set only before the barrier above
    }
    tc::tc_fence_after();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, M::kTmemCols);
}

// ------------------------------------------------------------------ four-step inner rows
// The inner 8192-point transforms of the four-step route (transforms longer than 16384 points,
// bf16 activations) on the tensor cores: each row of the complex plane Y (one column and one
// residue k1 of the outer factor) goes through the same 64 x 64 x 2 factorisation and products
// as prefill_monarch_kernel -- forward, times the row's spectrum, inverse -- and back in place.
// The rows are contiguous complex fp32, so every warpgroup loads and stores its own row with
// coalesced 16-byte accesses and the four warpgroups of a CTA run independently (no CTA-wide
// step inside the loop).  Stage A takes the full K (the row has no zero half); the output is
// staged in two halves of 64 columns through the free operand buffer.
__global__ void __launch_bounds__(512, 1)
fourstep_inner_tc_kernel(float2 *__restrict__ Y, int N1, int ncols, int nslots, int paired, int ch,
                         int H, const float2 *__restrict__ specm, int *err) {
    using M = Mon<2>;
    constexpr int N2 = M::N, C = M::C, P = M::P, R3 = 2;
    constexpr int kSmBarI = M::kSmB + P * M::kBop;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sp + kSmBarI);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sp + kSmBarI + 8 * P);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sp + kSmBarI + 8 * P + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p = warp >> 2, qd = warp & 3, r = 32 * qd + lane, c = r & 1, wt = tid - 128 * p;
    const uint32_t bar_p = tc::smem_u32(&bars[p]);
    uint8_t *bop = sp + M::kSmB + p * M::kBop;
    const uint32_t bop_s = sbase + M::kSmB + p * M::kBop;
    const long long rows = (long long)ncols * N1;
    const long long n_y = rows * N2;
    (void)n_y; (void)H;

    if (tid == 0) {
        for (int i = 0; i < P; ++i) tc::mbar_init(tc::smem_u32(&bars[i]), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_u32(tmem_slot), M::kTmemCols);
        tc::tmem_relinquish();
    }
    for (int e = tid; e < 128 * 128; e += blockDim.x) {
        const int row = e >> 7, kk = e & 127;
        const int kf = row >> 1, co = row & 1;
        const int n = 4 * (kk >> 3) + (kk & 3), ci = (kk >> 2) & 1;
        float s, cs;
        sincospif((float)((kf * n) & 63) / 32.0f, &s, &cs);
        const float val = co == 0 ? (ci == 0 ? cs : s) : (ci == 0 ? -s : cs);
        *reinterpret_cast<__nv_bfloat16 *>(sp + M::kSmA + amat_off(row, kk)) = __float2bfloat16_rn(val);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t dcol = tmem + p * C;
    const uint32_t trow = tmem + ((uint32_t)(32 * qd) << 16) + p * C;
    const bool issuer = (qd == 0 && lane == 0);
    uint32_t ph = 0;
    bool ok = true;
    auto issue = [&](int nks) {
        tc::tc_fence_after();
        if (ok) {
            const uint32_t idesc = tc::idesc_bf16(128, C, true);
#pragma unroll 1
            for (int ks = 0; ks < nks; ++ks) {
                const uint64_t ad = tc::smem_desc(sbase + M::kSmA + ks * 256, 128, 2048);
                const uint64_t bd = tc::smem_desc_sw128(bop_s + ks * 2048, M::kAtom, 1024);
                tc::mma_bf16(dcol, ad, bd, idesc, ks > 0);
            }
            tc::mma_commit(bar_p);
        }
    };
    auto wait_product = [&]() {
        if (ok && !tc::mbar_wait(bar_p, ph, abort_flag)) {
            ok = false;
            *abort_flag = 1;
            atomicCAS(err, 0, 1);
        }
        ph ^= 1;
        tc::tc_fence_after();
    };
    auto step_done = [&]() {
        tc::tmem_wait_ld();
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        wg_sync(p);
    };

#pragma unroll 1
    for (long long rw = (long long)blockIdx.x * P + p; rw < rows; rw += (long long)gridDim.x * P) {
        const int col = (int)(rw / N1), k1o = (int)(rw % N1);
        const int slot = col % nslots;
        const int hd = (paired ? 2 * slot : slot) / ch;
        float2 *rowp = Y + rw * N2;

        // gate-in: the row (8 complex values per thread and step) as Re / Im K-rows of the operand
#pragma unroll 1
        for (int it = wt; it < N2 / 8; it += 128) {
            const int t0 = it * 8;
            float4 a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = __ldcg(reinterpret_cast<const float4 *>(rowp + HB_IDX(t0 + 2 * i, n_y - rw * N2)));
            const int n1 = t0 / C, j0 = t0 % C;
            *reinterpret_cast<uint4 *>(bop + bop_off(kappa(n1, 0), j0)) =
                make_uint4(pack2(a[0].x, a[0].z), pack2(a[1].x, a[1].z), pack2(a[2].x, a[2].z), pack2(a[3].x, a[3].z));
            *reinterpret_cast<uint4 *>(bop + bop_off(kappa(n1, 1), j0)) =
                make_uint4(pack2(a[0].y, a[0].w), pack2(a[1].y, a[1].w), pack2(a[2].y, a[2].w), pack2(a[3].y, a[3].w));
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        wg_sync(p);
        if (issuer) issue(8);                         // stage A (full K)
        wait_product();

        // T1 (as in prefill_monarch_kernel)
        {
            const int k1 = r >> 1;
            const float2 st = fft::expi_neg((2 * k1) % N2, N2);
            const int colo = R3 * k1;
#pragma unroll 1
            for (int j0 = 0; j0 < C; j0 += 32) {
                float x[32];
                tc::tmem_ld32(trow + j0, x);
                tc::tmem_wait_ld();
                float2 w = fft::expi_neg(((j0 + c) * k1) % N2, N2);
                float o[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float rcv = __shfl_xor_sync(0xffffffffu, c ? x[2 * i] : x[2 * i + 1], 1);
                    const float2 V = c ? make_float2(rcv, x[2 * i + 1]) : make_float2(x[2 * i], rcv);
                    const float2 z = cmul(V, w);
                    w = cmul(w, st);
                    const float back = __shfl_xor_sync(0xffffffffu, c ? z.x : z.y, 1);
                    o[2 * i] = c ? back : z.x;
                    o[2 * i + 1] = c ? z.y : back;
                }
#pragma unroll
                for (int gq = 0; gq < 16; ++gq)
                    *reinterpret_cast<uint32_t *>(bop + bop_off(kappa(j0 / R3 + gq, c), colo)) = pack2(o[2 * gq], o[2 * gq + 1]);
            }
        }
        const float4 *hrow4 = reinterpret_cast<const float4 *>(specm + ((size_t)HB_IDX(hd, H) * N1 + k1o) * N2) + r;
        float4 ha[4], hb[4];
        step_done();
        if (issuer) issue(8);                         // stage B
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ha[i] = __ldg(&hrow4[i * 128]);
            hb[i] = __ldg(&hrow4[(4 + i) * 128]);
        }
        wait_product();

        // T2 (as in prefill_monarch_kernel, R3 = 2)
        {
            constexpr int CW = 16, OWN = 4;
            const int k2 = r >> 1;
            const float2 tw1 = fft::expi_neg(k2, 64 * R3);
            const int row = kappa(k2, c);
#pragma unroll 1
            for (int m0 = 0; m0 < C; m0 += CW) {
                float4 h4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    h4[i] = ha[i];
                    ha[i] = hb[i];
                }
                if (m0 + 2 * CW < C) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) hb[i] = __ldg(&hrow4[(((m0 + 2 * CW) / CW) * 4 + i) * 128]);
                }
                const float2 *hc = reinterpret_cast<const float2 *>(h4);
                float x[CW];
                tc::tmem_ld16(trow + m0, x);
                tc::tmem_wait_ld();
                float o[CW];
#pragma unroll
                for (int i = 0; i < OWN; ++i) {
                    float2 V[2];
#pragma unroll
                    for (int n3 = 0; n3 < 2; ++n3) {
                        const int je = (2 * i) * 2 + n3, jo = (2 * i + 1) * 2 + n3;
                        const float rcv = __shfl_xor_sync(0xffffffffu, c ? x[je] : x[jo], 1);
                        V[n3] = c ? make_float2(rcv, x[jo]) : make_float2(x[je], rcv);
                    }
                    V[1] = cmul(V[1], tw1);
                    fft::dft2<false>(V[0], V[1]);
                    V[0] = cmul(V[0], hc[i * 2]);
                    V[1] = cmul(V[1], hc[i * 2 + 1]);
                    fft::dft2<true>(V[0], V[1]);
                    V[1] = cmulc(V[1], tw1);
#pragma unroll
                    for (int n3 = 0; n3 < 2; ++n3) {
                        const float2 z = V[n3];
                        const int je = (2 * i) * 2 + n3, jo = (2 * i + 1) * 2 + n3;
                        const float rcv = __shfl_xor_sync(0xffffffffu, c ? z.x : -z.y, 1);
                        o[je] = c ? rcv : z.x;
                        o[jo] = c ? -z.y : rcv;
                    }
                }
                uint8_t *drow = bop + (m0 >> 6) * M::kAtom + row * 128;
#pragma unroll
                for (int i = 0; i < CW / 8; ++i) {
                    const int chunk = ((m0 & 63) >> 3) + i;
                    *reinterpret_cast<uint4 *>(drow + ((chunk ^ (row & 7)) << 4)) =
                        make_uint4(pack2(o[8 * i], o[8 * i + 1]), pack2(o[8 * i + 2], o[8 * i + 3]),
                                   pack2(o[8 * i + 4], o[8 * i + 5]), pack2(o[8 * i + 6], o[8 * i + 7]));
                }
            }
        }
        step_done();
        if (issuer) issue(8);                         // stage B, inverse direction
        wait_product();

        // T3 (as in prefill_monarch_kernel, R3 = 2)
        {
            const int n2 = r >> 1;
            const int ex = R3 * n2 + c;
            const float2 st = fft::expi_neg(ex % N2, N2);
            const int colo = R3 * n2;
#pragma unroll 1
            for (int m0 = 0; m0 < C; m0 += 32) {
                float x[32];
                tc::tmem_ld32(trow + m0, x);
                tc::tmem_wait_ld();
                const int k10 = m0 / R3;
                float2 w = fft::expi_neg((ex * k10) % N2, N2);
                float o[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float rcv = __shfl_xor_sync(0xffffffffu, c ? x[2 * i] : x[2 * i + 1], 1);
                    const float2 V = c ? make_float2(rcv, x[2 * i + 1]) : make_float2(x[2 * i], rcv);
                    const float2 z = cmul(V, w);
                    w = cmul(w, st);
                    const float back = __shfl_xor_sync(0xffffffffu, c ? z.x : z.y, 1);
                    o[2 * i] = c ? back : z.x;
                    o[2 * i + 1] = c ? z.y : back;
                }
#pragma unroll
                for (int gq = 0; gq < 16; ++gq)
                    *reinterpret_cast<uint32_t *>(bop + bop_off(kappa(k10 + gq, c), colo)) = pack2(o[2 * gq], o[2 * gq + 1]);
            }
        }
        step_done();
        if (issuer) issue(8);                         // stage A, inverse direction
        wait_product();

        // T4: the row out (conjugate of the product), two halves of 64 columns staged as Re / Im
        // planes [n1][64] fp32 (16-byte chunks XOR-ed by n1 % 8), then written back coalesced
        {
            const int n1 = r >> 1;
            const float sg = c ? -1.f : 1.f;
            float *plane = reinterpret_cast<float *>(bop + c * 64 * 64 * 4) + n1 * 64;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
#pragma unroll 1
                for (int j0 = 0; j0 < 64; j0 += 32) {
                    float x[32];
                    tc::tmem_ld32(trow + 64 * h + j0, x);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        *reinterpret_cast<float4 *>(plane + ((((j0 >> 2) + i) ^ (n1 & 7)) << 2)) =
                            make_float4(sg * x[4 * i], sg * x[4 * i + 1], sg * x[4 * i + 2], sg * x[4 * i + 3]);
                }
                wg_sync(p);
                const float *pr = reinterpret_cast<const float *>(bop), *pi = pr + 64 * 64;
#pragma unroll 4
                for (int e = wt; e < 64 * 32; e += 128) {
                    const int m = e >> 5, jp = (e & 31) * 2;
                    const int off = m * 64 + ((((jp >> 2)) ^ (m & 7)) << 2) + (jp & 3);
                    const float2 re = *reinterpret_cast<const float2 *>(pr + off);
                    const float2 im = *reinterpret_cast<const float2 *>(pi + off);
                    const long long t = 128LL * m + 64 * h + jp;
                    if (HB_OK(rw * N2 + t + 1, n_y))
                        *reinterpret_cast<float4 *>(rowp + t) = make_float4(re.x, im.x, re.y, im.y);
                }
                wg_sync(p);
            }
        }
        tc::tmem_wait_ld();
        tc::tc_fence_before();
    }
    tc::tc_fence_after();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, M::kTmemCols);
}

int sm_count_now() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 148;
    return n;
}

template <int R3>
cudaError_t launch_r(const void *q, const void *k, const void *v, int B, int L, int Dch, int H, int d,
                     const float2 *spec, const float2 *lam, void *y, float *state_out, int *err,
                     cudaStream_t s) {
    using M = Mon<R3>;
    const size_t smem = (size_t)M::kSmBytes + 1024;
    cudaError_t e = cudaFuncSetAttribute((const void *)prefill_monarch_kernel<R3>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long ngroups = (long long)B * (Dch / M::G);
    const long long grid = ngroups < sm_count_now() ? ngroups : sm_count_now();
    if (grid < 1) return cudaSuccess;
    prefill_monarch_kernel<R3><<<(unsigned)grid, M::kThreads, smem, s>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), static_cast<__nv_bfloat16 *>(y), B, L, Dch, Dch / H, d,
        spec, lam, state_out, err);
    return cudaGetLastError();
}

}  // namespace

HYENA_BOUNDS_READER(prefill_monarch)

void monarch_enable(int enable) { g_tensor_core_fft.store(enable ? 1 : 0); }

int monarch_r3(int dtype, int B, int L, int Dch, int H, int N, const void *q, const void *k, const void *v,
               const void *y) {
    if (!g_tensor_core_fft.load() || dtype != HYENA_BF16) return 0;
    const int r3 = (N == 4096) ? 1 : (N == 8192) ? 2 : (N == 16384) ? 4 : 0;
    if (r3 == 0 || B < 1 || L < 1 || 2LL * L > N || H < 1 || Dch % H != 0) return 0;
    const int ch = Dch / H;
    const int G = (r3 == 4) ? 4 : 8;
    if (ch % 2 != 0 || Dch % G != 0) return 0;
    const uintptr_t al = (uintptr_t)(2 * G);
    if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)y) % al != 0) return 0;
    return r3;
}

cudaError_t launch_prefill_monarch(int r3, const void *q, const void *k, const void *v, int B, int L, int Dch,
                                   int H, int d, const float2 *spec, const float2 *lam, void *y,
                                   float *state_out, int *err, cudaStream_t s) {
    switch (r3) {
        case 1: return launch_r<1>(q, k, v, B, L, Dch, H, d, spec, lam, y, state_out, err, s);
        case 2: return launch_r<2>(q, k, v, B, L, Dch, H, d, spec, lam, y, state_out, err, s);
        case 4: return launch_r<4>(q, k, v, B, L, Dch, H, d, spec, lam, y, state_out, err, s);
        default: return cudaErrorInvalidValue;
    }
}

bool fourstep_tc_enabled() { return g_tensor_core_fft.load() != 0; }

cudaError_t launch_fourstep_inner_tc(float2 *Y, int N1, int ncols, int nslots, int paired, int ch, int H,
                                     const float2 *specm, int *err, cudaStream_t s) {
    using M = Mon<2>;
    const size_t smem = (size_t)(M::kSmB + M::P * M::kBop) + 64 + 1024;
    cudaError_t e = cudaFuncSetAttribute((const void *)fourstep_inner_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)ncols * N1;
    const long long ctas = (rows + M::P - 1) / M::P;
    const long long grid = ctas < sm_count_now() ? ctas : sm_count_now();
    if (grid < 1) return cudaSuccess;
    fourstep_inner_tc_kernel<<<(unsigned)grid, 512, smem, s>>>(Y, N1, ncols, nslots, paired, ch, H, specm, err);
    return cudaGetLastError();
}

}  // namespace hyena
