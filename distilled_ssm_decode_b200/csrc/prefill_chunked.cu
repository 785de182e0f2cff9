// prefill_chunked.cu -- chunked modal prefill on tcgen05 tensor cores.
//
// The long convolution y = q * (h conv (k * v)) ("Hyena processes long
// sequences 100x faster than FlashAttention", lequren.com, "Hyena層次結構")
// with the modal filter h_0 = Dskip, h_j = Re sum_n R_n lambda_n^(j-1) of
// "Laughing Hyena Distillery" (nubint.ai review, "Proposed method") is
// evaluated chunk by chunk.  For a chunk of C tokens starting at c0, with
// tau, iota in [0, C):
//
//   z[c0+tau] = sum_{iota<=tau} h_{tau-iota} u[c0+iota]            (intra-chunk Toeplitz)
//             + Re sum_n R_n lambda_n^tau s_n(c0)                  (modal carry from the past)
//   s_n(c0+C) = lambda_n^C s_n(c0) + sum_iota lambda_n^(C-1-iota) u[c0+iota]
//
// where s(c0) is the recurrent state after c0 tokens -- the same O(d) state the
// decode step advances ("Main findings": O(d) memory per channel).  This is an
// exact regrouping of the causal convolution (the carry term is the tail of the
// sum over j < c0 with h_{t-j} = Re sum R lambda^(t-c0) lambda^(c0-1-j)), and
// the prompt -> state reduction falls out as the last carry.
//
// Per chunk and 128-channel tile (one head, M = 128 = channels on the MMA
// rows), three products run on the tensor cores in tf32 with fp32 accumulation
// in tensor memory:
//   D1[c][tau] = sum_iota U[c][iota] T[tau][iota]  +  sum_r S[c][r] A[tau][r]
//   D2[c][r]   = sum_iota U[c][iota] V[r][iota]
// with T[tau][iota] = h_{tau-iota} (iota <= tau), A = (Re, -Im) of R lambda^tau,
// V = (Re, Im) of lambda^(C-1-iota), S = (Re, Im) of the state.  The chunk's
// state update S <- lambda^C S + D2 runs on the CUDA cores in fp32 registers
// (one thread per channel, the thread that owns TMEM lane c), and
// y = q * D1 is gated and stored by the same thread.
//
// Work split: a sequence is cut into segments of whole chunks; each
// (batch, channel tile, segment) item first runs a state-only pass (k, v and
// the D2 product) to publish its segment's state contribution, then obtains the
// state entering its segment by a decoupled look-back over its predecessors'
// published contributions (bounded polls), then runs the full pass.  Items are
// handed out by an atomic ticket in launch order, so an item only ever waits on
// items already running; the state-only pass never waits, so the look-back
// always ends.  k and v are read twice per item, the second time mostly from L2.
//
// Roles in a 192-thread CTA: warps 0-3 (one thread per channel) compute
// u = k*v, the state and the gated output; warp 4 issues the TMA loads; warp 5
// owns tensor memory and issues the MMAs.  Every wait is bounded; on timeout
// the kernel records an error code, drains its copies and MMAs, frees tensor
// memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace hyena {

namespace {

constexpr int kC = 32;             // tokens per chunk
constexpr int kNC = 128;           // channels per tile (MMA M)
constexpr int kMaxModes = 16;      // d <= 16
constexpr int kKSMax = 32;         // state operand width: Re at [0,16), Im at [16,32)
constexpr int kIm = 16;
constexpr int kTileBytes = kC * kNC * 2;          // one bf16 [C][128] activation tile
constexpr int kHalfBytes = kTileBytes / 2;        // [C][64] half tile = one TMA box, 128-byte swizzled
// Ring depths.  A chunk's output product needs the U operand, the state operand and a D1
// accumulator; each of those is refilled only after the product that used it completes, so a
// ring of depth n lets n chunks be in flight between those round trips.
constexpr int kKVStages = 3;                      // k,v tiles
constexpr int kQStages = 4;                       // q tiles (y staged in place)
constexpr int kUBufs = 4;                         // U operands
constexpr int kSTBufs = 4;                        // state operands
constexpr int kNAcc = 4;                          // accumulators (TMEM): [C output cols | 32 state cols]
constexpr int kAccCols = kC + kKSMax;
constexpr int kPrefetch = 8;                      // chunks of q, k, v prefetched into L2 ahead of the loads
constexpr int kThreads = 512;                     // 16 warps, see the role map below
constexpr uint32_t kTmemCols = kNAcc * kAccCols;  // 256

// constant block per head (global, laid out exactly as in shared memory).  T (Toeplitz) and
// V (chunk powers) are adjacent so that they form one B operand [T; V] of C + 32 rows: the
// fused product U [T; V]^T yields the intra-chunk output and the chunk's state contribution
// in one pass over U (an MMA costs the same for any N <= 128 on B200).
constexpr int kTTBytes = kC * kC * 4;             // rows 0..C-1 of the fused B operand
constexpr int kVTBytes = kKSMax * kC * 4;         // rows C..C+31 of the fused B operand
constexpr int kATBytes = kC * kKSMax * 4;         // B operand of the carry product
constexpr int kConstBytes = kTTBytes + kATBytes + kVTBytes + 2 * kMaxModes * 8;   // + lambda^C, lambda^Lseg
constexpr int kConstStride = (kConstBytes + 255) & ~255;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kSmTT = 0;
constexpr int kSmVT = kSmTT + kTTBytes;
constexpr int kSmAT = kSmVT + kVTBytes;
constexpr int kSmLam = kSmAT + kATBytes;                      // lambda^C, lambda^Lseg [16] each (float2)
constexpr int kSmUT = kSmLam + 1024;                          // kUBufs x [128][C] tf32
constexpr int kUTBytes = kNC * kC * 4;
constexpr int kSmST = kSmUT + kUBufs * kUTBytes;              // kSTBufs x [128][32] tf32
constexpr int kSTBytes = kNC * kKSMax * 4;
constexpr int kSmKV = kSmST + kSTBufs * kSTBytes;             // kKVStages x {k, v}
constexpr int kSmQ = kSmKV + kKVStages * 2 * kTileBytes;      // kQStages x q (y staged in place)
constexpr int kSmBar = kSmQ + kQStages * kTileBytes;

// barrier slots (arrival counts in parentheses; "commit" = tcgen05.commit from the MMA thread)
enum : int {
    kBarKVFull = 0,                              // [kKVStages] k,v tile landed (1 + tx)
    kBarKVEmpty = kBarKVFull + kKVStages,        // [kKVStages] k,v consumed (128: U group, or S group for the prompt's last chunk)
    kBarQFull = kBarKVEmpty + kKVStages,         // [kQStages] q tile landed (1 + tx)
    kBarQEmpty = kBarQFull + kQStages,           // [kQStages] q/y buffer free (1: store warp)
    kBarURdy = kBarQEmpty + kQStages,            // [kUBufs] U operand written (128: U group)
    kBarUFree = kBarURdy + kUBufs,               // [kUBufs] U operand no longer read (commit)
    kBarWDone = kBarUFree + kUBufs,              // [kNAcc] fused product done (commit)
    kBarD2Free = kBarWDone + kNAcc,              // [kNAcc] state columns read out (128: S group)
    kBarSRdy = kBarD2Free + kNAcc,               // [kSTBufs] state operand written (128: S group)
    kBarSTFree = kBarSRdy + kSTBufs,             // [kSTBufs] state operand no longer read (commit)
    kBarYDone = kBarSTFree + kSTBufs,            // [kNAcc] carry product done: output complete (commit)
    kBarD1Free = kBarYDone + kNAcc,              // [kNAcc] output columns read out (128: E group)
    kBarYStaged = kBarD1Free + kNAcc,            // [kQStages] gated tile staged for the store (128: E group)
    kBarPub = kBarYStaged + kQStages,            // segment state written to global (128: S group)
    kBarDrain = kBarPub + 1,                     // every MMA of the CTA finished (commit)
    kNumBars = kBarDrain + 1
};
constexpr int kSmMisc = kSmBar + kNumBars * 8;
constexpr int kSmemBytes = kSmMisc + 64 + 1024;               // + misc words + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

__host__ __device__ constexpr int bar_count(int i) {
    return ((i >= kBarKVEmpty && i < kBarQFull) || (i >= kBarURdy && i < kBarUFree) ||
            (i >= kBarD2Free && i < kBarSTFree) || (i >= kBarD1Free && i < kBarDrain)) ? 128 : 1;
}

// byte offset of element (row, k) in a K-major, no-swizzle core-matrix tile whose K extent is K
__host__ __device__ __forceinline__ int cm_off(int row, int k, int K) {
    return (k >> 2) * 128 + (row >> 3) * (K * 32) + (row & 7) * 16 + (k & 3) * 4;
}

// byte offset of activation (token tau, channel c) in a [C][128] bf16 tile held as two
// [C][64] halves written by TMA with 128-byte swizzling (16-byte chunk ^= row % 8)
__device__ __forceinline__ int act_off(int tau, int c) {
    return (c >> 6) * kHalfBytes + tau * 128 + ((((c & 63) >> 3) ^ (tau & 7)) << 4) + (c & 7) * 2;
}

struct ChunkArgs {
    int L, Dch, d, ch;
    int ntiles;          // channel tiles per sequence (Dch / 128)
    int nchunks;         // chunks per sequence
    int nseg, segc;      // segments per sequence, chunks per segment (all but the last)
    const float2 *lam;   // [H][d]
    const uint8_t *consts;
    float *state_out;    // [B][d][Dch][2]
    int *sched;          // [0] ticket counter, [1] error code
    int *status;         // [items]: 0 none, 1 segment contribution, 2 inclusive state
    float2 *agg;         // [items][d][128]
    float2 *inc;         // [items][d][128]
};

enum : int { kErrWait = 1, kErrLookback = 2 };

__device__ __forceinline__ void record_error(const ChunkArgs &a, volatile int *abort, int code) {
    *abort = 1;
    atomicCAS(a.sched + 1, 0, code);
}

// ------------------------------------------------------------------ per-head constants
__global__ void __launch_bounds__(256)
chunk_consts_kernel(const float2 *__restrict__ lam, const float2 *__restrict__ R,
                    const float *__restrict__ Dskip, int d, int seg_tokens,
                    uint8_t *__restrict__ consts) {
    const int hd = blockIdx.x;
    uint8_t *base = consts + (size_t)hd * kConstStride;
    float *TT = reinterpret_cast<float *>(base + kSmTT);
    float *VT = reinterpret_cast<float *>(base + kSmVT);
    float *AT = reinterpret_cast<float *>(base + kSmAT);
    float2 *lamC = reinterpret_cast<float2 *>(base + kTTBytes + kATBytes + kVTBytes);
    float2 *lamS = lamC + kMaxModes;
    __shared__ double hs[kC];
    const float2 *lh = lam + (size_t)hd * d;
    const float2 *rh = R + (size_t)hd * d;
    // filter taps h_0 .. h_{C-1} in fp64
    for (int j = threadIdx.x; j < kC; j += blockDim.x) {
        double acc = 0.0;
        if (j == 0) {
            acc = Dskip[hd];
        } else {
            for (int n = 0; n < d; ++n) {
                const cd p = cdpow(cd{lh[n].x, lh[n].y}, j - 1);
                acc += (double)rh[n].x * p.x - (double)rh[n].y * p.y;
            }
        }
        hs[j] = acc;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kC * kC; e += blockDim.x) {
        const int tau = e / kC, io = e % kC;
        const float v = io <= tau ? (float)hs[tau - io] : 0.f;
        TT[cm_off(tau, io, kC) / 4] = tc::to_tf32(v);
    }
    // columns r < 16: real parts of mode r; columns 16 + n: imaginary parts of mode n
    for (int e = threadIdx.x; e < kC * kKSMax; e += blockDim.x) {
        const int tau = e / kKSMax, r = e % kKSMax;
        const int n = r & (kIm - 1);
        float v = 0.f;
        if (n < d) {
            const cd p = cdpow(cd{lh[n].x, lh[n].y}, tau);
            const double re = (double)rh[n].x * p.x - (double)rh[n].y * p.y;
            const double im = (double)rh[n].x * p.y + (double)rh[n].y * p.x;
            v = r < kIm ? (float)re : (float)(-im);
        }
        AT[cm_off(tau, r, kKSMax) / 4] = tc::to_tf32(v);
    }
    for (int e = threadIdx.x; e < kKSMax * kC; e += blockDim.x) {
        const int r = e / kC, io = e % kC;
        const int n = r & (kIm - 1);
        float v = 0.f;
        if (n < d) {
            const cd p = cdpow(cd{lh[n].x, lh[n].y}, kC - 1 - io);
            v = r < kIm ? (float)p.x : (float)p.y;
        }
        VT[cm_off(r, io, kC) / 4] = tc::to_tf32(v);
    }
    for (int n = threadIdx.x; n < kMaxModes; n += blockDim.x) {
        cd pc{0.0, 0.0}, ps{0.0, 0.0};
        if (n < d) {
            pc = cdpow(cd{lh[n].x, lh[n].y}, kC);
            ps = cdpow(cd{lh[n].x, lh[n].y}, seg_tokens);
        }
        lamC[n] = make_float2((float)pc.x, (float)pc.y);
        lamS[n] = make_float2((float)ps.x, (float)ps.y);
    }
}


// ------------------------------------------------------------------ main kernel
// Roles (warps):  0-3  U group: u = k*v -> U operand (ldmatrix transpose), one chunk at a time
//                 4-7  S group: one thread per channel; state chain, segment publish, look-back
//                 8-11 E group: one thread per channel; gate y = q * D1, stage y for the store
//                 12   k,v TMA loads    13  q TMA loads    14  y TMA stores (lane 0 each; a
//                      warp of their own so that one role's blocking wait never holds another)
//                 15   tensor memory owner and MMA issuer (lane 0)
// The groups run their own loops over the same chunk sequence and meet only at mbarriers, so
// the U group forms chunk i+1 while the S group advances chunk i and the E group gates i-1.
__global__ void __launch_bounds__(kThreads, 1)
prefill_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_y,
                     const ChunkArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int slot) { return sbase + kSmBar + 8u * slot; };
    volatile int *misc = reinterpret_cast<volatile int *>(sm + kSmMisc);   // item, abort, tmem, never
    volatile int *abort = misc + 1;
    volatile int *never = misc + 3;

    if (tid == 0) {
        misc[0] = atomicAdd(a.sched, 1);
        misc[1] = 0;
        misc[3] = 0;
        for (int i = 0; i < kNumBars; ++i) tc::mbar_init(bar(i), bar_count(i));
        tc::fence_mbar_init();
    }
    if (warp == 15) {
        tc::tmem_alloc(tc::smem_u32((const void *)(misc + 2)), kTmemCols);
        tc::tmem_relinquish();
    }
    __syncthreads();
    const int item = misc[0];
    const int unit = item / a.nseg, seg = item % a.nseg;
    const int b = unit / a.ntiles, c0 = (unit % a.ntiles) * kNC;
    const int hd = c0 / a.ch;
    const int ck0 = seg * a.segc;
    const int nck = min(a.nchunks, ck0 + a.segc) - ck0;
    const bool last_seg = (seg == a.nseg - 1);
    const bool phase1 = !last_seg;
    const int n1 = phase1 ? nck : 0;                  // state-only iterations
    const int niter = n1 + nck;
    const int d = a.d;

    // per-head constants -> shared memory; zero the state operands (their padding columns stay 0)
    {
        const int4 *src = reinterpret_cast<const int4 *>(a.consts + (size_t)hd * kConstStride);
        int4 *dst = reinterpret_cast<int4 *>(sm);
        for (int i = tid; i < (kTTBytes + kATBytes + kVTBytes + 2 * kMaxModes * 8) / 16; i += kThreads)
            dst[i] = __ldg(src + i);      // [T; V], A and lambda^C, lambda^Lseg
        int4 *stz = reinterpret_cast<int4 *>(sm + kSmST);
        for (int i = tid; i < kSTBufs * kSTBytes / 16; i += kThreads) stz[i] = make_int4(0, 0, 0, 0);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[2];
    auto chunk_of = [&](int it) { return ck0 + (it < n1 ? it : it - n1); };
    auto uni = [&](bool x) -> bool { return __all_sync(0xffffffffu, x && !*abort); };

    if (warp >= 12 && warp <= 14) {
        // ------------------------------------------------------------ TMA warps
        if (warp == 12 && lane == 0) {      // k, v for every iteration (state-only pass, then full pass)
            // L2 prefetch runs kPrefetch chunks ahead of the loads, so that many more bytes are in
            // flight than the shared-memory stages hold (loaded DRAM latency is several us here)
            for (int it = 0; it < min(kPrefetch, n1 > 0 ? n1 : nck); ++it)
                for (int h = 0; h < 2; ++h) {
                    tc::tma_prefetch_3d(&tm_k, c0 + 64 * h, chunk_of(it) * kC, b);
                    tc::tma_prefetch_3d(&tm_v, c0 + 64 * h, chunk_of(it) * kC, b);
                }
            int it = 0;
            for (; it < niter; ++it) {
                // the full pass re-reads k, v that the state-only pass brought into L2
                const int pf = it + kPrefetch;
                if (pf < (n1 > 0 ? n1 : nck))
                    for (int h = 0; h < 2; ++h) {
                        tc::tma_prefetch_3d(&tm_k, c0 + 64 * h, chunk_of(pf) * kC, b);
                        tc::tma_prefetch_3d(&tm_v, c0 + 64 * h, chunk_of(pf) * kC, b);
                    }
                const int s = it % kKVStages;
                if (!tc::mbar_wait(bar(kBarKVEmpty + s), ((it / kKVStages) & 1) ^ 1, abort)) {
                    record_error(a, abort, kErrWait);
                    break;
                }
                const uint32_t dst = sbase + kSmKV + s * 2 * kTileBytes;
                const int t0 = chunk_of(it) * kC;
                tc::mbar_expect_tx(bar(kBarKVFull + s), 2 * kTileBytes);
                for (int h = 0; h < 2; ++h) {
                    tc::tma_load_3d(dst + h * kHalfBytes, &tm_k, bar(kBarKVFull + s), c0 + 64 * h, t0, b);
                    tc::tma_load_3d(dst + kTileBytes + h * kHalfBytes, &tm_v, bar(kBarKVFull + s), c0 + 64 * h, t0, b);
                }
            }
            if (*abort)
                for (int j = max(0, it - kKVStages); j < it; ++j)
                    tc::mbar_wait(bar(kBarKVFull + j % kKVStages), (j / kKVStages) & 1, never);
        } else if (warp == 13 && lane == 0) {   // q for the full pass (the buffer then stages y)
            for (int j = 0; j < min(kPrefetch, nck); ++j)
                for (int h = 0; h < 2; ++h) tc::tma_prefetch_3d(&tm_q, c0 + 64 * h, (ck0 + j) * kC, b);
            int j = 0;
            for (; j < nck; ++j) {
                if (j + kPrefetch < nck)
                    for (int h = 0; h < 2; ++h)
                        tc::tma_prefetch_3d(&tm_q, c0 + 64 * h, (ck0 + j + kPrefetch) * kC, b);
                const int s = j % kQStages;
                if (!tc::mbar_wait(bar(kBarQEmpty + s), ((j / kQStages) & 1) ^ 1, abort)) {
                    record_error(a, abort, kErrWait);
                    break;
                }
                tc::mbar_expect_tx(bar(kBarQFull + s), kTileBytes);
                for (int h = 0; h < 2; ++h)
                    tc::tma_load_3d(sbase + kSmQ + s * kTileBytes + h * kHalfBytes, &tm_q, bar(kBarQFull + s),
                                    c0 + 64 * h, (ck0 + j) * kC, b);
            }
            if (*abort)
                for (int jj = max(0, j - kQStages); jj < j; ++jj)
                    tc::mbar_wait(bar(kBarQFull + jj % kQStages), (jj / kQStages) & 1, never);
        } else if (warp == 14 && lane == 0) {   // y: one TMA store per gated tile, then the buffer goes back to q
            for (int j = 0; j < nck; ++j) {
                const int s = j % kQStages;
                if (!tc::mbar_wait(bar(kBarYStaged + s), (j / kQStages) & 1, abort)) {
                    record_error(a, abort, kErrWait);
                    break;
                }
                for (int h = 0; h < 2; ++h)
                    tc::tma_store_3d(&tm_y, sbase + kSmQ + s * kTileBytes + h * kHalfBytes, c0 + 64 * h,
                                     (ck0 + j) * kC, b);
                tc::bulk_commit();
                tc::bulk_wait_read<0>();
                tc::mbar_arrive(bar(kBarQEmpty + s));
            }
            tc::bulk_wait<0>();     // every store of this CTA has completed
        }
    } else if (warp == 15) {
        // ------------------------------------------------------------ MMA issuer
        // Two streams issued out of order from one thread (polled with non-blocking tests, since
        // a suspending wait on one stream would hold back the other): the fused product of a chunk
        // (needs only its U operand and a free accumulator) runs ahead, the carry product
        // (needs the state entering the chunk) follows when the S group delivers it.  MMAs from
        // one thread execute in issue order, so a chunk's carry always lands after its fused part.
        if (lane == 0) {
            const uint32_t idesc_f = tc::idesc_tf32(kNC, kAccCols);
            const uint32_t idesc_c = tc::idesc_tf32(kNC, kC);
            int ic = 0, jn = 0;
            unsigned long long t_prog = tc::global_ns();
            while ((ic < niter || jn < nck) && !*abort) {
                bool progressed = false;
                if (jn < nck && n1 + jn < ic) {
                    const int sb = jn % kSTBufs, ab = (n1 + jn) % kNAcc;
                    if (tc::mbar_test(bar(kBarSRdy + sb), (jn / kSTBufs) & 1)) {
                        tc::tc_fence_after();
                        // carry: D[0:C) += S A^T
                        const uint32_t d = tmem + ab * kAccCols;
                        const uint32_t stb = sbase + kSmST + sb * kSTBytes;
                        for (int ks = 0; ks < kKSMax / 8; ++ks)
                            tc::mma_tf32(d, tc::smem_desc(stb + ks * 256, 128, kKSMax * 32),
                                         tc::smem_desc(sbase + kSmAT + ks * 256, 128, kKSMax * 32), idesc_c, 1);
                        tc::mma_commit(bar(kBarYDone + ab));
                        tc::mma_commit(bar(kBarSTFree + sb));
                        ++jn;
                        progressed = true;
                    }
                }
                if (ic < niter) {
                    const int ub = ic % kUBufs, ab = ic % kNAcc;
                    bool ready = tc::mbar_test(bar(kBarURdy + ub), (ic / kUBufs) & 1) &&
                                 tc::mbar_test(bar(kBarD2Free + ab), ((ic / kNAcc) & 1) ^ 1);
                    if (ready && ic >= n1)   // phase-2 uses of this accumulator (n1 % kNAcc == 0)
                        ready = tc::mbar_test(bar(kBarD1Free + ab), (((ic - n1) / kNAcc) & 1) ^ 1);
                    if (ready) {
                        tc::tc_fence_after();
                        // fused: D[0:C+32) = U [T; V]^T  (intra-chunk output | state contribution)
                        const uint32_t d = tmem + ab * kAccCols;
                        const uint32_t ut = sbase + kSmUT + ub * kUTBytes;
                        for (int ks = 0; ks < kC / 8; ++ks)
                            tc::mma_tf32(d, tc::smem_desc(ut + ks * 256, 128, kC * 32),
                                         tc::smem_desc(sbase + kSmTT + ks * 256, 128, kC * 32), idesc_f, ks > 0);
                        tc::mma_commit(bar(kBarWDone + ab));
                        tc::mma_commit(bar(kBarUFree + ub));
                        ++ic;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t_prog = tc::global_ns();
                } else {
                    if (tc::global_ns() - t_prog > tc::kWaitNs) {
                        record_error(a, abort, kErrWait);
                        break;
                    }
                    __nanosleep(32);      // polling: leave issue slots to the warps sharing the SMSP
                }
            }
            // all MMAs issued by this thread have completed once `drain` fires
            tc::mma_commit(bar(kBarDrain));
            tc::mbar_wait(bar(kBarDrain), 0, never);
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ U group
        // u = k*v of each chunk -> U operand buffer (it % kUBufs).  ldmatrix transposes the
        // 128-byte-swizzled k, v tiles: warp w covers channel groups 4w..4w+3 (8 channels each)
        // and each lane receives token pairs of one channel, the K-major row layout of U.
        // Tokens past the prompt were zero-filled by TMA.
        bool ok = true;
        const int r8 = lane & 7, mat = lane >> 3;
        for (int it = 0; it < niter && ok; ++it) {
            const int ub = it % kUBufs, s = it % kKVStages;
            ok = uni(tc::mbar_wait(bar(kBarUFree + ub), ((it / kUBufs) & 1) ^ 1, abort) &&
                     tc::mbar_wait(bar(kBarKVFull + s), (it / kKVStages) & 1, abort));
            if (!ok) break;
            const uint32_t kb = sbase + kSmKV + s * 2 * kTileBytes;
            uint8_t *ut = sm + kSmUT + ub * kUTBytes;
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
                const int cbase = 8 * (4 * warp + gi);
                const uint32_t off = (uint32_t)((cbase >> 6) * kHalfBytes + (8 * mat + r8) * 128 +
                                                ((((cbase & 63) >> 3) ^ r8) << 4));
                uint32_t kr[4], vr[4];
                tc::ldsm_x4_trans(kb + off, kr);
                tc::ldsm_x4_trans(kb + kTileBytes + off, vr);
                const int ch = cbase + (lane >> 2);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int tau = 8 * m + 2 * (lane & 3);
                    const float u0 = __uint_as_float(kr[m] << 16) * __uint_as_float(vr[m] << 16);
                    const float u1 = __uint_as_float(kr[m] & 0xffff0000u) * __uint_as_float(vr[m] & 0xffff0000u);
                    *reinterpret_cast<float2 *>(ut + cm_off(ch, tau, kC)) = make_float2(tc::to_tf32(u0), tc::to_tf32(u1));
                }
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(bar(kBarURdy + ub));
            // the prompt's last chunk stays until the S group has read it for the final state
            if (!(it >= n1 && chunk_of(it) == a.nchunks - 1)) tc::mbar_arrive(bar(kBarKVEmpty + s));
        }
        if (!ok) record_error(a, abort, kErrWait);
    } else if (warp < 8) {
        // ------------------------------------------------------------ S group (state chain)
        const int c = tid - 128;                     // channel within the tile == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        // lambda^C and lambda^Lseg stay in shared memory (broadcast reads) to keep this
        // group's registers for the state itself
        const float2 *lamC = reinterpret_cast<const float2 *>(sm + kSmLam);
        const float2 *lamS = lamC + kMaxModes;
        float2 st[kMaxModes];
#pragma unroll
        for (int n = 0; n < kMaxModes; ++n) st[n] = make_float2(0.f, 0.f);
        bool ok = true;
        int pub_phase = 0;
        // st <- lambda^C st + D2 of iteration it
        auto advance = [&](int it) -> bool {
            const int wb = it % kNAcc;
            if (!tc::mbar_wait(bar(kBarWDone + wb), (it / kNAcc) & 1, abort)) return false;
            tc::tc_fence_after();
            float w[kKSMax];
            const uint32_t taddr = tmem + lane_base + wb * kAccCols + kC;
            tc::tmem_ld16(taddr, w);
            tc::tmem_ld16(taddr + 16, w + 16);
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            tc::mbar_arrive(bar(kBarD2Free + wb));
#pragma unroll
            for (int n = 0; n < kMaxModes; ++n) {
                const float2 sv = st[n], lc = lamC[n];      // lambda^C is 0 for modes >= d
                st[n] = make_float2(fmaf(lc.x, sv.x, fmaf(-lc.y, sv.y, w[n])),
                                    fmaf(lc.x, sv.y, fmaf(lc.y, sv.x, w[kIm + n])));
            }
            return true;
        };
        auto publish = [&](float2 *dst, int code) -> bool {
            for (int n = 0; n < d; ++n) dst[(size_t)n * kNC + c] = st[n];
            __threadfence();
            tc::mbar_arrive(bar(kBarPub));
            bool r = true;
            if (c == 0) {
                r = tc::mbar_wait(bar(kBarPub), pub_phase & 1, abort);
                if (r) {
                    __threadfence();
                    atomicExch(a.status + item, code);
                }
            }
            ++pub_phase;
            return r;
        };

        // state-only pass over the segment, then publish its contribution
        for (int it = 0; it < n1 && ok; ++it) ok = uni(advance(it));
        if (ok && phase1) ok = uni(publish((seg == 0 ? a.inc : a.agg) + (size_t)item * d * kNC, seg == 0 ? 2 : 1));
        float2 sloc[kMaxModes];
#pragma unroll
        for (int n = 0; n < kMaxModes; ++n) { sloc[n] = st[n]; st[n] = make_float2(0.f, 0.f); }

        // look-back: the state entering this segment
        if (ok && seg > 0) {
            float2 scale[kMaxModes];
#pragma unroll
            for (int n = 0; n < kMaxModes; ++n) scale[n] = make_float2(1.f, 0.f);
            for (int p = item - 1; p >= item - seg && ok; --p) {
                int code = *(volatile int *)(a.status + p);
                const unsigned long long t0 = tc::global_ns();
                while (code == 0 && !*abort && tc::global_ns() - t0 < tc::kWaitNs) {
                    __nanosleep(100);
                    code = *(volatile int *)(a.status + p);
                }
                if (code == 0) {
                    record_error(a, abort, kErrLookback);
                    ok = false;
                    break;
                }
                __threadfence();
                const volatile float2 *src = (code == 2 ? a.inc : a.agg) + (size_t)p * d * kNC;
#pragma unroll
                for (int n = 0; n < kMaxModes; ++n) {
                    if (n < d) {
                        const float2 v = make_float2(src[(size_t)n * kNC + c].x, src[(size_t)n * kNC + c].y);
                        st[n] = cadd(st[n], cmul(scale[n], v));
                        scale[n] = cmul(scale[n], lamS[n]);
                    }
                }
                if (code == 2) break;
            }
            ok = uni(ok);
            if (ok && phase1) {
                // inclusive state at the end of this segment: lambda^Lseg s_in + own contribution
                float2 keep[kMaxModes];
#pragma unroll
                for (int n = 0; n < kMaxModes; ++n) {
                    keep[n] = st[n];
                    st[n] = cadd(cmul(lamS[n], st[n]), sloc[n]);
                }
                ok = uni(publish(a.inc + (size_t)item * d * kNC, 2));
#pragma unroll
                for (int n = 0; n < kMaxModes; ++n) st[n] = keep[n];
            }
        }

        // full pass: state operand for each chunk, then the state after it
        for (int j = 0; j < nck && ok; ++j) {
            const int it = n1 + j, sb = j % kSTBufs;
            if (!(ok = uni(tc::mbar_wait(bar(kBarSTFree + sb), ((j / kSTBufs) & 1) ^ 1, abort)))) break;
            uint8_t *stp = sm + kSmST + sb * kSTBytes;
#pragma unroll
            for (int n4 = 0; n4 < kMaxModes / 4; ++n4) {
                const int n = 4 * n4;
                *reinterpret_cast<float4 *>(stp + cm_off(c, n, kKSMax)) =
                    make_float4(tc::to_tf32(st[n].x), tc::to_tf32(st[n + 1].x), tc::to_tf32(st[n + 2].x),
                                tc::to_tf32(st[n + 3].x));
                *reinterpret_cast<float4 *>(stp + cm_off(c, kIm + n, kKSMax)) =
                    make_float4(tc::to_tf32(st[n].y), tc::to_tf32(st[n + 1].y), tc::to_tf32(st[n + 2].y),
                                tc::to_tf32(st[n + 3].y));
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(bar(kBarSRdy + sb));
            const int chunk = ck0 + j;
            if (chunk != a.nchunks - 1) {
                if (!(ok = uni(advance(it)))) break;
            } else {
                // last chunk of the prompt (possibly partial): exact fp32 Horner over its
                // tokens, st <- lambda^rem st + sum_{iota<rem} lambda^(rem-1-iota) u_iota
                const int s = it % kKVStages;
                if (!(ok = uni(tc::mbar_wait(bar(kBarKVFull + s), (it / kKVStages) & 1, abort)))) break;
                const int rem = a.L - chunk * kC;
                const uint8_t *kt = sm + kSmKV + s * 2 * kTileBytes;
                const uint8_t *vt = kt + kTileBytes;
                float2 lm[kMaxModes], acc[kMaxModes];
#pragma unroll
                for (int n = 0; n < kMaxModes; ++n) {
                    lm[n] = n < d ? __ldg(&a.lam[(size_t)hd * d + n]) : make_float2(0.f, 0.f);
                    acc[n] = make_float2(0.f, 0.f);
                }
                for (int io = 0; io < rem; ++io) {
                    const int o = act_off(io, c);
                    const float u = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(kt + o)) *
                                    __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(vt + o));
#pragma unroll
                    for (int n = 0; n < kMaxModes; ++n)
                        acc[n] = make_float2(fmaf(acc[n].x, lm[n].x, fmaf(-acc[n].y, lm[n].y, u)),
                                             fmaf(acc[n].x, lm[n].y, acc[n].y * lm[n].x));
                }
                tc::mbar_arrive(bar(kBarKVEmpty + s));
#pragma unroll
                for (int n = 0; n < kMaxModes; ++n) {
                    if (n < d) {
                        const cd pw = cdpow(cd{lm[n].x, lm[n].y}, rem);
                        st[n] = cadd(cmul(make_float2((float)pw.x, (float)pw.y), st[n]), acc[n]);
                    }
                }
            }
        }
        if (!ok) record_error(a, abort, kErrWait);
        if (ok && last_seg) {
            float2 *so = reinterpret_cast<float2 *>(a.state_out) + ((size_t)b * d) * a.Dch + c0 + c;
            for (int n = 0; n < d; ++n) so[(size_t)n * a.Dch] = st[n];
        }
    } else {
        // ------------------------------------------------------------ E group (gate and stage y)
        const int c = tid - 256;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = true;
        for (int j = 0; j < nck && ok; ++j) {
            const int db = j % kNAcc, s = j % kQStages;     // == (n1 + j) % kNAcc since n1 % kNAcc == 0
            ok = uni(tc::mbar_wait(bar(kBarYDone + db), (j / kNAcc) & 1, abort) &&
                     tc::mbar_wait(bar(kBarQFull + s), (j / kQStages) & 1, abort));
            if (!ok) break;
            tc::tc_fence_after();
            uint8_t *qy = sm + kSmQ + s * kTileBytes;
            __nv_bfloat16 qv[kC];
#pragma unroll
            for (int tau = 0; tau < kC; ++tau) qv[tau] = *reinterpret_cast<const __nv_bfloat16 *>(qy + act_off(tau, c));
            float z[kC];
            tc::tmem_ld16(tmem + lane_base + db * kAccCols, z);
            tc::tmem_ld16(tmem + lane_base + db * kAccCols + 16, z + 16);
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            tc::mbar_arrive(bar(kBarD1Free + db));
#pragma unroll
            for (int tau = 0; tau < kC; ++tau)
                *reinterpret_cast<__nv_bfloat16 *>(qy + act_off(tau, c)) =
                    __float2bfloat16_rn(__bfloat162float(qv[tau]) * z[tau]);
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(bar(kBarYStaged + s));
        }
        if (!ok) record_error(a, abort, kErrWait);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 15) tc::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [B][L][Dch] bf16 viewed as a 3-D tensor (Dch, L, B); box = 128 channels x C tokens x 1
bool make_map(CUtensorMap *m, const void *base, int B, int L, int Dch) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)Dch, (cuuint64_t)L, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)Dch * 2, (cuuint64_t)L * Dch * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kC, 1};     // 64 channels = 128 bytes, the swizzle span
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct ChunkPlan {
    int nchunks, nseg, segc, items;
    size_t consts_off, sched_off, status_off, agg_off, inc_off, total;
};

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

ChunkPlan plan(int B, int L, int Dch, int H, int d) {
    ChunkPlan p{};
    p.nchunks = (L + kC - 1) / kC;
    const long long units = (long long)B * (Dch / kNC);
    // enough items for ~2 waves of one CTA per SM, segments of at least 4 chunks
    long long want = (2 * 148 + units - 1) / units;
    long long maxseg = (p.nchunks + 3) / 4;
    if (want > maxseg) want = maxseg;
    if (want < 1) want = 1;
    p.segc = (int)((p.nchunks + want - 1) / want);
    p.segc = (p.segc + kNAcc - 1) / kNAcc * kNAcc;   // state-only passes cover whole accumulator rings
    p.nseg = (p.nchunks + p.segc - 1) / p.segc;
    p.items = (int)(units * p.nseg);
    p.consts_off = 0;
    p.sched_off = al256((size_t)H * kConstStride);
    p.status_off = p.sched_off + 256;
    p.agg_off = p.status_off + al256((size_t)p.items * 4);
    p.inc_off = p.agg_off + al256((size_t)p.items * d * kNC * 8);
    p.total = p.inc_off + al256((size_t)p.items * d * kNC * 8);
    return p;
}

}  // namespace

bool chunked_supported(int dtype, int Dch, int H, int d) {
    return dtype == HYENA_BF16 && H > 0 && Dch % H == 0 && (Dch / H) % kNC == 0 && d >= 1 && d <= kMaxModes;
}

size_t chunked_ws_bytes(int B, int L, int Dch, int H, int d) { return plan(B, L, Dch, H, d).total; }

cudaError_t launch_prefill_chunked(const void *q, const void *k, const void *v, int B, int L, int Dch,
                                   int H, int d, const float2 *lam, const float2 *R, const float *Dskip,
                                   void *y, float *state_out, void *ws, cudaStream_t s) {
    const ChunkPlan p = plan(B, L, Dch, H, d);
    uint8_t *w = static_cast<uint8_t *>(ws);

    cudaError_t e = cudaMemsetAsync(w + p.sched_off, 0, p.agg_off - p.sched_off, s);
    if (e != cudaSuccess) return e;
    chunk_consts_kernel<<<H, 256, 0, s>>>(lam, R, Dskip, d, p.segc * kC, w + p.consts_off);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap mq, mk, mv, my;
    if (!make_map(&mq, q, B, L, Dch) || !make_map(&mk, k, B, L, Dch) || !make_map(&mv, v, B, L, Dch) ||
        !make_map(&my, y, B, L, Dch))
        return cudaErrorInvalidValue;
    ChunkArgs a;
    a.L = L; a.Dch = Dch; a.d = d; a.ch = Dch / H;
    a.ntiles = Dch / kNC; a.nchunks = p.nchunks; a.nseg = p.nseg; a.segc = p.segc;
    a.lam = lam;
    a.consts = w + p.consts_off;
    a.state_out = state_out;
    a.sched = reinterpret_cast<int *>(w + p.sched_off);
    a.status = reinterpret_cast<int *>(w + p.status_off);
    a.agg = reinterpret_cast<float2 *>(w + p.agg_off);
    a.inc = reinterpret_cast<float2 *>(w + p.inc_off);
    e = cudaFuncSetAttribute(prefill_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    prefill_chunk_kernel<<<p.items, kThreads, kSmemBytes, s>>>(mq, mk, mv, my, a);
    return cudaGetLastError();
}

int chunked_error_offset(int B, int L, int Dch, int H, int d) {
    return (int)(plan(B, L, Dch, H, d).sched_off + 4);
}

}  // namespace hyena
