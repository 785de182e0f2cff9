// prefill_chunked.cu -- chunked modal prefill on tcgen05 tensor cores.
//
// The long convolution y = q * (h conv (k * v)) ("Hyena processes long
// sequences 100x faster than FlashAttention", lequren.com, "Hyena層次結構")
// with the modal filter h_0 = Dskip, h_j = Re sum_n R_n lambda_n^(j-1) of
// "Laughing Hyena Distillery" (nubint.ai review, "Proposed method") is
// evaluated chunk by chunk.  For a chunk of C tokens starting at token t0, with
// tau, iota in [0, C):
//
//   z[t0+tau] = sum_{iota<=tau} h_{tau-iota} u[t0+iota]            (intra-chunk Toeplitz)
//             + Re sum_n R_n lambda_n^tau s_n(t0)                  (modal carry from the past)
//   s_n(t0+C) = lambda_n^C s_n(t0) + sum_iota lambda_n^(C-1-iota) u[t0+iota]
//
// where s(t0) is the recurrent state after the tokens before t0 -- the same
// O(d) state the decode step advances ("Main findings": O(d) memory per
// channel).  This is an exact regrouping of the causal convolution (the carry
// is the tail of the sum over j < t0, with h_{t-j} = Re sum R lambda^(t-t0)
// lambda^(t0-1-j)), and the prompt -> state reduction is the last state.
//
// The chunk grid is aligned to the END of the prompt: chunk i covers tokens
// [L - (nchunks-i) C, L - (nchunks-1-i) C), so the first chunk may start before
// token 0 (its missing tokens are zero-filled by TMA and contribute nothing)
// and the state after the last chunk is exactly the state after token L-1.
//
// Per chunk and channel tile (NC = 128 or 64 channels) the tensor cores evaluate, in bf16 with
// fp32 accumulation in tensor memory (rows on MMA M, the NC channels on MMA N):
//   fused:  [Z; W] = [T; V] U          T[tau][iota] = h_{tau-iota} (iota <= tau)
//                                      V[r][iota]   = (Re | Im) lambda_r^(C-1-iota)
//   carry:  Z     += A S               A[tau][r]    = (Re | -Im) R_r lambda_r^tau
// where U[iota][c] = k v is formed elementwise (packed bf16 products) over the TMA'd k tile
// (its natural [token][channel] 128-byte-swizzled layout is already an MN-major operand),
// S[r][c] = (Re | Im) s(t0) and W[r][c] is the chunk's state contribution.  The two A
// operands are per-head constants: the 64-channel tile keeps them in tensor memory (copied
// there once per head), the 128-channel tile reads them from shared memory.  The state chain
// s <- lambda^C s + W runs on the CUDA cores in fp32 (one thread per state row and NC/4
// channels), and y = q (Z + carry) is gated and stored per token row.  The carry accumulates
// onto the fused product in the same tensor-memory columns (A's rows 64..127 are zero, so it
// adds nothing to the state rows W); the chain reads W out before it posts the state operand
// that lets the carry start, so the two never overlap.  A slot is thus NC columns, and up to 7
// (64-channel tile) or 4 chunks are in flight between the products, the chain and the gate.
//
// Work split: a sequence is cut into segments of whole chunks; each
// (batch, channel tile, segment) item but the last of its sequence first runs a
// state-only pass (k, v and the fused product) to publish its segment's state
// contribution, then (segments after the first) obtains the
// state entering its segment by a decoupled look-back over its predecessors'
// published contributions (bounded polls), then runs the full pass.  The grid is
// persistent: items come from an atomic ticket counter, and each CTA's
// pipelines run on across item boundaries.  Tickets are segment-major (all
// heads' and units' first segments, then all second segments, ...), so an item's
// predecessors were handed out a whole round of units earlier and have usually
// published by the time it looks back.
//
// Progress does not depend on the order in which CTAs become resident: an item
// only ever waits on items with lower tickets, and a ticket is only ever held by
// a CTA that is running (it took the ticket from the counter), whose earlier
// items have lower tickets still; the state-only pass never waits.  By induction
// over the tickets every look-back ends, even when other kernels hold most SMs.
// When sequences are split, the counter is therefore cleared by a memset ahead
// of the constants kernel, so the loaders can take tickets at once.  When they
// are not (no item waits on another), each CTA's first ticket is fixed
// (blockIdx.x) and only later tickets come from the counter, which the constants
// kernel clears.  Every wait is bounded; on timeout the kernel records an error
// code, drains its copies and MMAs, frees tensor memory and returns.
//
// Several independent layers of the same shape can share one launch: their heads
// are the heads of one ticket space (layer = head / heads per layer), each with
// its own constants and its own tensor maps, y and state.
#include <atomic>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace hyena {

namespace {

constexpr int kC = 64;              // tokens per chunk (K of the fused product)
constexpr int kMaxModes = 16;       // d <= 16
constexpr int kKS = 32;             // state rows: Re of modes 0..15, then Im
constexpr int kIm = 16;
constexpr int kAtom = kC * 64 * 2;  // one bf16 [C][64] TMA box, 128-byte swizzled (8 KB)
constexpr int kSBufs = 2;           // state operands
constexpr int kItemQ = 4;           // item ids handed from the k,v loader to the other roles
constexpr int kThreads = 512;
constexpr int kMaxSeg = 128;        // segments per sequence (bounds look-back walks)
constexpr int kPubQ = 4;            // segment states written and waiting for their status word
constexpr uint32_t kTmemCols = 512; // all of tensor memory (one CTA per SM)
// item readers: q loader, store lane, fused and carry MMA lanes (1 each) + lane 0 of the 3 U,
// 4 S and 4 E warps
constexpr int kItemReaders = 4 + 11;
constexpr int kUThreads = 96;       // U group (3 warps)
constexpr int kEThreads = 128;      // E group (4 warps); it helps to form U in state-only iterations
constexpr int kUHelp = kUThreads + kEThreads;

// per-head constants: the two A operands (copied verbatim into shared memory) and the powers
// lambda^C, lambda^Lseg (read from global by the state group)
constexpr int kFABytes = 128 * kC * 2;       // [T; V; 0]: 128 rows x 64 K bf16
constexpr int kCABytes = 128 * kKS * 2;      // [A; 0]:    128 rows x 32 K bf16
constexpr int kOpBytes = kFABytes + kCABytes;
constexpr int kLamOff = kOpBytes;            // float2 lambda^C [16], lambda^Lseg [16]
constexpr int kConstStride = kOpBytes + 256;

// shared memory map (offsets from a 1024-byte aligned base): constants, then the rings
constexpr int kSmFA = 0;
constexpr int kSmCA = kSmFA + kFABytes;
constexpr int kSmKV = kSmCA + kCABytes;                   // 1024-aligned (swizzle atoms)

// Layout for a channel tile of NC = 128 or 64 channels (MMA N).  The narrow tile gives twice
// the (sequence, tile) units, so that small batches fill the GPU without splitting sequences;
// its rings are twice as deep (same bytes), and it keeps its A operands in tensor memory next
// to seven accumulator slots (the 128-channel tile has four and reads A from shared memory).
template <int NC>
struct Geo {
    static_assert(NC == 64 || NC == 128, "channel tile");
    static constexpr int kTile = kC * NC * 2;                 // one bf16 [C][NC] activation tile
    static constexpr int kStageBytes = 2 * kTile;             // k (overwritten by U) then v
    static constexpr int kKVStages = NC == 128 ? 4 : 8;
    static constexpr int kQStages = NC == 128 ? 3 : 6;        // q tiles; y is staged in place
    // One accumulator slot per chunk in flight: NC columns, into which the fused product writes
    // [Z; W] and the carry product then adds A S.  The carry operand's rows 64..127 are zero, so
    // it leaves the state rows W as they are; the S group reads them out before it posts the
    // state operand that lets the carry start, so the two never overlap.
    static constexpr int kSlotCols = NC;
    // The 64-channel tile keeps both A operands (constant per head) in tensor memory, so the MMAs
    // read only their B operand from shared memory: 7 accumulator slots + 48 columns of A
    // (fused A: K = 64 -> 32 columns, carry A: K = 32 -> 16 columns).  The 128-channel tile
    // gives every column to its 4 slots and reads A from shared memory.
    static constexpr bool kATmem = NC == 64;
    // The 64-channel tile also splits the fused products of a state-only pass between the two
    // product issuers (there the issue work paces the pass; the 128-channel tile's code is left
    // as it is, since its longer code measured slower without using the split).
    static constexpr bool kDualSO = NC == 64;
    static constexpr int kSlots = kATmem ? ((int)kTmemCols - 48) / kSlotCols : (int)kTmemCols / kSlotCols;
    static constexpr int kACol = kSlots * kSlotCols;          // first column of A (kATmem)
    static_assert(!kATmem || kACol + 48 <= (int)kTmemCols, "tensor memory budget");
    static constexpr int kSBytes = kKS * NC * 2;              // [32 rows][NC ch] bf16, 128-byte swizzled
    static constexpr int kSmQ = kSmKV + kKVStages * kStageBytes;
    static constexpr int kSmS = kSmQ + kQStages * kTile;
    static constexpr int kSmBar = kSmS + kSBufs * kSBytes;
    // barrier slots (arrival counts in parentheses; "commit" = tcgen05.commit from the MMA thread)
    static constexpr int kBarKVFull = 0;                              // [kKVStages] k,v landed (1 + tx)
    static constexpr int kBarKVEmpty = kBarKVFull + kKVStages;        // [kKVStages] fused product read U (commit)
    static constexpr int kBarURdy = kBarKVEmpty + kKVStages;          // [kKVStages] U formed over k (128: U group)
    static constexpr int kBarQFull = kBarURdy + kKVStages;            // [kQStages] q landed (1 + tx)
    static constexpr int kBarQEmpty = kBarQFull + kQStages;           // [kQStages] y stored, buffer free (1)
    static constexpr int kBarYStaged = kBarQEmpty + kQStages;         // [kQStages] gated y staged (128: E group)
    static constexpr int kBarWDone = kBarYStaged + kQStages;          // [kSlots] fused product done (commit)
    static constexpr int kBarD2Free = kBarWDone + kSlots;             // [kSlots] state rows read out (128: S)
    static constexpr int kBarYDone = kBarD2Free + kSlots;             // [kSlots] carry done (commit)
    static constexpr int kBarD1Free = kBarYDone + kSlots;             // [kSlots] output rows read out (128: E)
    static constexpr int kBarSRdy = kBarD1Free + kSlots;              // [kSBufs] state operand written (128: S)
    static constexpr int kBarSTFree = kBarSRdy + kSBufs;              // [kSBufs] state operand read (commit)
    static constexpr int kBarItemFull = kBarSTFree + kSBufs;          // [kItemQ] item id posted (1)
    static constexpr int kBarItemEmpty = kBarItemFull + kItemQ;       // [kItemQ] id read by every consumer
    static constexpr int kBarConst = kBarItemEmpty + kItemQ;          // head constants landed (1 + tx)
    static constexpr int kBarConstFree = kBarConst + 1;               // MMAs on the old constants done (commit)
    static constexpr int kBarPubFull = kBarConstFree + 1;             // [kPubQ] segment state written (128: S)
    static constexpr int kBarPubEmpty = kBarPubFull + kPubQ;          // [kPubQ] status posted (1: publisher)
    static constexpr int kBarDrain = kBarPubEmpty + kPubQ;            // fused issuer's MMAs finished (commit)
    static constexpr int kBarDrainC = kBarDrain + 1;                  // carry issuer's MMAs finished (commit)
    static constexpr int kBarSOFin = kBarDrainC + 1;                  // carry issuer's state-only products of an item done (commit)
    static constexpr int kBarAReady = kBarSOFin + 1;                  // a head's A operands in place (commit, once per head switch)
    static constexpr int kNumBars = kBarAReady + 1;
    static constexpr int kSmMisc = kSmBar + kNumBars * 8;
    static constexpr int kSmemBytes = kSmMisc + 128 + 1024;           // + ids, misc words, queues, slack
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kSmQ % 1024 == 0 && kSmS % 1024 == 0, "swizzle atoms");

    __host__ __device__ static constexpr int count(int i) {
        return (i >= kBarURdy && i < kBarQFull) ? kUHelp
               : ((i >= kBarYStaged && i < kBarWDone) || (i >= kBarD2Free && i < kBarYDone) ||
                  (i >= kBarD1Free && i < kBarSTFree) || (i >= kBarPubFull && i < kBarPubEmpty))
                   ? 128
                   : (i >= kBarItemEmpty && i < kBarConst) ? kItemReaders : 1;
    }
};

// warp roles (16 warps).  The state group must sit on warps w % 4 == 2 (TMEM lanes 64..95, the
// state rows); the output group on w % 4 in {0, 1} (lanes 0..63, the token rows).
constexpr int kWarpKV = 0, kWarpQ = 1, kWarpMMA = 3, kWarpStore = 12, kWarpCarry = 13;
__host__ __device__ constexpr bool is_s_warp(int w) { return (w & 3) == 2; }                 // 2, 6, 10, 14
__host__ __device__ constexpr bool is_e_warp(int w) { return w == 4 || w == 5 || w == 8 || w == 9; }
__host__ __device__ constexpr int u_index(int w) { return w == 7 ? 0 : w == 11 ? 1 : w == 15 ? 2 : -1; }
__host__ __device__ constexpr int e_index(int w) { return w == 4 ? 0 : w == 5 ? 1 : w == 8 ? 2 : 3; }


// byte offset of bf16 element (row, k) in a K-major, no-swizzle core-matrix tile of K columns
__host__ __device__ __forceinline__ int cm_off16(int row, int k, int K) {
    return (k >> 3) * 128 + (row >> 3) * (K * 16) + (row & 7) * 16 + (k & 7) * 2;
}

struct ChunkArgs {
    int L, Dch, d, ch;
    int H;               // heads of the ticket space: layers x Hl (one counter and constant block each)
    int Hl;              // heads per layer
    int tph;             // channel tiles per head (ch / NC)
    int units_h;         // (sequence, tile) units per head: B * tph
    int ih;              // items per head: units_h * nseg
    int nchunks;         // chunks per sequence
    int tok_base;        // first token of chunk 0 (L - nchunks * C, <= 0)
    int nseg, segc;      // segments per sequence, chunks per segment (all but the last)
    const uint8_t *consts;
    int *sched;          // [1] error code
    int *tickets;        // [1] ticket counter
    int *status;         // [items]: 0 none, 1 segment contribution, 2 inclusive state
    float *agg;          // [items][32 rows][NC ch]
    float *inc;          // [items][32 rows][NC ch]
    int fixed_first;     // 1: each CTA's first item has a fixed ticket (only when nseg == 1)
    int suppress_item;   // fault injection for tests: this item's status word is never posted (-1: none)
    unsigned long long lookback_ns;   // bound of one look-back poll
};

struct Item {
    int id, b, c0, hd, layer, seg, ck0, nck, n1, niter;
    bool last_seg;
};

// Per-layer tensors of one launch (LMAX = 1 for a single layer, kMaxGroupLayers for a group of
// independent layers): the TMA maps of q, k, v, y and the y and state pointers.  Passed by value
// as a __grid_constant__ parameter, so the maps are in parameter space where TMA can read them.
template <int LMAX>
struct LayerMaps {
    CUtensorMap q[LMAX], k[LMAX], v[LMAX], y[LMAX];
    __nv_bfloat16 *yp[LMAX];   // y, for the rows of a chunk that starts before token 0
    float *state[LMAX];        // [B][d][Dch][2]
};
template <int LMAX>
struct ParamPtrs {
    const float2 *lam[LMAX], *R[LMAX];
    const float *Dskip[LMAX];
};
constexpr int kMaxGroupLayers = 32;

template <int NC>
__device__ __forceinline__ Item decode_item(const ChunkArgs &a, int id) {
    Item it;
    it.id = id;
    it.hd = id / a.ih;                      // head of the ticket space
    it.layer = it.hd / a.Hl;
    const int t = id % a.ih;                // ticket within the head, segment-major: the
    const int unit = t % a.units_h;         // predecessor of item id is id - units_h
    it.seg = t / a.units_h;
    it.b = unit / a.tph;
    it.c0 = (it.hd % a.Hl) * a.ch + (unit % a.tph) * NC;
    it.ck0 = it.seg * a.segc;
    it.nck = min(a.nchunks, it.ck0 + a.segc) - it.ck0;
    it.last_seg = (it.seg == a.nseg - 1);
    it.n1 = it.last_seg ? 0 : it.nck;        // state-only iterations
    it.niter = it.n1 + it.nck;
    return it;
}

// Item of ticket t: tickets run segment-major over all heads (t = (seg * H + head) * units_h + unit),
// items are numbered head-major (id = head * ih + seg * units_h + unit, so that the predecessor of
// item id is id - units_h).  Unsplit sequences: the identity.
__device__ __forceinline__ int ticket_item(const ChunkArgs &a, int t) {
    const int round = a.H * a.units_h;
    const int seg = t / round, r = t % round;
    return (r / a.units_h) * a.ih + seg * a.units_h + r % a.units_h;
}

enum : int { kErrWait = 1, kErrLookback = 2 };

// The code is recorded before the CTA's other roles are told to stop, so the error word holds the
// cause (a role that then gives up on a wait only finds the word already set).
__device__ __forceinline__ void record_error(const ChunkArgs &a, volatile int *abort, int code) {
    atomicCAS(a.sched + 1, 0, code);
    __threadfence();
    *abort = 1;
}

// Load with acquire semantics at GPU scope (pairs with the publisher's fence + status write).
__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// One step x <- lam x + a of a complex recurrence held as (Re, Im) in the lanes r and r ^ 16 of a
// warp (sgn = -1 in the Re lanes, +1 in the Im lanes).  Used for every segment-state combination,
// so that the same inputs always give the same bits.
__device__ __forceinline__ float seg_step(float x, float a, float2 lam, float sgn) {
    const float xp = __shfl_xor_sync(0xffffffffu, x, 16);
    return fmaf(lam.x, x, fmaf(sgn * lam.y, xp, a));
}

// In-register transpose of a 32 x 32 block held one row per lane (v[j] = M[lane][j]) into one
// column per lane (v[j] = M[j][lane]): five butterfly stages of warp shuffles.
__device__ __forceinline__ void warp_transpose32(float *v, int lane) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & m) continue;
            const float send = upper ? v[i] : v[i | m];
            const float recv = __shfl_xor_sync(0xffffffffu, send, m);
            if (upper) v[i] = recv; else v[i | m] = recv;
        }
    }
}

// The same within each half-warp for a 16 x 16 block: lanes 16 h + i hold rows 16 h + i
// (v[j] = M[16 h + i][j]) and end up with columns (v[j] = M[16 h + j][i]).
__device__ __forceinline__ void warp_transpose16x2(float *v, int lane) {
#pragma unroll
    for (int m = 8; m >= 1; m >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i & m) continue;
            const float send = upper ? v[i] : v[i | m];
            const float recv = __shfl_xor_sync(0xffffffffu, send, m);
            if (upper) v[i] = recv; else v[i | m] = recv;
        }
    }
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float *v) {
    if constexpr (N == 32) tc::tmem_ld32(taddr, v);
    else tc::tmem_ld16(taddr, v);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }
// Two bf16 products rounded to nearest bf16 in one instruction.  The exact product of two bf16
// values has at most 16 significant bits, so this is the same rounding as an fp32 product
// followed by a conversion to bf16 (outside the subnormal range).
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// U = k v in place over the k half of a k,v stage (the same byte offset in k, v and U), 16 bytes
// per piece: thread `t` of kThreads takes pieces t, t + kThreads, ...  Every load is issued
// before the first product, so a thread waits for one shared-memory round trip, not one per
// piece (the latency is long while TMA and the tensor cores also use shared memory).
template <int kTileBytes, int kThreads>
__device__ __forceinline__ void form_u(uint8_t *kt, int t) {
    constexpr int kPieces = kTileBytes / 16, kPer = (kPieces + kThreads - 1) / kThreads;
    uint4 kk[kPer], vv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int off = (t + i * kThreads) * 16;
        if (i < kPer - 1 || t + i * kThreads < kPieces) {
            kk[i] = *reinterpret_cast<const uint4 *>(kt + off);
            vv[i] = *reinterpret_cast<const uint4 *>(kt + kTileBytes + off);
        }
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int off = (t + i * kThreads) * 16;
        if (i < kPer - 1 || t + i * kThreads < kPieces)
            *reinterpret_cast<uint4 *>(kt + off) = make_uint4(mul_bf16x2(kk[i].x, vv[i].x), mul_bf16x2(kk[i].y, vv[i].y),
                                                              mul_bf16x2(kk[i].z, vv[i].z), mul_bf16x2(kk[i].w, vv[i].w));
    }
}

// ------------------------------------------------------------------ per-head constants
// One block of kConstThreads threads per head.  Every entry is a power lambda_n^k with
// 0 <= k <= C, so the powers are tabulated first (one entry per thread, by binary powering) and
// the taps and operands are then filled from the table, one tap and one 16-byte operand piece
// per thread, so that no thread runs a long dependent chain (the whole kernel sits on the
// prefill's critical path).  fp32 suffices: the operands are rounded to bf16 (relative 2^-9) and
// the chain powers lambda^C, lambda^Lseg enter an fp32 recurrence, while binary powering to an
// exponent below 2^31 loses at most a few tens of fp32 ulps.
__device__ __forceinline__ float2 cfpow(float2 lam, long long m) {
    float2 r = make_float2(1.f, 0.f), b = lam;
    while (m > 0) {
        if (m & 1) r = cmul(r, b);
        b = cmul(b, b);
        m >>= 1;
    }
    return r;
}

constexpr int kConstThreads = 1024;
static_assert(kConstThreads == kMaxModes * kC, "one power-table entry per thread");
static_assert(128 * (kC / 8) == kConstThreads && 128 * (kKS / 8) <= kConstThreads, "one operand piece per thread");

// It also clears the main kernel's schedule words (`zero`, `nzero` ints: error word, ticket
// counters, segment status words), and allows the main kernel to launch at once (programmatic
// dependent launch): where the main kernel's CTAs find room early, their set-up and first loads
// overlap this kernel; its griddepcontrol.wait returns once everything written here is visible.
// One block per head of the ticket space (layer hd / Hl, head hd % Hl of that layer).
template <int LMAX>
__global__ void __launch_bounds__(kConstThreads)
chunk_consts_kernel(const __grid_constant__ ParamPtrs<LMAX> pp, int Hl, int d, int seg_tokens,
                    uint8_t *__restrict__ consts, int *__restrict__ zero, int nzero) {
    asm volatile("griddepcontrol.launch_dependents;");
    const int t = threadIdx.x;
    for (int i = blockIdx.x * kConstThreads + t; i < nzero; i += gridDim.x * kConstThreads) zero[i] = 0;
    const int hd = blockIdx.x, layer = hd / Hl, hl = hd % Hl;
    const float2 *__restrict__ lam = pp.lam[layer];
    const float2 *__restrict__ R = pp.R[layer];
    const float *__restrict__ Dskip = pp.Dskip[layer];
    uint8_t *base = consts + (size_t)hd * kConstStride;
    float2 *lamC = reinterpret_cast<float2 *>(base + kLamOff);
    float2 *lamS = lamC + kMaxModes;
    __shared__ float2 pw[kMaxModes][kC];         // lambda_n^k, k < C; zero for modes >= d
    __shared__ float2 ls[kMaxModes], rs[kMaxModes];   // lambda_n, R_n
    __shared__ float hs[kC];                     // filter taps h_0 .. h_{C-1}
    __shared__ float dskip;
    const long long n_par = (long long)Hl * d;
    (void)n_par;
    if (t < kMaxModes) ls[t] = t < d ? lam[HB_IDX((size_t)hl * d + t, n_par)] : make_float2(0.f, 0.f);
    else if (t < 2 * kMaxModes) rs[t - kMaxModes] = t - kMaxModes < d ? R[HB_IDX((size_t)hl * d + t - kMaxModes, n_par)] : make_float2(0.f, 0.f);
    else if (t == 2 * kMaxModes) dskip = Dskip[HB_IDX(hl, Hl)];
    __syncthreads();
    {
        const int n = t / kC, k = t % kC;
        pw[n][k] = cfpow(ls[n], k);               // ls[n] = 0 for modes >= d: 0^0 = 1 is never read there
        if (t < kMaxModes) lamC[t] = cfpow(ls[t], kC);
        else if (t < 2 * kMaxModes) lamS[t - kMaxModes] = cfpow(ls[t - kMaxModes], seg_tokens);
    }
    __syncthreads();
    {
        // tap j (j >= 1) = Re sum_n R_n lambda_n^(j-1): lane group of 16 threads per tap, one mode
        // each, summed by a fixed shuffle tree (modes >= d contribute zero)
        const int j = t >> 4, n = t & 15;
        const float2 p = pw[n][j > 0 ? j - 1 : 0];
        float v = n < d ? fmaf(rs[n].x, p.x, -rs[n].y * p.y) : 0.f;
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (n == 0) hs[j] = j == 0 ? dskip : v;
    }
    __syncthreads();
    // fused A operand: rows 0..C-1 Toeplitz taps, rows C..C+31 chunk powers (Re at r < 16, Im at
    // 16 + n), rows C+32..127 zero; one 16-byte core-matrix row (8 consecutive K entries of one
    // row) per thread
    {
        __nv_bfloat16 *FA = reinterpret_cast<__nv_bfloat16 *>(base);
        const int row = t / (kC / 8), io0 = 8 * (t % (kC / 8));
        float v[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            const int io = io0 + x;
            v[x] = 0.f;
            if (row < kC) {
                v[x] = io <= row ? hs[row - io] : 0.f;
            } else if (row < kC + kKS) {
                const int r = row - kC;
                const float2 q = pw[r & (kIm - 1)][kC - 1 - io];
                v[x] = (r & (kIm - 1)) < d ? (r < kIm ? q.x : q.y) : 0.f;
            }
        }
        if (HB_OK(cm_off16(row, io0, kC) + 15, kFABytes))
            *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(FA) + cm_off16(row, io0, kC)) =
                make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
    }
    // carry A operand: rows 0..C-1: (Re, -Im) of R_n lambda_n^tau; rows C..127 zero
    if (t < 128 * (kKS / 8)) {
        __nv_bfloat16 *CA = reinterpret_cast<__nv_bfloat16 *>(base + kFABytes);
        const int row = t / (kKS / 8), r0 = 8 * (t % (kKS / 8));
        float v[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            const int r = r0 + x, n = r & (kIm - 1);
            v[x] = 0.f;
            if (row < kC) {
                const float2 c = cmul(rs[n], pw[n][row]);
                v[x] = r < kIm ? c.x : -c.y;
            }
        }
        if (HB_OK(cm_off16(row, r0, kKS) + 15, kCABytes))
            *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(CA) + cm_off16(row, r0, kKS)) =
                make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
    }
}

// ------------------------------------------------------------------ main kernel
// Roles (warps):  0  k,v TMA loads; takes item tickets and posts them to the other roles
//                 1  q TMA loads            12  y TMA stores, segment-state publisher (lanes 0, 1)
//                 3  tensor memory owner and fused-product issuer (lane 0)
//                13  carry-product issuer (lane 0); with 64-channel tiles also the fused products
//                    of the odd chunks of a state-only pass
//                 7, 11, 15       U group: U = k v over the k tile (elementwise)
//                 2, 6, 10, 14    S group: state rows 0..31 x NC/4 channels each; chain, publish, look-back
//                 4, 5, 8, 9      E group: token rows 0..63 x NC/2 channels each; gate and stage y
// Each role loops over the same item sequence and the same chunk order; they meet only at
// mbarriers, so loads, U, the products, the chain and the epilogue of different chunks overlap.
template <int NC, int LMAX>
__global__ void __launch_bounds__(kThreads, 1)
prefill_chunk_kernel(const __grid_constant__ LayerMaps<LMAX> m, const ChunkArgs a) {
    using G = Geo<NC>;
    constexpr int kNC = NC, kTile = G::kTile, kStageBytes = G::kStageBytes, kKVStages = G::kKVStages,
                  kQStages = G::kQStages, kSlots = G::kSlots, kSlotCols = G::kSlotCols, kSBytes = G::kSBytes,
                  kACol = G::kACol,
                  kSmQ = G::kSmQ, kSmS = G::kSmS, kSmBar = G::kSmBar, kSmMisc = G::kSmMisc;
    constexpr int kBarKVFull = G::kBarKVFull, kBarKVEmpty = G::kBarKVEmpty, kBarURdy = G::kBarURdy,
                  kBarQFull = G::kBarQFull, kBarQEmpty = G::kBarQEmpty, kBarYStaged = G::kBarYStaged,
                  kBarWDone = G::kBarWDone, kBarD2Free = G::kBarD2Free, kBarYDone = G::kBarYDone,
                  kBarD1Free = G::kBarD1Free, kBarSRdy = G::kBarSRdy, kBarSTFree = G::kBarSTFree,
                  kBarItemFull = G::kBarItemFull, kBarItemEmpty = G::kBarItemEmpty, kBarConst = G::kBarConst,
                  kBarConstFree = G::kBarConstFree, kBarPubFull = G::kBarPubFull, kBarPubEmpty = G::kBarPubEmpty,
                  kBarDrain = G::kBarDrain, kBarDrainC = G::kBarDrainC, kBarSOFin = G::kBarSOFin,
                  kBarAReady = G::kBarAReady, kNumBars = G::kNumBars;
    constexpr int kCh = kNC / 4;        // channels of one S-group thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int slot) { return sbase + kSmBar + 8u * slot; };
    volatile int *itemq = reinterpret_cast<volatile int *>(sm + kSmMisc);   // [kItemQ]
    volatile int *misc = itemq + kItemQ;                                     // abort, tmem, never
    volatile int *pubq = misc + 16;                                          // [kPubQ]: 4 item + code, -1 = end
    volatile int *carry_issued = pubq + kPubQ;                               // carries issued so far
    volatile int *so_items = carry_issued + 1;     // items whose state-only products of the carry issuer are done
    volatile int *abort = misc;
    volatile int *never = misc + 2;

    if (tid == 0) {
        misc[0] = 0;
        misc[2] = 0;
        *carry_issued = 0;
        *so_items = 0;
        for (int i = 0; i < kNumBars; ++i) tc::mbar_init(bar(i), G::count(i));
        tc::fence_mbar_init();
    } else if (tid == 32) {
        // the maps of the layer of this CTA's first item if its ticket is fixed, else of layer 0
        // (the others are fetched on first use)
        const int l0 = a.fixed_first ? (ticket_item(a, (int)blockIdx.x) / a.ih) / a.Hl : 0;
        tc::prefetch_tensormap(&m.q[l0]);
        tc::prefetch_tensormap(&m.k[l0]);
        tc::prefetch_tensormap(&m.v[l0]);
        tc::prefetch_tensormap(&m.y[l0]);
    }
    if (warp == kWarpMMA) {
        tc::tmem_alloc(tc::smem_u32((const void *)(misc + 1)), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    // Launched as a programmatic dependent of the constants kernel: the set-up above overlapped it.
    // The loaders and the U group touch only their inputs and shared memory, so they start at
    // once: each CTA's first item has a fixed ticket (blockIdx / H of head blockIdx % H), so its
    // tiles can be loaded and U formed while the constants are still being built.  Every other
    // role, and the k,v loader before its first counted ticket, waits here until the constants
    // and the cleared schedule words are visible.
    if (!(warp == kWarpKV || warp == kWarpQ || u_index(warp) >= 0)) asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t tmem = (uint32_t)misc[1];
    const int d = a.d;
    auto uni = [&](bool x) -> bool { return __all_sync(0xffffffffu, x && !*abort); };
    auto tok_of = [&](int chunk) { return a.tok_base + chunk * kC; };

    // The fused product [Z; W] = [T; V] U of iteration gi, once its U tile is formed and its slot
    // has been read out by the S group and, after the slot's last full-pass use, by the E group
    // (parity bits `c2bits` of the issuing thread); its commits mark the slot's product done and
    // free the k,v stage.  Issued by one lane (the fused issuer, or the carry issuer for the odd
    // chunks of a state-only pass); false if a wait gave up.
    auto fused_product = [&](int gi, int c2bits) -> bool {
        const int slot = gi % kSlots, st = gi % kKVStages;
        if (!tc::mbar_wait(bar(kBarURdy + st), (gi / kKVStages) & 1, abort) ||
            !tc::mbar_wait(bar(kBarD2Free + slot), ((gi / kSlots) & 1) ^ 1, abort) ||
            !tc::mbar_wait(bar(kBarD1Free + slot), ((c2bits >> slot) & 1) ^ 1, abort))
            return false;
        tc::tc_fence_after();
        const uint32_t idesc = tc::idesc_bf16(128, kNC, true);
        const uint32_t dcol = tmem + slot * kSlotCols;
        const uint32_t u_addr = sbase + kSmKV + st * kStageBytes;
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
            const uint64_t bdesc = tc::smem_desc_sw128(u_addr + ks * 2048, kAtom, 1024);
            if constexpr (G::kATmem)
                tc::mma_bf16_ta(dcol, tmem + kACol + 8 * ks, bdesc, idesc, ks > 0);
            else
                tc::mma_bf16(dcol, tc::smem_desc(sbase + kSmFA + ks * 256, 128, kC * 16), bdesc, idesc, ks > 0);
        }
        tc::mma_commit(bar(kBarWDone + slot));
        tc::mma_commit(bar(kBarKVEmpty + st));
        return true;
    };

    // consumer side of the item queue: the id of the k-th item (-1 at the end), or -2 on abort.
    // `lead` threads (one per consumer role or warp) release the slot after reading it.
    // Warp-wide callers (all 32 lanes) pass warpwide = true: every lane reads before lane 0 releases.
    auto take_item = [&](int k, bool warpwide) -> int {
        const int s = k % kItemQ;
        bool got = tc::mbar_wait(bar(kBarItemFull + s), (k / kItemQ) & 1, abort);
        if (warpwide) got = __all_sync(0xffffffffu, got);
        if (!got) return -2;
        const int id = itemq[s];
        if (warpwide) __syncwarp();
        if (!warpwide || lane == 0) tc::mbar_arrive(bar(kBarItemEmpty + s));
        return id;
    };

    if (warp == kWarpKV) {
        // ------------------------------------------------------------ k,v loads + tickets
        if (lane == 0) {
            int g = 0;
            bool ok = true, counted = false;
            const uint64_t pol_keep = tc::l2_policy_evict_last(), pol_drop = tc::l2_policy_evict_first();
            const int n_items = a.H * a.ih;
            for (int k = 0; ok; ++k) {
                const int s = k % kItemQ;
                if (!tc::mbar_wait(bar(kBarItemEmpty + s), ((k / kItemQ) & 1) ^ 1, abort)) {
                    ok = false;
                    break;
                }
                // One ticket counter for all items, handed out segment-major: all heads' first segments,
                // then all second segments, ..., so an item's predecessors always have lower tickets.
                // With unsplit sequences each CTA's first ticket is fixed (blockIdx.x) and the counter,
                // which the constants kernel clears, hands out the tickets after them; the first counted
                // ticket waits for that kernel.  With split sequences every ticket comes from the
                // counter, cleared before this launch.
                int t = -1;
                if (a.fixed_first && k == 0) {
                    t = (int)blockIdx.x;
                } else {
                    if (!counted) {
                        if (a.fixed_first) asm volatile("griddepcontrol.wait;" ::: "memory");
                        counted = true;
                    }
                    t = atomicAdd(a.tickets, 1) + (a.fixed_first ? (int)gridDim.x : 0);
                }
                const int id = t < n_items ? ticket_item(a, t) : -1;
                itemq[s] = id;
                tc::mbar_arrive(bar(kBarItemFull + s));
                if (id < 0) break;
                const Item it = decode_item<NC>(a, id);
                for (int i = 0; i < it.niter; ++i, ++g) {
                    const int chunk = it.ck0 + (i < it.n1 ? i : i - it.n1);
                    const int st = g % kKVStages;
                    if (!tc::mbar_wait(bar(kBarKVEmpty + st), ((g / kKVStages) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = sbase + kSmKV + st * kStageBytes;
                    tc::mbar_expect_tx(bar(kBarKVFull + st), kStageBytes);
                    // the state-only pass reads k, v that the full pass reads again soon: ask L2 to keep
                    // them; the full pass reads them for the last time
                    const uint64_t pol = i < it.n1 ? pol_keep : pol_drop;
                    for (int h = 0; h < kNC / 64; ++h) {
                        tc::tma_load_3d_hint(dst + h * kAtom, &m.k[it.layer], bar(kBarKVFull + st), it.c0 + 64 * h, tok_of(chunk),
                                             it.b, pol);
                        tc::tma_load_3d_hint(dst + kTile + h * kAtom, &m.v[it.layer], bar(kBarKVFull + st), it.c0 + 64 * h,
                                             tok_of(chunk), it.b, pol);
                    }
                }
            }
            if (!ok) {
                record_error(a, abort, kErrWait);
                // drain the loads still in flight before the CTA may exit
                for (int j = max(0, g - kKVStages); j < g; ++j)
                    tc::mbar_wait(bar(kBarKVFull + j % kKVStages), (j / kKVStages) & 1, never);
            }
        }
    } else if (warp == kWarpQ) {
        // ------------------------------------------------------------ q loads (full passes only)
        if (lane == 0) {
            int qg = 0;
            bool ok = true;
            const uint64_t pol_drop = tc::l2_policy_evict_first();
            for (int k = 0; ok; ++k) {
                const int id = take_item(k, false);
                if (id == -2) ok = false;
                if (id < 0) break;
                const Item it = decode_item<NC>(a, id);
                for (int j = 0; j < it.nck; ++j, ++qg) {
                    const int s = qg % kQStages;
                    if (!tc::mbar_wait(bar(kBarQEmpty + s), ((qg / kQStages) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_expect_tx(bar(kBarQFull + s), kTile);
                    for (int h = 0; h < kNC / 64; ++h)     // q is read once
                        tc::tma_load_3d_hint(sbase + kSmQ + s * kTile + h * kAtom, &m.q[it.layer], bar(kBarQFull + s),
                                             it.c0 + 64 * h, tok_of(it.ck0 + j), it.b, pol_drop);
                }
            }
            if (!ok) {
                record_error(a, abort, kErrWait);
                for (int j = max(0, qg - kQStages); j < qg; ++j)
                    tc::mbar_wait(bar(kBarQFull + j % kQStages), (j / kQStages) & 1, never);
            }
        }
    } else if (warp == kWarpStore) {
        // ------------------------------------------------------------ y stores
        if (lane == 0) {
            // each chunk's stores form one bulk group (empty for a chunk that starts before token 0,
            // whose rows the E group wrote directly); a staging buffer goes back to the q loader
            // once its group has been read, checked one chunk later so that two stores overlap
            int qg = 0, prev = -1;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int id = take_item(k, false);
                if (id == -2) ok = false;
                if (id < 0) break;
                const Item it = decode_item<NC>(a, id);
                for (int j = 0; j < it.nck; ++j, ++qg) {
                    const int s = qg % kQStages;
                    if (!tc::mbar_wait(bar(kBarYStaged + s), (qg / kQStages) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    const int tok = tok_of(it.ck0 + j);
                    if (tok >= 0)
                        for (int h = 0; h < kNC / 64; ++h)
                            tc::tma_store_3d(&m.y[it.layer], sbase + kSmQ + s * kTile + h * kAtom, it.c0 + 64 * h, tok, it.b);
                    tc::bulk_commit();
                    tc::bulk_wait_read<1>();        // every group but this one has been read
                    if (prev >= 0) tc::mbar_arrive(bar(kBarQEmpty + prev));
                    prev = s;
                }
            }
            tc::bulk_wait_read<0>();
            if (prev >= 0) tc::mbar_arrive(bar(kBarQEmpty + prev));
            if (!ok) record_error(a, abort, kErrWait);
            tc::bulk_wait<0>();     // every store of this CTA has completed
        } else if (lane == 1) {
            // publisher: after the S group has written a segment state (seen through the barrier),
            // one GPU-scope fence orders all of its rows before the status word that other CTAs poll
            for (int k = 0;; ++k) {
                const int ps = k % kPubQ;
                if (!tc::mbar_wait(bar(kBarPubFull + ps), (k / kPubQ) & 1, abort)) {
                    if (!*abort) record_error(a, abort, kErrWait);
                    break;
                }
                const int v = pubq[ps];
                if (v < 0) break;
                __threadfence();
                if ((v >> 2) != a.suppress_item && HB_OK(v >> 2, (long long)a.H * a.ih)) atomicExch(a.status + (v >> 2), v & 3);
                tc::mbar_arrive(bar(kBarPubEmpty + ps));
            }
        }
    } else if (warp == kWarpMMA) {
        // ------------------------------------------------------------ fused-product issuer
        // [Z; W] = [T; V] U for every iteration, in order.  Its waits only involve the U
        // operand and a free accumulator slot, so it runs ahead of the state chain; the carries
        // are issued by their own thread (a chunk's carry waits for that chunk's fused product,
        // onto which it adds, so the two threads need no other mutual order).  Waits suspend in
        // hardware (no polling loop on this thread).
        if (lane == 0) {
            int g = 0, pcf = 0, cur_hd = -1, cphase = 0, fphase = 0;
            int c2bits = 0;                 // bit s: parity of the full-pass uses of slot s issued so far
            int c2cnt[kSlots];              // per-slot full-pass uses (const switches only)
#pragma unroll
            for (int i = 0; i < kSlots; ++i) c2cnt[i] = 0;
            bool any = false, ok = true;
            for (int k = 0; ok; ++k) {
                const int id = take_item(k, false);
                if (id == -2) { ok = false; break; }
                if (id < 0) break;
                const Item it = decode_item<NC>(a, id);
                if (it.hd != cur_hd) {
                    // constants of a new head (consecutive tickets of a CTA may belong to different
                    // heads; the switch costs about one chunk's MMA issue, measured cheaper than
                    // keeping CTAs on one head).  No MMA may still read the old ones: every carry issued so far must be
                    // issued and finished (each slot then has at most one carry outstanding, so
                    // its last completion is unambiguous), and so must this thread's own MMAs.
                    if (any) {
                        const unsigned long long t0 = tc::global_ns();
                        const int so_need = G::kDualSO ? k : 0;
                        while ((*carry_issued < pcf || *so_items < so_need) && !*abort && tc::global_ns() - t0 < tc::kWaitNs) {}
                        if (*carry_issued < pcf || *so_items < so_need) { ok = false; break; }
#pragma unroll
                        for (int sl = 0; sl < kSlots; ++sl)
                            if (c2cnt[sl] > 0 && !tc::mbar_wait(bar(kBarYDone + sl), (c2cnt[sl] - 1) & 1, abort)) ok = false;
                        if (!ok) break;
                        tc::mma_commit(bar(kBarConstFree));
                        if (!tc::mbar_wait(bar(kBarConstFree), fphase & 1, abort)) { ok = false; break; }
                        ++fphase;
                    }
                    tc::mbar_expect_tx(bar(kBarConst), kOpBytes);
                    tc::bulk_load(sbase + kSmFA, a.consts + (size_t)HB_IDX(it.hd, a.H) * kConstStride, kOpBytes, bar(kBarConst));
                    if (!tc::mbar_wait(bar(kBarConst), cphase & 1, never)) { ok = false; break; }
                    ++cphase;
                    cur_hd = it.hd;
                    if constexpr (G::kATmem) {
                        // both A operands into tensor memory, one K = 16 slice (8 columns) per copy; the
                        // copies run in order with this thread's MMAs, and the commits that follow
                        // (seen by the carry issuer through WDone) cover them
                        tc::tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            tc::tmem_cp_128x256b(tmem + kACol + 8 * ks, tc::smem_desc(sbase + kSmFA + ks * 256, 128, kC * 16));
#pragma unroll
                        for (int ks = 0; ks < kKS / 16; ++ks)
                            tc::tmem_cp_128x256b(tmem + kACol + 32 + 8 * ks,
                                                 tc::smem_desc(sbase + kSmCA + ks * 256, 128, kKS * 16));
                    }
                    if constexpr (G::kDualSO) tc::mma_commit(bar(kBarAReady));   // for the carry issuer's state-only products
                }
                for (int i = 0; i < it.niter; ++i, ++g) {
                    if (G::kDualSO && i < it.n1 && (i & 1)) continue;     // the carry issuer's (state-only, odd)
                    const int slot = g % kSlots;
                    if (!fused_product(g, c2bits)) {
                        ok = false;
                        break;
                    }
                    if (i >= it.n1) {
                        c2bits ^= 1 << slot;
                        ++c2cnt[slot];
                        ++pcf;
                    }
                    any = true;
                }
            }
            if (*abort) ok = false;
            if (!ok) record_error(a, abort, kErrWait);
            // all MMAs issued by this thread have completed once `drain` fires
            tc::mma_commit(bar(kBarDrain));
            tc::mbar_wait(bar(kBarDrain), 0, never);
        }
    } else if (warp == kWarpCarry) {
        // ------------------------------------------------------------ carry issuer
        // Z += A S for every full-pass chunk, in order, once the S group has written the state
        // entering the chunk (after reading the chunk's W out of the slot) and the chunk's fused
        // product, onto which the carry adds, has finished.
        //
        // With the 64-channel tile it also issues the fused products of the odd iterations of a
        // state-only pass (the fused issuer takes the even ones), so that the two threads' issue
        // work overlaps.  Before the first of them it waits until the fused issuer has put the
        // item's head operands in place (one commit per head switch; the next switch cannot
        // complete before this item's state-only products are counted, so the phase is
        // unambiguous).  At the end of the pass it waits for its own products and counts the item,
        // which the fused issuer checks before it replaces the operands.
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16(128, kNC, true);
            int g = 0, pc = 0, sofin = 0, nsw = 0, cur_hd = -1;
            int c2bits = 0;                 // as the fused issuer's: parity of the full-pass uses of each slot
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int id = take_item(k, false);
                if (id == -2) { ok = false; break; }
                if (id < 0) break;
                const Item it = decode_item<NC>(a, id);
                if (it.hd != cur_hd) { cur_hd = it.hd; ++nsw; }
                if (G::kDualSO && it.n1 > 1) {
                    const int g0 = g;
                    if (!tc::mbar_wait(bar(kBarAReady), (nsw - 1) & 1, abort)) { ok = false; break; }
                    for (int i = 1; i < it.n1; i += 2)
                        if (!fused_product(g0 + i, c2bits)) {
                            ok = false;
                            break;
                        }
                    if (!ok) break;
                    tc::mma_commit(bar(kBarSOFin));
                    if (!tc::mbar_wait(bar(kBarSOFin), sofin & 1, abort)) { ok = false; break; }
                    ++sofin;
                }
                if constexpr (G::kDualSO) *so_items = k + 1;
                g += it.n1;
                for (int j = 0; j < it.nck; ++j, ++g, ++pc) {
                    const int slot = g % kSlots, sb = pc % kSBufs;
                    if (!tc::mbar_wait(bar(kBarSRdy + sb), (pc / kSBufs) & 1, abort) ||
                        !tc::mbar_wait(bar(kBarWDone + slot), (g / kSlots) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t dcol = tmem + slot * kSlotCols;     // onto the fused product
                    const uint32_t sb_addr = sbase + kSmS + sb * kSBytes;
#pragma unroll
                    for (int ks = 0; ks < kKS / 16; ++ks) {
                        const uint64_t bdesc = tc::smem_desc_sw128(sb_addr + ks * 2048, kKS * 128, 1024);
                        if constexpr (G::kATmem)
                            tc::mma_bf16_ta(dcol, tmem + kACol + 32 + 8 * ks, bdesc, idesc, 1);
                        else
                            tc::mma_bf16(dcol, tc::smem_desc(sbase + kSmCA + ks * 256, 128, kKS * 16), bdesc, idesc, 1);
                    }
                    tc::mma_commit(bar(kBarYDone + slot));
                    tc::mma_commit(bar(kBarSTFree + sb));
                    *carry_issued = pc + 1;
                    c2bits ^= 1 << slot;
                }
            }
            if (*abort) ok = false;
            if (!ok) record_error(a, abort, kErrWait);
            tc::mma_commit(bar(kBarDrainC));
            tc::mbar_wait(bar(kBarDrainC), 0, never);
        }
    } else if (u_index(warp) >= 0) {
        // ------------------------------------------------------------ U group: U = k v in place
        const int ut = u_index(warp) * 32 + lane;       // 0 .. kUThreads - 1
        int g = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int id = take_item(k, true);
            if (id == -2) ok = false;
            if (id < 0) break;
            const Item it = decode_item<NC>(a, id);
            for (int i = 0; i < it.niter; ++i, ++g) {
                const int st = g % kKVStages;
                if (!(ok = uni(tc::mbar_wait(bar(kBarKVFull + st), (g / kKVStages) & 1, abort)))) break;
                uint8_t *kt = sm + kSmKV + st * kStageBytes;
                // state-only iterations: the E group takes part (it has no epilogue to run there);
                // full-pass iterations: the U group alone, thread 0 arriving for the E group too
                const bool shared = i < it.n1;
                if (shared) form_u<kTile, kUHelp>(kt, ut);
                else form_u<kTile, kUThreads>(kt, ut);
                tc::fence_proxy_async_smem();
                if (!shared && ut == 0) tc::mbar_arrive_cnt(bar(kBarURdy + st), 1 + kEThreads);
                else tc::mbar_arrive(bar(kBarURdy + st));
            }
        }
        if (!ok) record_error(a, abort, kErrWait);
    } else if (is_s_warp(warp)) {
        // ------------------------------------------------------------ S group (state chain)
        // thread: state row r = lane (mode r % 16, Re for r < 16, Im above) for channels
        // kCh q4 .. kCh q4 + kCh - 1 of the tile; TMEM lane 64 + r holds row r of the state product W
        const int q4 = warp >> 2, r = lane, n = r & (kIm - 1);
        const bool leader = (warp == 2 && lane == 0);
        const float sgn = (r < kIm) ? -1.f : 1.f;
        const uint32_t lane_base = (uint32_t)64 << 16;
        int g = 0, pc = 0, pub_k = 0, cur_hd = -1;
        bool ok = true;
        float st[kCh];
        float2 lamC = make_float2(0.f, 0.f), lamS = lamC;
        // hand one entry to the publisher lane (all 128 threads call this after their writes)
        auto post = [&](int v) -> bool {
            const int ps = pub_k % kPubQ;
            bool res = true;
            if (leader) {
                res = tc::mbar_wait(bar(kBarPubEmpty + ps), ((pub_k / kPubQ) & 1) ^ 1, abort);
                pubq[ps] = res ? v : -1;
            }
            tc::mbar_arrive(bar(kBarPubFull + ps));
            ++pub_k;
            return res;
        };
        for (int k = 0; ok; ++k) {
            const int id = take_item(k, true);
            if (id == -2) ok = false;
            if (id < 0) break;
            const Item it = decode_item<NC>(a, id);
            if (it.hd != cur_hd) {
                const float2 *lp = reinterpret_cast<const float2 *>(a.consts + (size_t)HB_IDX(it.hd, a.H) * kConstStride + kLamOff);
                lamC = lp[n];               // zero for modes >= d
                lamS = lp[kMaxModes + n];
                cur_hd = it.hd;
            }
#pragma unroll
            for (int i = 0; i < kCh; ++i) st[i] = 0.f;

            // W of iteration gi out of its slot (then free for the next fused product)
            auto read_w = [&](int gi, float *w) -> bool {
                const int slot = gi % kSlots;
                if (!uni(tc::mbar_wait(bar(kBarWDone + slot), (gi / kSlots) & 1, abort))) return false;
                tc::tc_fence_after();
                tmem_ld<kCh>(tmem + lane_base + slot * kSlotCols + kCh * q4, w);
                tc::tmem_wait_ld();
                tc::tc_fence_before();
                tc::mbar_arrive(bar(kBarD2Free + slot));
                return true;
            };
            // st <- lambda^C st + W
            auto chain = [&](const float *w) {
#pragma unroll
                for (int i = 0; i < kCh; ++i) {
                    const float p = __shfl_xor_sync(0xffffffffu, st[i], 16);    // the other part of mode n
                    st[i] = fmaf(lamC.x, st[i], fmaf(sgn * lamC.y, p, w[i]));
                }
            };
            auto advance = [&](int gi) -> bool {
                float w[kCh];
                if (!read_w(gi, w)) return false;
                chain(w);
                return true;
            };
            // this thread's row of a published [32 rows][NC ch] state (bypassing L1); `item` is the
            // publishing item (checked against the item count in the bounds-checked build)
            auto load_rows = [&](const float *base, long long item, float *o) {
                const float *src = base + (size_t)HB_IDX(item, (long long)a.H * a.ih) * kKS * kNC;
                const float4 *p4 = reinterpret_cast<const float4 *>(src + (size_t)r * kNC + kCh * q4);
#pragma unroll
                for (int i = 0; i < kCh / 4; ++i) {
                    const float4 v4 = __ldcg(p4 + i);
                    o[4 * i] = v4.x; o[4 * i + 1] = v4.y; o[4 * i + 2] = v4.z; o[4 * i + 3] = v4.w;
                }
            };
            // write the state rows of this thread to dst [32 rows][NC ch] and hand `code` to the
            // publisher lane, which posts it once every row is written (no wait here)
            auto publish = [&](const float *v, float *base, int code) -> bool {
                float *dst = base + (size_t)HB_IDX(it.id, (long long)a.H * a.ih) * kKS * kNC;
                float4 *o = reinterpret_cast<float4 *>(dst + (size_t)r * kNC + kCh * q4);
#pragma unroll
                for (int i = 0; i < kCh / 4; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                return post(it.id * 4 + code);
            };

            // state-only pass over the segment, then publish its contribution
            for (int i = 0; i < it.n1 && ok; ++i, ++g) ok = uni(advance(g));
            if (!ok) break;
            if (it.n1 > 0 && !(ok = uni(publish(st, it.seg == 0 ? a.inc : a.agg, it.seg == 0 ? 2 : 1))))
                break;
            float sloc[kCh];
#pragma unroll
            for (int i = 0; i < kCh; ++i) { sloc[i] = st[i]; st[i] = 0.f; }

            // look-back: the state entering this segment.  The inclusive states follow the fixed
            // fp32 recurrence inc(s) = lambda^Lseg inc(s-1) + agg(s), inc(0) = agg(0): find the
            // nearest predecessor that has posted its inclusive state, then replay the recurrence
            // over the aggregates after it.  The result is bit-identical whichever predecessor
            // was found, so the output does not depend on timing.
            if (it.seg > 0) {
                int p0 = -1;
                const int units = a.units_h;
                for (int p = it.id - units; p >= it.id - it.seg * units; p -= units) {
                    int code = 0;
                    if (lane == 0 && HB_OK(p, (long long)a.H * a.ih)) {
                        code = ld_acquire(a.status + p);
                        const unsigned long long t0 = tc::global_ns();
                        while (code == 0 && !*abort && tc::global_ns() - t0 < a.lookback_ns) {
                            __nanosleep(64);
                            code = ld_acquire(a.status + p);
                        }
                    }
                    code = __shfl_sync(0xffffffffu, code, 0);
                    if (code == 0) break;
                    if (code == 2) { p0 = p; break; }
                }
                if (p0 < 0) {           // segment 0 always posts an inclusive state: only a timeout lands here
                    record_error(a, abort, kErrLookback);
                    ok = false;
                }
                if (!(ok = uni(ok))) break;
                __syncwarp();       // lane 0's acquire loads order the other lanes' reads below
                load_rows(a.inc, p0, st);
                for (int p = p0 + units; p < it.id; p += units) {
                    float ag[kCh];
                    load_rows(a.agg, p, ag);
#pragma unroll
                    for (int i = 0; i < kCh; ++i) st[i] = seg_step(st[i], ag[i], lamS, sgn);
                }
                if (it.n1 > 0) {
                    // inclusive state at the end of this segment (sloc is not needed after this)
#pragma unroll
                    for (int i = 0; i < kCh; ++i) sloc[i] = seg_step(st[i], sloc[i], lamS, sgn);
                    if (!(ok = uni(publish(sloc, a.inc, 2)))) break;
                }
            }

            // full pass: the chunk's W, then the state operand entering the chunk (which lets its
            // carry product add onto the slot), then the state after the chunk
            for (int j = 0; j < it.nck && ok; ++j, ++g, ++pc) {
                const int sb = pc % kSBufs;
                float w[kCh];
                if (!(ok = read_w(g, w))) break;
                if (!(ok = uni(tc::mbar_wait(bar(kBarSTFree + sb), ((pc / kSBufs) & 1) ^ 1, abort)))) break;
                // row r of the MN-major, 128-byte swizzled [32 rows][NC ch] operand: this thread's
                // channels are kCh * 2 bytes of row r in swizzle atom (kCh q4) / 64 (atoms of
                // 64 channels x 32 rows, 4 KB apart)
                constexpr int kC16 = kCh / 8;                       // 16-byte chunks of the thread
                const int cb = kCh * q4;
                uint8_t *sp = sm + kSmS + sb * kSBytes + (cb / 64) * (kKS * 128) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int i = 0; i < kC16; ++i) {
                    uint4 v;
                    v.x = pack_bf16(st[8 * i + 0], st[8 * i + 1]);
                    v.y = pack_bf16(st[8 * i + 2], st[8 * i + 3]);
                    v.z = pack_bf16(st[8 * i + 4], st[8 * i + 5]);
                    v.w = pack_bf16(st[8 * i + 6], st[8 * i + 7]);
                    *reinterpret_cast<uint4 *>(sp + (((((cb & 63) >> 3) + i) ^ (r & 7)) << 4)) = v;
                }
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(bar(kBarSRdy + sb));
                chain(w);
            }
            if (!ok) break;
            if (it.last_seg) {
                if constexpr (kCh == 32) {
                    // transpose the warp's 32 x 32 block (rows r in lanes -> channels in lanes) so
                    // that each lane writes the (Re, Im) pairs of one channel: coalesced float2 stores
                    warp_transpose32(st, lane);
                    const size_t s0 = ((size_t)it.b * d) * a.Dch + it.c0 + kCh * q4 + lane;
                    float2 *so = reinterpret_cast<float2 *>(m.state[it.layer]) + s0;
#pragma unroll
                    for (int m = 0; m < kMaxModes; ++m)
                        if (m < d && HB_OK(s0 + (size_t)m * a.Dch, (long long)(a.units_h / a.tph) * d * a.Dch))
                            so[(size_t)m * a.Dch] = make_float2(st[m], st[kIm + m]);
                } else {
                    // 16 channels: transpose each half-warp's 16 x 16 block; lane 16 h + i then holds
                    // part h (Re, Im) of every mode for channel i, and a warp store covers 16
                    // channels x (Re, Im) = 128 contiguous bytes
                    warp_transpose16x2(st, lane);
                    const size_t s0 = (((size_t)it.b * d) * a.Dch + it.c0 + kCh * q4 + (lane & 15)) * 2 + (lane >> 4);
                    float *so = m.state[it.layer] + s0;
#pragma unroll
                    for (int m = 0; m < kMaxModes; ++m)
                        if (m < d && HB_OK(s0 + (size_t)m * a.Dch * 2, (long long)(a.units_h / a.tph) * d * a.Dch * 2))
                            so[(size_t)m * a.Dch * 2] = st[m];
                }
            }
        }
        if (!ok) record_error(a, abort, kErrWait);
        post(-1);       // end of this CTA's posts
    } else if (is_e_warp(warp)) {
        // ------------------------------------------------------------ E group (gate and stage y)
        // thread: token row tau = 32 q4 + lane (TMEM lane tau) for channels NC/2 hh .. NC/2 (hh+1) - 1
        const int q4 = warp & 3, hh = warp >> 3, tau = 32 * q4 + lane;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        int g = 0, qg = 0;
        int e2bits = 0;             // bit s: parity of the full-pass uses of slot s consumed so far
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int id = take_item(k, true);
            if (id == -2) ok = false;
            if (id < 0) break;
            const Item it = decode_item<NC>(a, id);
            // state-only iterations: help the U group form U (threads kUThreads .. kUHelp - 1)
            for (int i = 0; i < it.n1 && ok; ++i, ++g) {
                const int st = g % kKVStages;
                if (!(ok = uni(tc::mbar_wait(bar(kBarKVFull + st), (g / kKVStages) & 1, abort)))) break;
                form_u<kTile, kUHelp>(sm + kSmKV + st * kStageBytes, kUThreads + 32 * e_index(warp) + lane);
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(bar(kBarURdy + st));
            }
            if (!ok) break;
            for (int j = 0; j < it.nck; ++j, ++g, ++qg) {
                const int slot = g % kSlots, s = qg % kQStages;
                ok = uni(tc::mbar_wait(bar(kBarYDone + slot), (e2bits >> slot) & 1, abort) &&
                         tc::mbar_wait(bar(kBarWDone + slot), (g / kSlots) & 1, abort) &&
                         tc::mbar_wait(bar(kBarQFull + s), (qg / kQStages) & 1, abort));
                if (!ok) break;
                e2bits ^= 1 << slot;
                tc::tc_fence_after();
                const int tok = tok_of(it.ck0 + j);
                const bool store_direct = tok < 0, row_valid = tok + tau >= 0;
                __nv_bfloat16 *yrow = m.yp[it.layer] + ((size_t)it.b * a.L + (row_valid ? tok + tau : 0)) * a.Dch + it.c0;
#pragma unroll
                for (int x = 0; x < kNC / 64; ++x) {
                    const int cbase = hh * (kNC / 2) + 32 * x;      // first of 32 channels
                    uint8_t *qrow = sm + kSmQ + s * kTile + (cbase / 64) * kAtom + tau * 128;
                    // the four q pieces (16 bytes = 8 channels each) are loaded before the tensor-memory
                    // reads and before any y piece overwrites its slot, so the round trips overlap
                    uint4 *qp[4], qvs[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int chunk16 = ((cbase & 63) >> 3) + i;
                        qp[i] = reinterpret_cast<uint4 *>(qrow + ((chunk16 ^ (tau & 7)) << 4));
                        qvs[i] = *qp[i];
                    }
                    float z[32];            // Z + carry: the carry product added onto the fused one
                    const uint32_t col = tmem + lane_base + slot * kSlotCols + cbase;
                    tc::tmem_ld32(col, z);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 qv = qvs[i];
                        const float *zz = z + 8 * i;
                        uint4 yv;
                        yv.x = pack_bf16(bf_lo(qv.x) * zz[0], bf_hi(qv.x) * zz[1]);
                        yv.y = pack_bf16(bf_lo(qv.y) * zz[2], bf_hi(qv.y) * zz[3]);
                        yv.z = pack_bf16(bf_lo(qv.z) * zz[4], bf_hi(qv.z) * zz[5]);
                        yv.w = pack_bf16(bf_lo(qv.w) * zz[6], bf_hi(qv.w) * zz[7]);
                        if (!store_direct)
                            *qp[i] = yv;
                        else if (row_valid && HB_OK(((long long)it.b * a.L + tok + tau) * a.Dch + it.c0 + cbase + 8 * i + 7,
                                                    (long long)(a.units_h / a.tph) * a.L * a.Dch))
                            *reinterpret_cast<uint4 *>(yrow + cbase + 8 * i) = yv;
                    }
                }
                tc::tc_fence_before();
                tc::mbar_arrive(bar(kBarD1Free + slot));
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(bar(kBarYStaged + s));
            }
        }
        if (!ok) record_error(a, abort, kErrWait);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == kWarpMMA) tc::tmem_dealloc(tmem, kTmemCols);
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

// [B][L][Dch] bf16 viewed as a 3-D tensor (Dch, L, B); box = 64 channels x C tokens x 1
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

constexpr size_t kTicketOff = 64;    // byte offset of the ticket counter in the schedule block

struct ChunkPlan {
    int nc, nchunks, nseg, segc, items;
    size_t consts_off, sched_off, status_off, agg_off, inc_off, total;
};

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kPlanSMs = 148;

// Channel tile and segment count.  Costs are in units of one 128-channel chunk pass: a pass of
// an NC-channel tile costs NC/128 plus a fixed 0.1, an item 1 more, and 6 more when its sequence
// is split (the state-only pass is counted in the work; the look-back and publication latency
// is the 6).  The estimated makespan is the larger of the even share and the largest item, plus
// half an item of tail when there are more items than SMs.  The narrow tile and unsplit
// sequences are preferred whenever they do not cost more.  `layers` independent layers of the
// same shape share one launch: their (sequence, tile) units add up.
ChunkPlan plan(int B, int L, int Dch, int H, int layers = 1) {
    ChunkPlan p{};
    p.nchunks = (L + kC - 1) / kC;
    const int ch = Dch / H;
    double best = 1e300;
    p.nc = ch % 128 == 0 ? 128 : 64;
    p.segc = p.nchunks > 0 ? p.nchunks : 1;
    for (int nc : {128, 64}) {
        if (ch % nc != 0) continue;
        const double units = (double)layers * B * (Dch / nc);
        const double pass = nc / 128.0 + 0.1;
        const int nch = p.nchunks > 0 ? p.nchunks : 1;
        for (int want = 1; want <= kMaxSeg && want <= nch; ++want) {
            const int segc = (nch + want - 1) / want;
            const int nseg = (nch + segc - 1) / segc;
            const double items = units * nseg;
            const double ovh = nseg > 1 ? 7.0 : 1.0;
            const double work = units * (nch + (double)(nseg - 1) * segc) * pass + items * ovh;
            const double ctas = items < kPlanSMs ? items : kPlanSMs;
            const double item_max = (nseg > 1 ? 2.0 * segc : (double)segc) * pass + ovh;
            double est = work / ctas > item_max ? work / ctas : item_max;
            if (items > kPlanSMs) est += 0.5 * item_max;
            if (est < best * (1 - 1e-9)) { best = est; p.nc = nc; p.segc = segc; }
        }
    }
    p.nseg = p.nchunks > 0 ? (p.nchunks + p.segc - 1) / p.segc : 1;
    p.items = (int)((long long)layers * B * (Dch / p.nc) * p.nseg);
    // status words and published segment states exist only when sequences are split
    const size_t split_items = p.nseg > 1 ? (size_t)p.items : 0;
    p.consts_off = 0;
    p.sched_off = al256((size_t)layers * H * kConstStride);
    p.status_off = p.sched_off + al256(kTicketOff + 4);
    p.agg_off = p.status_off + al256(split_items * 4);
    p.inc_off = p.agg_off + al256(split_items * kKS * p.nc * 4);
    p.total = p.inc_off + al256(split_items * kKS * p.nc * 4);
    return p;
}

// SM count of the current device (the persistent grid is at most one CTA per SM), cached per device
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

int sm_count() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return kPlanSMs;
    if (dev < kMaxDevices && (v = g_sm_count[dev].load(std::memory_order_relaxed)) > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return kPlanSMs;
    if (dev < kMaxDevices) g_sm_count[dev].store(v, std::memory_order_relaxed);
    return v;
}

// fault injection for tests (hyena_test_chunked_inject): applied to every later launch
std::atomic<int> g_inject_item{-1};
std::atomic<unsigned long long> g_inject_wait_ns{0};

}  // namespace

HYENA_BOUNDS_READER(prefill_chunked)

bool chunked_supported(int dtype, int Dch, int H, int d) {
    return dtype == HYENA_BF16 && H > 0 && Dch % H == 0 && (Dch / H) % 64 == 0 && d >= 1 && d <= kMaxModes;
}

size_t chunked_ws_bytes(int B, int L, int Dch, int H, int d, int layers) {
    (void)d;
    return plan(B, L, Dch, H, layers).total;
}

namespace {
template <int NC, int LMAX>
cudaError_t launch_tile(const LayerMaps<LMAX> &m, const ChunkArgs &a, int items, cudaStream_t s) {
    constexpr int smem = Geo<NC>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(prefill_chunk_kernel<NC, LMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = items < sm_count() ? items : sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, prefill_chunk_kernel<NC, LMAX>, m, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The constants kernel, then the main kernel, for `layers` layers of the same shape (LMAX >= layers).
template <int LMAX>
cudaError_t launch_group(int layers, const void *const *q, const void *const *k, const void *const *v, int B, int L,
                         int Dch, int H, int d, const float2 *const *lam, const float2 *const *R,
                         const float *const *Dskip, void *const *y, float *const *state_out, void *ws, cudaStream_t s) {
    const ChunkPlan p = plan(B, L, Dch, H, layers);
    uint8_t *w = static_cast<uint8_t *>(ws);
    // schedule words (error word, ticket counters, status words): with split sequences they are
    // cleared ahead of the constants kernel, so that every ticket can come from a counter at once
    const bool fixed_first = p.nseg == 1;
    const int nzero = (int)((p.agg_off - p.sched_off) / 4);
    cudaError_t e;
    if (!fixed_first && (e = cudaMemsetAsync(w + p.sched_off, 0, (size_t)nzero * 4, s)) != cudaSuccess) return e;
    ParamPtrs<LMAX> pp;
    LayerMaps<LMAX> m;
    for (int l = 0; l < LMAX; ++l) {
        const int j = l < layers ? l : 0;       // unused entries repeat layer 0
        pp.lam[l] = lam[j];
        pp.R[l] = R[j];
        pp.Dskip[l] = Dskip[j];
        m.yp[l] = static_cast<__nv_bfloat16 *>(y[j]);
        m.state[l] = state_out[j];
        if (l < layers && (!make_map(&m.q[l], q[l], B, L, Dch) || !make_map(&m.k[l], k[l], B, L, Dch) ||
                           !make_map(&m.v[l], v[l], B, L, Dch) || !make_map(&m.y[l], y[l], B, L, Dch)))
            return cudaErrorInvalidValue;
        if (l >= layers) {
            m.q[l] = m.q[0];
            m.k[l] = m.k[0];
            m.v[l] = m.v[0];
            m.y[l] = m.y[0];
        }
    }
    chunk_consts_kernel<LMAX><<<layers * H, kConstThreads, 0, s>>>(pp, H, d, p.segc * kC, w + p.consts_off,
                                                                 reinterpret_cast<int *>(w + p.sched_off),
                                                                 fixed_first ? nzero : 0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ChunkArgs a;
    a.L = L; a.Dch = Dch; a.d = d; a.ch = Dch / H; a.H = layers * H; a.Hl = H;
    a.tph = a.ch / p.nc; a.units_h = B * a.tph; a.ih = a.units_h * p.nseg;
    a.nchunks = p.nchunks; a.tok_base = L - p.nchunks * kC;
    a.nseg = p.nseg; a.segc = p.segc;
    a.consts = w + p.consts_off;
    a.sched = reinterpret_cast<int *>(w + p.sched_off);
    a.tickets = reinterpret_cast<int *>(w + p.sched_off + kTicketOff);
    a.status = reinterpret_cast<int *>(w + p.status_off);
    a.agg = reinterpret_cast<float *>(w + p.agg_off);
    a.inc = reinterpret_cast<float *>(w + p.inc_off);
    a.fixed_first = fixed_first ? 1 : 0;
    a.suppress_item = g_inject_item.load();
    const unsigned long long inj_ns = g_inject_wait_ns.load();
    a.lookback_ns = inj_ns ? inj_ns : tc::kWaitNs;
    return p.nc == 128 ? launch_tile<128, LMAX>(m, a, p.items, s) : launch_tile<64, LMAX>(m, a, p.items, s);
}
}  // namespace

cudaError_t launch_prefill_chunked(const void *q, const void *k, const void *v, int B, int L, int Dch,
                                   int H, int d, const float2 *lam, const float2 *R, const float *Dskip,
                                   void *y, float *state_out, void *ws, cudaStream_t s) {
    return launch_group<1>(1, &q, &k, &v, B, L, Dch, H, d, &lam, &R, &Dskip, &y, &state_out, ws, s);
}

int chunked_max_layers() { return kMaxGroupLayers; }

cudaError_t launch_prefill_chunked_layers(int layers, const void *const *q, const void *const *k,
                                          const void *const *v, int B, int L, int Dch, int H, int d,
                                          const float *const *lam, const float *const *R, const float *const *Dskip,
                                          void *const *y, float *const *state_out, void *ws, cudaStream_t s) {
    if (layers < 1 || layers > kMaxGroupLayers) return cudaErrorInvalidValue;
    const float2 *lam2[kMaxGroupLayers], *R2[kMaxGroupLayers];
    for (int l = 0; l < layers; ++l) {
        lam2[l] = reinterpret_cast<const float2 *>(lam[l]);
        R2[l] = reinterpret_cast<const float2 *>(R[l]);
    }
    return launch_group<kMaxGroupLayers>(layers, q, k, v, B, L, Dch, H, d, lam2, R2, Dskip, y, state_out, ws, s);
}

int chunked_error_offset(int B, int L, int Dch, int H, int d, int layers) {
    (void)d;
    return (int)(plan(B, L, Dch, H, layers).sched_off + 4);
}

void chunked_inject(int suppress_item, unsigned long long wait_ns) {
    g_inject_item.store(suppress_item);
    g_inject_wait_ns.store(wait_ns);
}

}  // namespace hyena
