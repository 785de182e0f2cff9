/*
 * hyena.h -- C ABI of libhyena_b200: the gated modal long convolution on B200.
 *
 * The operator (order-2 Hyena block; "Hyena processes long sequences 100x
 * faster than FlashAttention", lequren.com, sections "Hyena層次結構" and
 * "Hyena塊": a long convolution whose filter is as long as the input, between
 * element-wise gates):
 *
 *     u_t = k_t * v_t,    z_t = sum_{j<=t} h_{t-j} u_j,    y_t = q_t * z_t
 *
 * with one filter per head shared by the head's Dch/H channels (weight tying,
 * "Laughing Hyena Distillery", nubint.ai review, "Proposed method", and the
 * abstract on the CoChat page), given in modal state-space form (the
 * low-order SSM extracted from each convolution, same sources):
 *
 *     h_0 = Dskip,    h_j = Re sum_{n<d} R_n lambda_n^(j-1)   (j >= 1, |lambda_n| < 1)
 *
 * and its O(d)-state recurrent form for generation ("Main findings": O(d)
 * memory and O(dK) time for K generated tokens):
 *
 *     y_t = q_t (Dskip u_t + Re sum_n R_n s_n),   then   s_n <- lambda_n s_n + u_t
 *     prompt state:  s_n = sum_{j<L} lambda_n^(L-1-j) u_j
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Channel c belongs to head c / (Dch / H); Dch must be a multiple of H.
 *  - Activations q, k, v, y: row-major [B][L][Dch] (prefill) or [B][Dch]
 *    (decode), channel innermost, dtype HYENA_F32 (float) or HYENA_BF16
 *    (bfloat16 bits).  All arithmetic is fp32; bf16 outputs are rounded to
 *    nearest-even once, on store.
 *  - Modal parameters (always fp32): lambda, R as [H][d][2] (re, im
 *    interleaved complex64), Dskip as [H].
 *  - Recurrent state: [B][d][Dch][2] complex64 (mode-major, channel
 *    innermost, re/im interleaved), so that one mode of consecutive channels
 *    is one contiguous run.
 *  - Every pointer is DEVICE memory of the current CUDA device, owned by the
 *    caller.  The library never allocates, frees or synchronises; work is
 *    enqueued on `stream` (NULL = the legacy default stream) and returns
 *    immediately.  Inputs must not alias outputs unless stated.
 *  - Arguments are validated on the host before anything is enqueued; a
 *    failed check returns a negative hyena_status and enqueues nothing.  A
 *    launch failure returns HYENA_ERR_CUDA.  Not checked (would need a device
 *    read): |lambda| < 1 and finiteness of the data.
 *  - Empty problems (B == 0, Dch == 0, or L == 0 for the convolution) are
 *    valid: nothing is read, and outputs that have no elements are left alone.
 *    A prefill with L == 0 writes a zero state.
 */
#ifndef HYENA_B200_H
#define HYENA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *hyena_stream_t;

typedef enum {
    HYENA_OK = 0,
    HYENA_ERR_ARG = -1,          /* NULL pointer, unknown dtype */
    HYENA_ERR_SHAPE = -2,        /* negative size, Dch % H != 0, fft_len too short / not 2^k, d out of range */
    HYENA_ERR_ALIGN = -3,        /* pointer not aligned as the layout requires */
    HYENA_ERR_WORKSPACE = -4,    /* workspace NULL or smaller than the query says */
    HYENA_ERR_UNSUPPORTED = -5,  /* valid operator, size outside what the library implements */
    HYENA_ERR_CUDA = -6,         /* a CUDA launch/runtime call failed */
    HYENA_ERR_CAPACITY = -7      /* problem needs more than the library's built-in scratch */
} hyena_status;

typedef enum {
    HYENA_F32 = 0,
    HYENA_BF16 = 1
} hyena_dtype;

/* Largest number of poles per head the kernels accept. */
#define HYENA_MAX_MODES 64

/* Human-readable text for a hyena_status value (static storage, never NULL). */
const char *hyena_status_string(int status);

/* ABI version of this header: (major << 16) | minor. */
int hyena_abi_version(void);

/*
 * Filter materialisation (modal form above; Laughing Hyena Distillery review,
 * "Proposed method").
 *   lambda, R : [H][d][2] fp32 device;  Dskip : [H] fp32 device
 *   h_out     : [H][L] fp32 device, h_out[hd][0] = Dskip[hd],
 *               h_out[hd][j] = Re sum_n R[hd][n] lambda[hd][n]^(j-1).
 * Powers are formed in fp64 (binary powering of lambda, then a short run of
 * multiplications), so lambda = 0 gives the 2-tap filter [Dskip, Re sum R].
 * Requires H >= 0, 1 <= d <= HYENA_MAX_MODES, L >= 0.
 */
int hyena_filter_from_modes(const float *lambda, const float *R, const float *Dskip,
                            int H, int d, int L, float *h_out, hyena_stream_t stream);

/*
 * Spectrum of each head's filter zero-padded to fft_len (the transform the
 * FFT long convolution multiplies by; "Hyena層次結構": fast convolution
 * without forming the full matrix):
 *   spec_out[hd][f] = sum_{j<L} h[hd][j] exp(-2 pi i j f / fft_len),  f = 0..fft_len/2
 *   h        : [H][L] fp32 device
 *   spec_out : [H][fft_len/2+1][2] fp32 device (complex64)
 * fft_len must be a power of two >= L; the library implements 64 <= fft_len
 * <= 2^17 (HYENA_ERR_UNSUPPORTED otherwise).
 * workspace: device scratch of hyena_filter_spectrum_workspace_bytes() bytes,
 * 256-byte aligned.
 */
size_t hyena_filter_spectrum_workspace_bytes(int H, int L, int fft_len);
int hyena_filter_spectrum(const float *h, int H, int L, int fft_len, float *spec_out,
                          void *workspace, size_t ws_bytes, hyena_stream_t stream);

/*
 * Prefill by FFT long convolution: materialise the filter, transform it,
 * convolve each channel's u = k*v causally through a zero-padded FFT of
 * length fft_len, gate by q, and reduce the prompt to the recurrent state.
 *   q, k, v, y : [B][L][Dch] activations (dtype), y written
 *   state_out  : [B][d][Dch][2] fp32, overwritten with s_n = sum_j lambda_n^(L-1-j) u_j
 *                (summed over the last W tokens, W chosen per head from
 *                r = max|lambda| so that the older tokens weigh at most
 *                r^W/(1-r) max|u| <= 2^-40 max|u|, far below fp32 resolution)
 *   fft_len    : power of two, >= 2L-1 (so the circular convolution equals the
 *                linear one on the first L outputs).  Any such length gives the
 *                same result up to rounding; lengths below 64 are raised to 64
 *                internally.  The library implements fft_len <= 2^17, B <= 65535.
 *                fft_len <= 16384 runs one fused kernel per channel pair with
 *                the whole sequence in shared memory; longer transforms take a
 *                four-step route through the workspace.
 *   workspace  : device scratch, >= hyena_prefill_workspace_bytes(...) bytes,
 *                256-byte aligned; contents on entry are ignored.
 * Alignment: all activation pointers 4-byte aligned (bf16) / 8-byte (f32).
 * Routes.  Beyond 16384 points (the four-step route), the inner 8192-point
 * transforms of bf16 activations run on the tensor cores the same way.
 * bf16 activations with an internal FFT length of 4096, 8192 or 16384,
 * an even number of channels per head, Dch a multiple of 8 (of 4 at 16384)
 * and q, k, v, y aligned to 16 bytes (8 at 16384) run on the tensor cores: each
 * transform is factored as 64 x 64 x (N/4096) and its two 64-point DFT stages
 * are dense matrix products (a Monarch-style factorisation; bf16 operands,
 * fp32 accumulation, twiddles and the spectral product in fp32).  Measured on
 * the library's test shapes: y within about 5e-3 of max|y| (the bar for bf16
 * activations is 2e-2); the state is summed in fp32 from fp32 u over the last
 * 1024 prompt tokens and from bf16-rounded u before them.  Every other call
 * (fp32 activations, other lengths or layouts) runs the transforms on the CUDA
 * cores in fp32.  The tensor-core route waits on its own products with bounded
 * waits; if one gives up, the int at hyena_prefill_error_offset(...) bytes into
 * the workspace is nonzero after the call and y and state_out are not valid
 * (every call with L > 0 clears it first, whichever route it takes).
 */
size_t hyena_prefill_workspace_bytes(int B, int L, int Dch, int H, int d, int fft_len);
size_t hyena_prefill_error_offset(int B, int L, int Dch, int H, int d, int fft_len);
/* 1 if hyena_prefill with these arguments runs its DFT stages on the tensor cores
 * (all of them up to 16384 points; the inner 8192-point transforms of the
 * four-step route beyond), 0 if on the CUDA cores; HYENA_ERR_ARG / HYENA_ERR_SHAPE / HYENA_ERR_UNSUPPORTED as
 * hyena_prefill would return for invalid arguments.  Pointers are only
 * inspected for alignment.  Host-only (no CUDA call). */
int hyena_prefill_uses_tensor_cores(int dtype, int B, int L, int Dch, int H, int d, int fft_len,
                                    const void *q, const void *k, const void *v, const void *y);
int hyena_prefill(const void *q, const void *k, const void *v, int dtype,
                  int B, int L, int Dch, int H, int d, int fft_len,
                  const float *lambda, const float *R, const float *Dskip,
                  void *y, float *state_out,
                  void *workspace, size_t ws_bytes, hyena_stream_t stream);

/*
 * hyena_prefill without a caller-supplied workspace.  The pages have no
 * counterpart to this entry point: it exists for callers that cannot allocate
 * or pass device scratch where they call (a plugin or FFI layer that only sees
 * the tensors it was given, a latency-critical loop that must not risk the
 * device synchronisation of cudaMalloc/cudaFree, a fixed start-up memory
 * budget).  It runs hyena_prefill with its scratch in a fixed array inside the
 * library: hyena_prefill_noalloc_capacity() bytes (4 MiB), held on every GPU
 * that loads the library until the process exits.
 *   Arguments and results as hyena_prefill, minus the workspace.  It never
 *   calls cudaMalloc, cudaFree or any allocating routine.
 *   HYENA_ERR_CAPACITY when hyena_prefill_workspace_bytes(...) exceeds the
 *   capacity.  For fft_len <= 16384 that size is about 4*H*L + 8*H*fft_len
 *   bytes (the filter and the head spectra), so the limit depends on H and L
 *   as well: e.g. fft_len = 8192 and L = 4096 fit up to 51 heads, fft_len =
 *   16384 and L = 8192 up to 25; transforms longer than 16384 points need far
 *   more.  Check hyena_prefill_workspace_bytes() against
 *   hyena_prefill_noalloc_capacity() before relying on it.
 *   The first call on each device looks up the array's device address (with
 *   that device current) and may load the module there: make it before any
 *   stream capture.  The address is cached per device for the life of the
 *   process; after cudaDeviceReset on a device, do not call this entry point
 *   there again.  Every call uses the same array, so calls whose work
 *   overlaps on the GPU (other streams, other host threads) race on it; the
 *   caller must serialise them.  Nothing needs clearing between calls.
 */
size_t hyena_prefill_noalloc_capacity(void);
int hyena_prefill_noalloc(const void *q, const void *k, const void *v, int dtype,
                          int B, int L, int Dch, int H, int d, int fft_len,
                          const float *lambda, const float *R, const float *Dskip,
                          void *y, float *state_out, hyena_stream_t stream);

/*
 * Prefill by chunked modal evaluation on the tensor cores: the same operator
 * and outputs as hyena_prefill, computed as an exact regrouping of the causal
 * convolution.  Per chunk of 64 tokens, the intra-chunk part is a Toeplitz
 * product with the filter taps h_0..h_63 and the older tokens enter through the
 * recurrent state: z_t = sum_{j in chunk, j<=t} h_{t-j} u_j
 * + Re sum_n R_n lambda_n^(t-c0) s_n(c0), with s advanced chunk by chunk
 * (s(c0+C) = lambda^C s(c0) + sum_j lambda^(c0+C-1-j) u_j); the last state is
 * the prompt state.  (The "FFT (or chunked)" evaluation of the long
 * convolution; the carry is the distilled recurrence of "Laughing Hyena
 * Distillery", "Main findings".)  The products take bf16 operands (u = k v,
 * the taps, the powers and the state rounded to bf16) with fp32 accumulation;
 * the state chain itself runs in fp32.  Measured against an fp64 evaluation on
 * the library's test shapes: y within 6.5e-3 of max|y| (hyena_prefill: 3.3e-3,
 * its bf16 output rounding), the prompt state within 4e-3 of its maximum.
 * Chunks are aligned to the end of the prompt, so the last one ends at token L-1.
 *   Arguments as hyena_prefill, without fft_len.
 *   Implemented for: dtype HYENA_BF16, Dch/H a multiple of 64, d <= 16, all
 *   activation pointers 16-byte aligned; HYENA_ERR_UNSUPPORTED otherwise.
 *   workspace: >= hyena_prefill_chunked_workspace_bytes() bytes, 256-byte aligned.
 *   Calls on different streams may run at the same time (for instance independent
 *   layers), each with its own workspace.  Progress does not depend on how many
 *   SMs other work leaves free: a part of the kernel only waits for parts that
 *   are already running.
 *   The int32 at byte offset hyena_prefill_chunked_error_offset() of the
 *   workspace is 0 after a successful run; a nonzero value means a bounded
 *   wait inside the kernel gave up and the outputs are invalid: 1 = a pipeline
 *   wait (2 s), 2 = the wait for the state of an earlier segment of the same
 *   sequence.  Read it after synchronising the stream if needed.
 */
size_t hyena_prefill_chunked_workspace_bytes(int B, int L, int Dch, int H, int d);
size_t hyena_prefill_chunked_error_offset(int B, int L, int Dch, int H, int d);
int hyena_prefill_chunked(const void *q, const void *k, const void *v, int dtype,
                          int B, int L, int Dch, int H, int d,
                          const float *lambda, const float *R, const float *Dskip,
                          void *y, float *state_out,
                          void *workspace, size_t ws_bytes, hyena_stream_t stream);

/* Largest number of layers one hyena_prefill_chunked_layers call takes. */
#define HYENA_MAX_PREFILL_LAYERS 32

/*
 * hyena_prefill_chunked for `layers` independent operator layers of the same
 * shape in one launch (e.g. the 24 operator layers of a 1.3B-shaped
 * generation workload, each with its own prompt activations, modal filter and
 * state).  The results of layer i are those of hyena_prefill_chunked on layer
 * i's arguments; the layers' work items share one persistent grid, so no layer
 * pays its own start and end.  (The prefill of the "Laughing Hyena Distillery"
 * review, "Main findings": every layer hands its O(d) state to generation.)
 *   q, k, v, y, state_out, lambda, R, Dskip: HOST arrays of `layers` device
 *   pointers each, as hyena_prefill_chunked's arguments of each layer (read
 *   during the call only).  B, L, Dch, H, d and dtype are shared.
 *   0 <= layers <= HYENA_MAX_PREFILL_LAYERS (HYENA_ERR_UNSUPPORTED above).
 *   Implemented and aligned as hyena_prefill_chunked.  Layers must not share
 *   output buffers.
 *   workspace: >= hyena_prefill_chunked_layers_workspace_bytes() bytes, 256-byte
 *   aligned; its error word (hyena_prefill_chunked_layers_error_offset()) is 0
 *   after a successful run, as for hyena_prefill_chunked.
 */
size_t hyena_prefill_chunked_layers_workspace_bytes(int layers, int B, int L, int Dch, int H, int d);
size_t hyena_prefill_chunked_layers_error_offset(int layers, int B, int L, int Dch, int H, int d);
int hyena_prefill_chunked_layers(int layers, const void *const *q, const void *const *k, const void *const *v,
                                 int dtype, int B, int L, int Dch, int H, int d,
                                 const float *const *lambda, const float *const *R, const float *const *Dskip,
                                 void *const *y, float *const *state_out,
                                 void *workspace, size_t ws_bytes, hyena_stream_t stream);

/*
 * Bounds-checked build (no counterpart in the pages): libhyena_b200_dbg.so is
 * the same library compiled with every kernel checking the index of each
 * global load and store against the extent its arguments give that buffer.
 * The first index out of range in each source file is recorded and the access
 * is skipped (no trap, no fault).  This call waits for the device, then reads
 * and clears the records.  Returns 0 when no access was out of range, 1 when
 * one was, with record = {file, source line, index, extent} (file: 1 decode.cu,
 * 2 filter.cu, 3 fir.cu, 4 prefill_chunked.cu, 5 prefill_fft.cu, 6 state.cu,
 * 7 truncate.cu, 8 prefill_monarch.cu); HYENA_ERR_UNSUPPORTED from the release build, which has no
 * checks; HYENA_ERR_ARG for a NULL record.
 */
int hyena_debug_bounds_check(long long *record);

/*
 * Test hook (no counterpart in the pages): the next `n` calls of any entry
 * point that pass argument validation return HYENA_ERR_CUDA without enqueuing
 * anything, as if their launch had failed; 0 disarms it.  Lets a caller test
 * its handling of launch failures without a GPU fault (or without a GPU).
 * HYENA_ERR_ARG for n < 0.  Process-wide; meant for tests only.
 */
int hyena_test_fail_next_launches(int n);

/*
 * Test hook (no counterpart in the pages): fault injection for the bounded
 * waits of hyena_prefill_chunked, so that a test can make a wait run out
 * without any GPU fault.  Every later hyena_prefill_chunked launch in the
 * process skips posting the completion word of work item `suppress_item`
 * (-1: none), and bounds each wait for an earlier segment's state by
 * `lookback_limit_s` seconds (0: the default 2 s).  A launch whose sequences
 * are split into segments then ends with error word 2 instead of waiting
 * forever.  (-1, 0) restores normal operation.  HYENA_ERR_ARG for
 * suppress_item < -1 or a limit outside [0, 60].  Not thread-safe against
 * concurrent launches; meant for tests only.
 */
int hyena_test_chunked_inject(int suppress_item, double lookback_limit_s);

/*
 * Test hook (no counterpart in the pages): enable = 0 makes every later
 * hyena_prefill / hyena_prefill_noalloc call run its transforms on the CUDA
 * cores, also where the tensor-core route would apply (so that both routes
 * can be tested and timed on the same inputs); 1 (the default) restores the
 * automatic choice.  HYENA_ERR_ARG for other values.  Process-wide; meant for
 * tests and benchmarks only.
 */
int hyena_test_fft_tensor_cores(int enable);

/*
 * Prompt -> state reduction alone (the Vandermonde contraction over the
 * prompt; "Main findings": the O(d) state that generation continues from):
 *   state_out[b][n][c] = sum_{j<L} lambda[head(c)][n]^(L-1-j) k[b][j][c] v[b][j][c]
 *   k, v      : [B][L][Dch] (dtype)
 *   state_out : [B][d][Dch][2] fp32, overwritten (zero for L == 0); the same
 *               trailing-window rule as hyena_prefill applies.
 *   workspace : device scratch, 256-byte aligned, of
 *               hyena_prompt_state_workspace_bytes() bytes (partial states of
 *               prompt segments, summed in a fixed order: deterministic).
 */
size_t hyena_prompt_state_workspace_bytes(int B, int L, int Dch, int d);
int hyena_prompt_state(const void *k, const void *v, int dtype,
                       int B, int L, int Dch, int H, int d,
                       const float *lambda, float *state_out,
                       void *workspace, size_t ws_bytes, hyena_stream_t stream);

/*
 * One O(1) decode step for a batch of sequences (one token per call):
 *   y[b][c] = q[b][c] * (Dskip[h] u + Re sum_n R[h][n] s[b][n][c]),  u = k[b][c] v[b][c]
 *   then    s[b][n][c] <- lambda[h][n] s[b][n][c] + u
 * The output uses the state from before the update, so a prompt state from
 * hyena_prefill followed by decode steps reproduces the full-length
 * convolution.
 *   q, k, v, y : [B][Dch] (dtype);  state : [B][d][Dch][2] fp32, updated in place.
 * Alignment: state 8-byte aligned (16-byte for the vectorised path, taken when
 * Dch is even and all pointers allow it).
 */
int hyena_decode_step(const void *q, const void *k, const void *v, int dtype,
                      int B, int Dch, int H, int d,
                      const float *lambda, const float *R, const float *Dskip,
                      float *state, void *y, hyena_stream_t stream);

/* Largest number of layers one hyena_decode_step_layers call takes. */
#define HYENA_MAX_LAYERS 64

/*
 * One decode step (as hyena_decode_step) for `layers` independent operator
 * layers in a single launch, e.g. the 24 operator layers of a 1.3B-shaped
 * generation workload, whose tokens all advance by one at a time.  Layer i
 * has its own activations q[i], k[i], v[i], y[i] ([B][Dch], dtype), state[i]
 * ([B][d][Dch][2] fp32, updated in place) and modal parameters lambda[i],
 * R[i] ([H][d][2] fp32) and Dskip[i] ([H] fp32); B, Dch, H, d and dtype are
 * shared.  Each layer's results are those of hyena_decode_step on the same
 * arguments (up to the summation order of Re sum_n R_n s_n).  Per step this
 * is the O(d) recurrence of the distilled modal SSM ("Laughing Hyena
 * Distillery", nubint.ai review, "Main findings"), applied layer by layer.
 *   q, k, v, y, state, lambda, R, Dskip: HOST arrays of `layers` device
 *   pointers each (read during the call only; the pointers travel to the
 *   kernel by value, so a captured CUDA graph keeps them).
 *   0 <= layers <= HYENA_MAX_LAYERS (HYENA_ERR_UNSUPPORTED above).
 *   Implemented for Dch and Dch/H even (HYENA_ERR_UNSUPPORTED otherwise);
 *   every state pointer 16-byte aligned and every activation pointer aligned
 *   to two elements (HYENA_ERR_ALIGN otherwise).  Layers must not share state
 *   or output buffers.
 */
int hyena_decode_step_layers(int layers, const void *const *q, const void *const *k,
                             const void *const *v, int dtype, int B, int Dch, int H, int d,
                             const float *const *lambda, const float *const *R,
                             const float *const *Dskip, float *const *state, void *const *y,
                             hyena_stream_t stream);

/*
 * Undistilled decode baseline: one token by convolving the cached history with
 * the long filter, as generation works without the distilled recurrence.  Its
 * cost grows with the sequence (O(t) per token and O(t) cached activations per
 * channel), against O(d) for hyena_decode_step ("Laughing Hyena Distillery",
 * nubint.ai review, "Main findings"): it is the comparison point for that
 * claim, on the same hardware and with the same filter.
 *
 * hyena_fir_cache_prompt writes the history of a prompt:
 *   u_cache[b][j][c] = k[b][j][c] v[b][j][c] for j < L (fp32, exact for bf16 inputs)
 *   k, v    : [B][L][Dch] (dtype);  u_cache : [B][t_max][Dch] fp32, rows >= L untouched
 *   Requires t_max >= L.
 * hyena_fir_decode_step emits token t and appends it to the history:
 *   y[b][c] = q[b][c] (sum_{j<t} h[hd][t-j] u_cache[b][j][c] + h[hd][0] u),  u = k[b][c] v[b][c]
 *   then u_cache[b][t][c] = u.
 *   q, k, v, y : [B][Dch] (dtype);  h : [H][t_max] fp32 filter taps (for example from
 *   hyena_filter_from_modes with L = t_max);  rows 0..t-1 of u_cache must hold the history.
 *   Requires 0 <= t < t_max and B <= 65535.  Alignment: activations to their
 *   element size, h and u_cache to 4 bytes.
 * The sum over the history runs in fp32 in a fixed order (deterministic).
 */
int hyena_fir_cache_prompt(const void *k, const void *v, int dtype, int B, int L, int Dch, int t_max,
                           float *u_cache, hyena_stream_t stream);
int hyena_fir_decode_step(const void *q, const void *k, const void *v, int dtype, int B, int Dch, int H,
                          int t, int t_max, const float *h, float *u_cache, void *y,
                          hyena_stream_t stream);

/*
 * Modal truncation of each head's SSM to k modes (the model-order reduction
 * step of the distillation: balanced and modal truncation, "Laughing Hyena
 * Distillery", nubint.ai review, "Proposed method").  Mode n of a head adds
 * Re(R_n lambda_n^(j-1)) to tap j (j >= 1); the l1 norm of that is at most
 * score_n = |R_n| / (1 - |lambda_n|).  The k modes with the largest scores are
 * kept (equal scores: the lower index), in index order, so that
 * lambda_out, R_out with Dskip unchanged give the truncated filter.
 *   lambda, R          : [H][d][2] fp32 device (d <= HYENA_MAX_MODES, 0 <= k <= d)
 *   kept               : [H][k] int32 device, indices of the kept modes
 *   lambda_out, R_out  : [H][k][2] fp32 device (copies of the kept modes)
 *   bound              : [H] fp64 device, sum of the dropped scores: an upper
 *                        bound on sum_j |h_j - h'_j|, hence on max|dy| / max|u|
 *   err_l2             : [H] fp64 device, the exact l2 norm of the tap error
 *                        (sqrt sum_{j>=1} (h_j - h'_j)^2, summed in closed form
 *                        over pairs of dropped modes); +inf if a dropped mode has
 *                        |lambda| >= 1
 * kept, lambda_out and R_out may be NULL when k == 0.
 */
int hyena_modal_truncate(const float *lambda, const float *R, int H, int d, int k, int *kept,
                         float *lambda_out, float *R_out, double *bound, double *err_l2,
                         hyena_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* HYENA_B200_H */
