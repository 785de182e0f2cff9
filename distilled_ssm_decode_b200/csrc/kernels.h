// kernels.h -- internal launchers of libhyena_b200 (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace hyena {

// Largest FFT handled by one CTA in shared memory; longer transforms take the
// four-step route through the workspace.
constexpr int kFusedMaxN = 16384;
// Size of the inner (shared-memory) transform of the four-step route.
constexpr int kFourStepN2 = 8192;
constexpr int kMaxFFT = 1 << 17;
// FFT lengths below this are raised to it internally (same result).
constexpr int kMinFFT = 64;

inline int fft_internal_len(int fft_len) { return fft_len < kMinFFT ? kMinFFT : fft_len; }

// filter.cu
// (block 0 also clears *clear when it is given)
cudaError_t launch_filter(const float2 *lam, const float2 *R, const float *Dskip,
                          int H, int d, int L, float *h, cudaStream_t s, int *clear = nullptr);

// prefill_fft.cu
size_t spectrum_ws_bytes(int H, int N);               // digit-reversed spectra (+ four-step scratch)
// scale multiplies the transform (1/N for the convolution, 1 for the plain DFT)
cudaError_t launch_spectrum_perm(const float *h, int H, int L, int N, float2 *spec_perm,
                                 float scale, cudaStream_t s);
cudaError_t launch_spectrum_natural(const float2 *spec_perm, int H, int N, float2 *out,
                                    cudaStream_t s);
size_t fourstep_ws_bytes(int B, int Dch, int ch, int N);
cudaError_t launch_prefill_fft(const void *q, const void *k, const void *v, int dtype,
                               int B, int L, int Dch, int H, int d, int N,
                               const float2 *spec_perm, const float2 *lam,
                               void *y, float *state_out, void *scratch, size_t scratch_bytes,
                               int *err, cudaStream_t s);

// spectrum for the tensor-core route: frequency k = k1 + 64 k2 + 4096 k3 stored per head in the
// order its lanes read it (N = 4096, 8192 or 16384; see spectrum_fused_kernel)
cudaError_t launch_spectrum_monarch(const float *h, int H, int L, int N, float2 *spec, float scale,
                                    cudaStream_t s);

// prefill_monarch.cu (FFT route on the tensor cores; bf16 activations)
// R3 = N / 4096 when the tensor-core route takes this call, else 0 (the CUDA-core route)
int monarch_r3(int dtype, int B, int L, int Dch, int H, int N, const void *q, const void *k, const void *v,
               const void *y);
void monarch_enable(int enable);
// the four-step route's inner 8192-point rows on the tensor cores (bf16 activations); specm holds
// each (head, k1) row's spectrum in the order fourstep_spec_tc_kernel writes
bool fourstep_tc_enabled();
cudaError_t launch_fourstep_inner_tc(float2 *Y, int N1, int ncols, int nslots, int paired, int ch, int H,
                                     const float2 *specm, int *err, cudaStream_t s);
cudaError_t launch_prefill_monarch(int r3, const void *q, const void *k, const void *v, int B, int L, int Dch,
                                   int H, int d, const float2 *spec, const float2 *lam, void *y,
                                   float *state_out, int *err, cudaStream_t s);

// prefill_chunked.cu (bf16 activations, heads of a multiple of 64 channels, d <= 16)
bool chunked_supported(int dtype, int Dch, int H, int d);
// workspace and error-word offset for `layers` layers of the same shape in one launch
size_t chunked_ws_bytes(int B, int L, int Dch, int H, int d, int layers = 1);
int chunked_error_offset(int B, int L, int Dch, int H, int d, int layers = 1);
int chunked_max_layers();
cudaError_t launch_prefill_chunked_layers(int layers, const void *const *q, const void *const *k,
                                          const void *const *v, int B, int L, int Dch, int H, int d,
                                          const float *const *lam, const float *const *R, const float *const *Dskip,
                                          void *const *y, float *const *state_out, void *ws, cudaStream_t s);
// fault injection for tests: suppress one item's status word (-1: none) and bound each look-back
// poll by wait_ns (0: the default bound); applies to every later launch
void chunked_inject(int suppress_item, unsigned long long wait_ns);
cudaError_t launch_prefill_chunked(const void *q, const void *k, const void *v, int B, int L, int Dch,
                                   int H, int d, const float2 *lam, const float2 *R, const float *Dskip,
                                   void *y, float *state_out, void *ws, cudaStream_t s);

// state.cu
size_t state_ws_bytes(int B, int L, int Dch, int d);
cudaError_t launch_prompt_state(const void *k, const void *v, int dtype, int B, int L, int Dch,
                                int H, int d, const float2 *lam, float *state_out,
                                void *scratch, cudaStream_t s);

// decode.cu
cudaError_t launch_decode_step(const void *q, const void *k, const void *v, int dtype,
                               int B, int Dch, int H, int d, const float2 *lam, const float2 *R,
                               const float *Dskip, float *state, void *y, cudaStream_t s);
// grouped step of `layers` independent layers (host arrays of device pointers); requires the
// paired-channel layout (decode_layers_vec_ok) and aligned pointers, checked by the caller
bool decode_layers_vec_ok(int Dch, int H);
cudaError_t launch_decode_layers(int layers, const void *const *q, const void *const *k, const void *const *v,
                                 int dtype, int B, int Dch, int H, int d, const float *const *lam,
                                 const float *const *R, const float *const *Dskip, float *const *state,
                                 void *const *y, cudaStream_t s);

// fir.cu (undistilled baseline: cached-activation long convolution per token)
cudaError_t launch_fir_fill(const void *k, const void *v, int dtype, int B, int L, int Dch, int t_max,
                            float *u_cache, cudaStream_t s);
cudaError_t launch_fir_step(const void *q, const void *k, const void *v, int dtype, int B, int Dch, int H, int t,
                            int t_max, const float *h, float *u_cache, void *y, cudaStream_t s);

// truncate.cu (modal truncation of each head's SSM)
cudaError_t launch_modal_truncate(const float2 *lam, const float2 *R, int H, int d, int k, int *kept,
                                  float2 *lam_out, float2 *R_out, double *bound, double *err_l2, cudaStream_t s);

// bounds-checked build: per source file, read and clear the record of the first global access
// out of range (see common.cuh); in the release build they report nothing
int bounds_read_decode(long long *rec);
int bounds_read_filter(long long *rec);
int bounds_read_fir(long long *rec);
int bounds_read_prefill_chunked(long long *rec);
int bounds_read_prefill_fft(long long *rec);
int bounds_read_prefill_monarch(long long *rec);
int bounds_read_state(long long *rec);
int bounds_read_truncate(long long *rec);

}  // namespace hyena
