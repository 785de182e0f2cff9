// abi.cu -- the extern "C" entry points of libhyena_b200 (declared in include/hyena.h).
//
// Every entry point validates its arguments on the host and returns a
// negative hyena_status before enqueuing anything when a check fails.  No
// entry point allocates, frees or synchronises; all work goes on `stream`.
#include <stdint.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

using namespace hyena;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

bool is_pow2(long long x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA; }

// Test hook (hyena_test_fail_next_launches): the next n calls that pass validation report a CUDA
// failure instead of enqueuing anything, as a failed launch would.
std::atomic<int> g_fail_launches{0};
bool injected_launch_failure() {
    int n = g_fail_launches.load();
    while (n > 0 && !g_fail_launches.compare_exchange_weak(n, n - 1)) {}
    return n > 0;
}
#define HYENA_LAUNCH_GUARD() \
    do {                     \
        if (injected_launch_failure()) return HYENA_ERR_CUDA; \
    } while (0)

int check_common(int H, int d, int Dch) {
    if (H < 1 || Dch < 0) return HYENA_ERR_SHAPE;
    if (Dch % H != 0) return HYENA_ERR_SHAPE;
    if (d < 1 || d > HYENA_MAX_MODES) return HYENA_ERR_SHAPE;
    return HYENA_OK;
}

// Prefill workspace layout: [h: H*L f32][spectra: H*N c64][four-step planes][state partials]
// [error word of the tensor-core route]
struct PrefillWs {
    size_t h_off, spec_off, four_off, state_off, err_off, total;
};

PrefillWs prefill_ws(int B, int L, int Dch, int H, int d, int fft_len) {
    PrefillWs w{};
    const int N = fft_internal_len(fft_len);
    const int ch = Dch / H;
    w.h_off = 0;
    w.spec_off = align_up((size_t)H * L * sizeof(float));
    w.four_off = w.spec_off + align_up(spectrum_ws_bytes(H, N));
    w.state_off = w.four_off + align_up(fourstep_ws_bytes(B, Dch, ch, N));
    // beyond 16384 points: the state partials, then the spectrum rows of the tensor-core inner kernel
    w.err_off = w.state_off + (N > kFusedMaxN ? align_up(state_ws_bytes(B, L, Dch, d)) + align_up(spectrum_ws_bytes(H, N)) : 0);
    w.total = w.err_off + kAlign;
    return w;
}

int check_prefill_shape(int B, int L, int Dch, int H, int d, int fft_len) {
    if (B < 0 || L < 0) return HYENA_ERR_SHAPE;
    int st = check_common(H, d, Dch);
    if (st != HYENA_OK) return st;
    if (!is_pow2(fft_len) || (long long)fft_len < 2LL * L - 1) return HYENA_ERR_SHAPE;
    if (fft_len > kMaxFFT) return HYENA_ERR_UNSUPPORTED;
    const int ch = Dch / H;
    const long long slots = (ch % 2 == 0) ? Dch / 2 : Dch;
    if (B > 65535) return HYENA_ERR_UNSUPPORTED;
    if (fft_internal_len(fft_len) > kFusedMaxN && (long long)B * slots > 65535) return HYENA_ERR_UNSUPPORTED;
    return HYENA_OK;
}

}  // namespace

extern "C" {

const char *hyena_status_string(int status) {
    switch (status) {
        case HYENA_OK: return "ok";
        case HYENA_ERR_ARG: return "invalid argument (null pointer or unknown dtype)";
        case HYENA_ERR_SHAPE: return "invalid shape (negative size, Dch % H != 0, d out of range, or bad fft_len)";
        case HYENA_ERR_ALIGN: return "pointer misaligned for the required layout";
        case HYENA_ERR_WORKSPACE: return "workspace missing or too small";
        case HYENA_ERR_UNSUPPORTED: return "size outside what the library implements";
        case HYENA_ERR_CUDA: return "CUDA launch or runtime error";
        case HYENA_ERR_CAPACITY: return "problem needs more scratch than the library's built-in array holds";
        default: return "unknown status";
    }
}

int hyena_abi_version(void) { return (1 << 16) | 0; }

int hyena_filter_from_modes(const float *lambda, const float *R, const float *Dskip, int H, int d,
                            int L, float *h_out, hyena_stream_t stream) {
    if (H < 0 || L < 0 || d < 1 || d > HYENA_MAX_MODES) return HYENA_ERR_SHAPE;
    if (H > 65535) return HYENA_ERR_UNSUPPORTED;
    if (H == 0 || L == 0) return HYENA_OK;
    if (!lambda || !R || !Dskip || !h_out) return HYENA_ERR_ARG;
    if (!aligned(lambda, 8) || !aligned(R, 8) || !aligned(Dskip, 4) || !aligned(h_out, 4))
        return HYENA_ERR_ALIGN;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_filter(reinterpret_cast<const float2 *>(lambda),
                                     reinterpret_cast<const float2 *>(R), Dskip, H, d, L, h_out,
                                     (cudaStream_t)stream));
}

size_t hyena_filter_spectrum_workspace_bytes(int H, int L, int fft_len) {
    if (H < 0 || L < 0 || !is_pow2(fft_len)) return 0;
    return align_up(spectrum_ws_bytes(H, fft_len));
}

int hyena_filter_spectrum(const float *h, int H, int L, int fft_len, float *spec_out, void *workspace,
                          size_t ws_bytes, hyena_stream_t stream) {
    if (H < 0 || L < 0 || !is_pow2(fft_len) || fft_len < L || fft_len < 2) return HYENA_ERR_SHAPE;
    if (fft_len < kMinFFT || fft_len > kMaxFFT || H > 65535) return HYENA_ERR_UNSUPPORTED;
    if (H == 0) return HYENA_OK;
    if (!h || !spec_out || !workspace) return HYENA_ERR_ARG;
    if (!aligned(h, 4) || !aligned(spec_out, 8) || !aligned(workspace, kAlign)) return HYENA_ERR_ALIGN;
    if (ws_bytes < hyena_filter_spectrum_workspace_bytes(H, L, fft_len)) return HYENA_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    float2 *perm = static_cast<float2 *>(workspace);
    HYENA_LAUNCH_GUARD();
    cudaError_t e = launch_spectrum_perm(h, H, L, fft_len, perm, 1.0f, s);
    if (e != cudaSuccess) return HYENA_ERR_CUDA;
    return cuda_status(launch_spectrum_natural(perm, H, fft_len, reinterpret_cast<float2 *>(spec_out), s));
}

size_t hyena_prefill_workspace_bytes(int B, int L, int Dch, int H, int d, int fft_len) {
    if (check_prefill_shape(B, L, Dch, H, d, fft_len) != HYENA_OK) return 0;
    return prefill_ws(B, L, Dch, H, d, fft_len).total;
}

int hyena_prefill(const void *q, const void *k, const void *v, int dtype, int B, int L, int Dch,
                  int H, int d, int fft_len, const float *lambda, const float *R, const float *Dskip,
                  void *y, float *state_out, void *workspace, size_t ws_bytes,
                  hyena_stream_t stream) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    int st = check_prefill_shape(B, L, Dch, H, d, fft_len);
    if (st != HYENA_OK) return st;
    if (B == 0 || Dch == 0) return HYENA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (!state_out || !lambda || !R || !Dskip) return HYENA_ERR_ARG;
    if (!aligned(state_out, 8) || !aligned(lambda, 8) || !aligned(R, 8) || !aligned(Dskip, 4))
        return HYENA_ERR_ALIGN;
    if (L == 0) {
        HYENA_LAUNCH_GUARD();
        return cuda_status(cudaMemsetAsync(state_out, 0, (size_t)B * d * Dch * 2 * sizeof(float), s));
    }
    if (!q || !k || !v || !y || !workspace) return HYENA_ERR_ARG;
    const size_t ab = (dtype == HYENA_BF16) ? 2 : 4;
    if (!aligned(q, 2 * ab) || !aligned(k, 2 * ab) || !aligned(v, 2 * ab) || !aligned(y, 2 * ab) ||
        !aligned(workspace, kAlign))
        return HYENA_ERR_ALIGN;
    const PrefillWs w = prefill_ws(B, L, Dch, H, d, fft_len);
    if (ws_bytes < w.total) return HYENA_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    float *h = reinterpret_cast<float *>(ws + w.h_off);
    float2 *spec = reinterpret_cast<float2 *>(ws + w.spec_off);
    const int N = fft_internal_len(fft_len);
    const float2 *lam2 = reinterpret_cast<const float2 *>(lambda);
    int *err = reinterpret_cast<int *>(ws + w.err_off);
    HYENA_LAUNCH_GUARD();
    // the filter kernel also clears the error word
    cudaError_t e = launch_filter(lam2, reinterpret_cast<const float2 *>(R), Dskip, H, d, L, h, s, err);
    if (e != cudaSuccess) return HYENA_ERR_CUDA;
    // the inverse transform is unnormalised: fold its 1/N into the spectrum
    const int r3 = monarch_r3(dtype, B, L, Dch, H, N, q, k, v, y);
    if (r3) {
        // tensor-core route: spectrum in its frequency order
        e = launch_spectrum_monarch(h, H, L, N, spec, 1.0f / (float)N, s);
        if (e != cudaSuccess) return HYENA_ERR_CUDA;
        return cuda_status(launch_prefill_monarch(r3, q, k, v, B, L, Dch, H, d, spec, lam2, y, state_out,
                                                  err, s));
    }
    e = launch_spectrum_perm(h, H, L, N, spec, 1.0f / (float)N, s);
    if (e != cudaSuccess) return HYENA_ERR_CUDA;
    e = launch_prefill_fft(q, k, v, dtype, B, L, Dch, H, d, N, spec, lam2, y, state_out,
                           ws + w.four_off, w.err_off - w.four_off, err, s);
    return cuda_status(e);
}

int hyena_prefill_uses_tensor_cores(int dtype, int B, int L, int Dch, int H, int d, int fft_len,
                                    const void *q, const void *k, const void *v, const void *y) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    const int st = check_prefill_shape(B, L, Dch, H, d, fft_len);
    if (st != HYENA_OK) return st;
    const int N = fft_internal_len(fft_len);
    if (monarch_r3(dtype, B, L, Dch, H, N, q, k, v, y) != 0) return 1;
    // beyond 16384 points the four-step route's inner transforms run on the tensor cores for bf16
    return (N > kFusedMaxN && dtype == HYENA_BF16 && fourstep_tc_enabled()) ? 1 : 0;
}

size_t hyena_prefill_error_offset(int B, int L, int Dch, int H, int d, int fft_len) {
    if (check_prefill_shape(B, L, Dch, H, d, fft_len) != HYENA_OK) return 0;
    return prefill_ws(B, L, Dch, H, d, fft_len).err_off;
}

int hyena_test_fft_tensor_cores(int enable) {
    if (enable != 0 && enable != 1) return HYENA_ERR_ARG;
    monarch_enable(enable);
    return HYENA_OK;
}

static int check_chunked(int dtype, int B, int L, int Dch, int H, int d) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    if (B < 0 || L < 0) return HYENA_ERR_SHAPE;
    int st = check_common(H, d, Dch);
    if (st != HYENA_OK) return st;
    if (B > 65535 || !chunked_supported(dtype, Dch, H, d)) return HYENA_ERR_UNSUPPORTED;
    return HYENA_OK;
}

size_t hyena_prefill_chunked_workspace_bytes(int B, int L, int Dch, int H, int d) {
    if (check_chunked(HYENA_BF16, B, L, Dch, H, d) != HYENA_OK) return 0;
    return chunked_ws_bytes(B, L, Dch, H, d);
}

size_t hyena_prefill_chunked_error_offset(int B, int L, int Dch, int H, int d) {
    if (check_chunked(HYENA_BF16, B, L, Dch, H, d) != HYENA_OK) return 0;
    return (size_t)chunked_error_offset(B, L, Dch, H, d);
}

int hyena_prefill_chunked(const void *q, const void *k, const void *v, int dtype, int B, int L, int Dch,
                          int H, int d, const float *lambda, const float *R, const float *Dskip, void *y,
                          float *state_out, void *workspace, size_t ws_bytes, hyena_stream_t stream) {
    int st = check_chunked(dtype, B, L, Dch, H, d);
    if (st != HYENA_OK) return st;
    if (B == 0 || Dch == 0) return HYENA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (!state_out || !lambda || !R || !Dskip) return HYENA_ERR_ARG;
    if (!aligned(state_out, 8) || !aligned(lambda, 8) || !aligned(R, 8) || !aligned(Dskip, 4))
        return HYENA_ERR_ALIGN;
    if (L == 0) {
        HYENA_LAUNCH_GUARD();
        return cuda_status(cudaMemsetAsync(state_out, 0, (size_t)B * d * Dch * 2 * sizeof(float), s));
    }
    if (!q || !k || !v || !y || !workspace) return HYENA_ERR_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(y, 16) || !aligned(workspace, kAlign))
        return HYENA_ERR_ALIGN;
    if (ws_bytes < chunked_ws_bytes(B, L, Dch, H, d)) return HYENA_ERR_WORKSPACE;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_prefill_chunked(q, k, v, B, L, Dch, H, d, reinterpret_cast<const float2 *>(lambda),
                                              reinterpret_cast<const float2 *>(R), Dskip, y, state_out,
                                              workspace, s));
}

int hyena_debug_bounds_check(long long *record) {
    if (!record) return HYENA_ERR_ARG;
    for (int i = 0; i < 4; ++i) record[i] = 0;
    if (!kBoundsChecked) return HYENA_ERR_UNSUPPORTED;
    // file ids as documented in hyena.h
    int (*const readers[])(long long *) = {bounds_read_decode, bounds_read_filter, bounds_read_fir,
                                           bounds_read_prefill_chunked, bounds_read_prefill_fft,
                                           bounds_read_state, bounds_read_truncate,
                                           bounds_read_prefill_monarch};
    int found = 0;
    for (int f = 0; f < 8; ++f) {
        long long rec[4];
        const int r = readers[f](rec);      // every record is read (and cleared), the first one kept
        if (r < 0) return HYENA_ERR_CUDA;
        if (r > 0 && !found) {
            found = 1;
            record[0] = f + 1;
            record[1] = rec[1];
            record[2] = rec[2];
            record[3] = rec[3];
        }
    }
    return found;
}

int hyena_test_fail_next_launches(int n) {
    if (n < 0) return HYENA_ERR_ARG;
    g_fail_launches.store(n);
    return HYENA_OK;
}

int hyena_test_chunked_inject(int suppress_item, double lookback_limit_s) {
    if (suppress_item < -1 || !(lookback_limit_s >= 0.0) || lookback_limit_s > 60.0) return HYENA_ERR_ARG;
    chunked_inject(suppress_item, (unsigned long long)(lookback_limit_s * 1e9));
    return HYENA_OK;
}

size_t hyena_prefill_chunked_layers_workspace_bytes(int layers, int B, int L, int Dch, int H, int d) {
    if (layers < 1 || layers > chunked_max_layers()) return 0;
    if (check_chunked(HYENA_BF16, B, L, Dch, H, d) != HYENA_OK) return 0;
    return chunked_ws_bytes(B, L, Dch, H, d, layers);
}

size_t hyena_prefill_chunked_layers_error_offset(int layers, int B, int L, int Dch, int H, int d) {
    if (layers < 1 || layers > chunked_max_layers()) return 0;
    if (check_chunked(HYENA_BF16, B, L, Dch, H, d) != HYENA_OK) return 0;
    return (size_t)chunked_error_offset(B, L, Dch, H, d, layers);
}

int hyena_prefill_chunked_layers(int layers, const void *const *q, const void *const *k, const void *const *v,
                                 int dtype, int B, int L, int Dch, int H, int d, const float *const *lambda,
                                 const float *const *R, const float *const *Dskip, void *const *y,
                                 float *const *state_out, void *workspace, size_t ws_bytes, hyena_stream_t stream) {
    if (layers < 0) return HYENA_ERR_SHAPE;
    if (layers > chunked_max_layers()) return HYENA_ERR_UNSUPPORTED;
    int st = check_chunked(dtype, B, L, Dch, H, d);
    if (st != HYENA_OK) return st;
    if (layers == 0 || B == 0 || Dch == 0) return HYENA_OK;
    if (!state_out || !lambda || !R || !Dskip) return HYENA_ERR_ARG;
    for (int i = 0; i < layers; ++i) {
        if (!state_out[i] || !lambda[i] || !R[i] || !Dskip[i]) return HYENA_ERR_ARG;
        if (!aligned(state_out[i], 8) || !aligned(lambda[i], 8) || !aligned(R[i], 8) || !aligned(Dskip[i], 4))
            return HYENA_ERR_ALIGN;
    }
    cudaStream_t s = (cudaStream_t)stream;
    if (L == 0) {
        HYENA_LAUNCH_GUARD();
        for (int i = 0; i < layers; ++i) {
            const cudaError_t e = cudaMemsetAsync(state_out[i], 0, (size_t)B * d * Dch * 2 * sizeof(float), s);
            if (e != cudaSuccess) return HYENA_ERR_CUDA;
        }
        return HYENA_OK;
    }
    if (!q || !k || !v || !y || !workspace) return HYENA_ERR_ARG;
    for (int i = 0; i < layers; ++i) {
        if (!q[i] || !k[i] || !v[i] || !y[i]) return HYENA_ERR_ARG;
        if (!aligned(q[i], 16) || !aligned(k[i], 16) || !aligned(v[i], 16) || !aligned(y[i], 16)) return HYENA_ERR_ALIGN;
    }
    if (!aligned(workspace, kAlign)) return HYENA_ERR_ALIGN;
    if (ws_bytes < chunked_ws_bytes(B, L, Dch, H, d, layers)) return HYENA_ERR_WORKSPACE;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_prefill_chunked_layers(layers, q, k, v, B, L, Dch, H, d, lambda, R, Dskip, y, state_out,
                                                     workspace, s));
}

size_t hyena_prompt_state_workspace_bytes(int B, int L, int Dch, int d) {
    if (B < 0 || L < 0 || Dch < 0 || d < 1 || d > HYENA_MAX_MODES) return 0;
    return align_up(state_ws_bytes(B, L, Dch, d));
}

int hyena_prompt_state(const void *k, const void *v, int dtype, int B, int L, int Dch, int H, int d,
                       const float *lambda, float *state_out, void *workspace, size_t ws_bytes,
                       hyena_stream_t stream) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    if (B < 0 || L < 0) return HYENA_ERR_SHAPE;
    int st = check_common(H, d, Dch);
    if (st != HYENA_OK) return st;
    if (B > 65535) return HYENA_ERR_UNSUPPORTED;
    if (B == 0 || Dch == 0) return HYENA_OK;
    if (!state_out || !lambda) return HYENA_ERR_ARG;
    if (!aligned(state_out, 8) || !aligned(lambda, 8)) return HYENA_ERR_ALIGN;
    cudaStream_t s = (cudaStream_t)stream;
    if (L == 0) {
        HYENA_LAUNCH_GUARD();
        return cuda_status(cudaMemsetAsync(state_out, 0, (size_t)B * d * Dch * 2 * sizeof(float), s));
    }
    if (!k || !v || !workspace) return HYENA_ERR_ARG;
    const size_t ab = (dtype == HYENA_BF16) ? 2 : 4;
    if (!aligned(k, ab) || !aligned(v, ab) || !aligned(workspace, kAlign)) return HYENA_ERR_ALIGN;
    if (ws_bytes < hyena_prompt_state_workspace_bytes(B, L, Dch, d)) return HYENA_ERR_WORKSPACE;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_prompt_state(k, v, dtype, B, L, Dch, H, d,
                                           reinterpret_cast<const float2 *>(lambda), state_out,
                                           workspace, s));
}

int hyena_decode_step(const void *q, const void *k, const void *v, int dtype, int B, int Dch, int H,
                      int d, const float *lambda, const float *R, const float *Dskip, float *state,
                      void *y, hyena_stream_t stream) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    if (B < 0) return HYENA_ERR_SHAPE;
    int st = check_common(H, d, Dch);
    if (st != HYENA_OK) return st;
    if (B == 0 || Dch == 0) return HYENA_OK;
    if (!q || !k || !v || !y || !state || !lambda || !R || !Dskip) return HYENA_ERR_ARG;
    const size_t ab = (dtype == HYENA_BF16) ? 2 : 4;
    if (!aligned(q, ab) || !aligned(k, ab) || !aligned(v, ab) || !aligned(y, ab) ||
        !aligned(state, 8) || !aligned(lambda, 8) || !aligned(R, 8) || !aligned(Dskip, 4))
        return HYENA_ERR_ALIGN;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_decode_step(q, k, v, dtype, B, Dch, H, d,
                                          reinterpret_cast<const float2 *>(lambda),
                                          reinterpret_cast<const float2 *>(R), Dskip, state, y,
                                          (cudaStream_t)stream));
}

int hyena_decode_step_layers(int layers, const void *const *q, const void *const *k, const void *const *v,
                             int dtype, int B, int Dch, int H, int d, const float *const *lambda,
                             const float *const *R, const float *const *Dskip, float *const *state,
                             void *const *y, hyena_stream_t stream) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    if (B < 0 || layers < 0) return HYENA_ERR_SHAPE;
    if (layers > HYENA_MAX_LAYERS) return HYENA_ERR_UNSUPPORTED;
    int st = check_common(H, d, Dch);
    if (st != HYENA_OK) return st;
    if (layers == 0 || B == 0 || Dch == 0) return HYENA_OK;
    if (!q || !k || !v || !y || !state || !lambda || !R || !Dskip) return HYENA_ERR_ARG;
    if (!decode_layers_vec_ok(Dch, H)) return HYENA_ERR_UNSUPPORTED;
    const size_t ab = (dtype == HYENA_BF16) ? 2 : 4;
    for (int i = 0; i < layers; ++i) {
        if (!q[i] || !k[i] || !v[i] || !y[i] || !state[i] || !lambda[i] || !R[i] || !Dskip[i])
            return HYENA_ERR_ARG;
        if (!aligned(q[i], 2 * ab) || !aligned(k[i], 2 * ab) || !aligned(v[i], 2 * ab) ||
            !aligned(y[i], 2 * ab) || !aligned(state[i], 16) || !aligned(lambda[i], 8) ||
            !aligned(R[i], 8) || !aligned(Dskip[i], 4))
            return HYENA_ERR_ALIGN;
    }
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_decode_layers(layers, q, k, v, dtype, B, Dch, H, d, lambda, R, Dskip, state, y,
                                            (cudaStream_t)stream));
}

int hyena_fir_cache_prompt(const void *k, const void *v, int dtype, int B, int L, int Dch, int t_max,
                           float *u_cache, hyena_stream_t stream) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    if (B < 0 || L < 0 || Dch < 0 || t_max < L) return HYENA_ERR_SHAPE;
    if ((long long)B * L * Dch == 0) return HYENA_OK;
    if (!k || !v || !u_cache) return HYENA_ERR_ARG;
    const size_t ab = (dtype == HYENA_BF16) ? 2 : 4;
    if (!aligned(k, ab) || !aligned(v, ab) || !aligned(u_cache, 4)) return HYENA_ERR_ALIGN;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_fir_fill(k, v, dtype, B, L, Dch, t_max, u_cache, (cudaStream_t)stream));
}

int hyena_fir_decode_step(const void *q, const void *k, const void *v, int dtype, int B, int Dch, int H, int t,
                          int t_max, const float *h, float *u_cache, void *y, hyena_stream_t stream) {
    if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_ARG;
    if (B < 0 || H < 1 || Dch < 0 || Dch % H != 0 || t < 0 || t >= t_max) return HYENA_ERR_SHAPE;
    if (B > 65535) return HYENA_ERR_UNSUPPORTED;
    if (B == 0 || Dch == 0) return HYENA_OK;
    if (!q || !k || !v || !y || !h || !u_cache) return HYENA_ERR_ARG;
    const size_t ab = (dtype == HYENA_BF16) ? 2 : 4;
    if (!aligned(q, ab) || !aligned(k, ab) || !aligned(v, ab) || !aligned(y, ab) || !aligned(h, 4) ||
        !aligned(u_cache, 4))
        return HYENA_ERR_ALIGN;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_fir_step(q, k, v, dtype, B, Dch, H, t, t_max, h, u_cache, y, (cudaStream_t)stream));
}

int hyena_modal_truncate(const float *lambda, const float *R, int H, int d, int k, int *kept,
                         float *lambda_out, float *R_out, double *bound, double *err_l2,
                         hyena_stream_t stream) {
    if (H < 0 || d < 1 || d > HYENA_MAX_MODES || k < 0 || k > d) return HYENA_ERR_SHAPE;
    if (H == 0) return HYENA_OK;
    if (!lambda || !R || !bound || !err_l2 || (k > 0 && (!kept || !lambda_out || !R_out))) return HYENA_ERR_ARG;
    if (!aligned(lambda, 8) || !aligned(R, 8) || !aligned(bound, 8) || !aligned(err_l2, 8) ||
        (k > 0 && (!aligned(kept, 4) || !aligned(lambda_out, 8) || !aligned(R_out, 8))))
        return HYENA_ERR_ALIGN;
    HYENA_LAUNCH_GUARD();
    return cuda_status(launch_modal_truncate(reinterpret_cast<const float2 *>(lambda),
                                             reinterpret_cast<const float2 *>(R), H, d, k, kept,
                                             reinterpret_cast<float2 *>(lambda_out),
                                             reinterpret_cast<float2 *>(R_out), bound, err_l2,
                                             (cudaStream_t)stream));
}

}  // extern "C"

