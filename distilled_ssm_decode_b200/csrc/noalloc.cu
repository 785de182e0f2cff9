// noalloc.cu -- hyena_prefill_noalloc: the FFT prefill without a caller-supplied workspace.
//
// Some callers cannot hand us scratch memory or allocate it at the point where
// they call: code behind a plugin or FFI boundary that only passes the tensors
// it was given and has no handle on the framework's allocator, latency-critical
// loops that must not risk the implicit device synchronisation a cudaMalloc or
// cudaFree can bring, and deployments whose device-memory budget is fixed when
// they start.  For them this entry point runs hyena_prefill with its scratch in
// a fixed array that lives in the library itself.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library holds kNoAllocScratchBytes of it until the process exits.  Host code
// must not use the array's name as a device address: the address is fetched
// with cudaGetSymbolAddress once per device (the first call on each device, with
// that device current) and cached for the life of the process (a cudaDeviceReset
// may move the array, so the entry point must not be used on a device after
// resetting it).  That first call may also load the module on the device, so
// make it before any stream capture.  All calls share the one
// array: calls whose work overlaps on the GPU (different streams, or different
// host threads on one device) race on it and must be serialised by the caller.
// The prefill overwrites everything it reads from the scratch, so no contents
// need clearing between calls.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_prefill_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on error).
void *scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

size_t hyena_prefill_noalloc_capacity(void) { return kNoAllocScratchBytes; }

int hyena_prefill_noalloc(const void *q, const void *k, const void *v, int dtype, int B, int L, int Dch,
                          int H, int d, int fft_len, const float *lambda, const float *R,
                          const float *Dskip, void *y, float *state_out, hyena_stream_t stream) {
    // an invalid shape reports 0 bytes here and is rejected by hyena_prefill itself
    const size_t need = hyena_prefill_workspace_bytes(B, L, Dch, H, d, fft_len);
    if (need > kNoAllocScratchBytes) return HYENA_ERR_CAPACITY;
    void *scratch = scratch_for_current_device();
    if (!scratch) return HYENA_ERR_CUDA;
    return hyena_prefill(q, k, v, dtype, B, L, Dch, H, d, fft_len, lambda, R, Dskip, y, state_out,
                         scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
