// hold_sms.cu -- test helper: occupy most SMs of the GPU for a bounded time.
//
// Each block takes enough shared memory that no CTA of the chunked prefill
// (about 200 KB of shared memory) fits next to it, and spins on the global
// timer until `ns` nanoseconds have passed, then exits.  It waits on nothing
// else, so it always ends.  Used to check that the chunked prefill makes
// progress when only a few SMs are free at its start.
#include <cuda_runtime.h>

extern "C" __global__ void hold_sms_kernel(unsigned long long ns) {
    extern __shared__ unsigned char pad[];
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    if (threadIdx.x == 0) pad[0] = 0;
    do {
        __nanosleep(2000);
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    } while (t - t0 < ns);
}

extern "C" int hold_sms(int blocks, unsigned long long ns, int smem_bytes, void *stream) {
    cudaError_t e = cudaFuncSetAttribute(hold_sms_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return (int)e;
    hold_sms_kernel<<<blocks, 32, smem_bytes, (cudaStream_t)stream>>>(ns);
    return (int)cudaGetLastError();
}

extern "C" int sm_count(void) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}
