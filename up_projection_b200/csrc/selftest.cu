// selftest.cu -- exercises the bounded-wait failure path on the device
// without any fault: a one-CTA kernel waits on an mbarrier that nothing ever
// completes, with a short bound; the wait gives up, the kernel records the
// timeout in its status word (as every product kernel does) and returns
// normally, so the context stays usable and the host sees SWIGLU_ERR_TIMEOUT
// from swiglu_sync_status.
#include "kernels.cuh"
#include "ptx.cuh"

namespace swiglu {

__device__ unsigned int g_selftest_status;

namespace {

__global__ void swiglu_selftest_wait_kernel(long long limit_cycles) {
    __shared__ __align__(8) unsigned long long bar_storage;
    const uint32_t bar = dev::smem_u32(&bar_storage);
    if (threadIdx.x != 0) return;
    dev::mbar_init(bar, 1);
    dev::fence_mbar_init();
    // Phase 0 of a fresh barrier with one expected arrival: nothing arrives.
    const long long t0 = clock64();
    bool done = false;
    while (!(done = dev::mbar_try_wait(bar, 0))) {
        if (clock64() - t0 > limit_cycles) break;
    }
    if (!done) atomicOr(&g_selftest_status, 1u);
}

}  // namespace

cudaError_t launch_selftest_wait(long long limit_cycles, cudaStream_t stream) {
    swiglu_selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_cycles);
    return cudaGetLastError();
}

cudaError_t selftest_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_selftest_status, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_selftest_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
