// read_floor.cu -- the bench-only pure-read probe: how fast two weight
// buffers can be streamed from HBM into shared memory when nothing else is
// done with them (the "pure-read floor" the AstrAI page measures beside its
// fused kernel, swiglu_benchmark.md, "HBM re-measurement and kernel
// simplification").
//
// Built as the best plain stream measured on B200 with the decode's bytes
// per stage: four CTAs per SM, each owning a contiguous balanced share of
// 12 KB chunks of A and of B, one bulk copy per chunk into a two-stage ring
// (24 KB per stage: the A chunk and the B chunk), four warps that read each
// stage out of shared memory and release it.  Consecutive calls overlap under
// programmatic dependent launch: a call's CTAs start reading while the
// previous call finishes, and only the one output, a word per CTA in `sink`,
// waits for the preceding work on the stream.  Waits are bounded.
#include "kernels.cuh"
#include "ptx.cuh"

namespace swiglu {
namespace {

using namespace dev;

constexpr int kFloorThreads = 160;      // warp 0 copies, warps 1..4 read
constexpr int kFloorCtasPerSm = 4;
constexpr int kFloorRing = 2;
constexpr uint32_t kFloorChunk = 12 * 1024;
constexpr uint32_t kFloorStage = 2 * kFloorChunk;
constexpr uint32_t kFloorSmem = kFloorRing * kFloorStage + 64 + 1024;

__global__ void __launch_bounds__(kFloorThreads, kFloorCtasPerSm)
    read_floor_kernel(const uint8_t *__restrict__ A, const uint8_t *__restrict__ B,
                      int64_t bytes, uint32_t *__restrict__ sink) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (sbase - raw);
    const uint32_t bar_full = sbase + kFloorRing * kFloorStage;
    const uint32_t bar_empty = bar_full + 8 * kFloorRing;
    volatile int *abort_flag =
        reinterpret_cast<volatile int *>(gbase + kFloorRing * kFloorStage + 16 * kFloorRing);
    __shared__ uint32_t part[kFloorThreads / 32];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int64_t chunks = (bytes + kFloorChunk - 1) / kFloorChunk;
    const int64_t c_begin = chunks * blockIdx.x / gridDim.x;
    const int64_t c_end = chunks * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFloorRing; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    uint32_t acc = 0;
    bool failed = false;
    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int64_t issued = 0;
            for (int64_t c = c_begin; c < c_end; ++c) {
                if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                    failed = true;
                    break;
                }
                const int64_t off = c * kFloorChunk;
                const uint32_t n = static_cast<uint32_t>(
                    bytes - off < static_cast<int64_t>(kFloorChunk) ? bytes - off : kFloorChunk);
                const uint32_t st = sbase + stage * kFloorStage;
                mbar_arrive_expect_tx(bar_full + 8 * stage, 2 * n);
                bulk_load(st, A + off, n, bar_full + 8 * stage);
                bulk_load(st + kFloorChunk, B + off, n, bar_full + 8 * stage);
                ++issued;
                if (++stage == kFloorRing) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // never leave while a copy may still write shared memory
            for (int s = 0; s < kFloorRing; ++s) {
                if (issued > s) {
                    const int64_t uses = (issued - 1 - s) / kFloorRing + 1;
                    int never = 0;
                    (void)mbar_wait(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1),
                                    reinterpret_cast<volatile int *>(&never));
                }
            }
        }
    } else {
        int stage = 0;
        uint32_t phase = 0;
        const int t = threadIdx.x - 32;  // 0..127
        for (int64_t c = c_begin; c < c_end; ++c) {
            if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                failed = true;
                break;
            }
            const uint32_t st = sbase + stage * kFloorStage;
            const int64_t off = c * kFloorChunk;
            const uint32_t n = static_cast<uint32_t>(
                bytes - off < static_cast<int64_t>(kFloorChunk) ? bytes - off : kFloorChunk);
            for (uint32_t o = 16u * t; o < n; o += 16u * 128u) {
                const uint4 a = lds_v4(st + o), b = lds_v4(st + kFloorChunk + o);
                acc ^= a.x ^ a.w ^ b.x ^ b.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
            if (++stage == kFloorRing) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) part[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t x = failed ? 0xFFFFFFFFu : 0u;
        for (int w = 0; w < kFloorThreads / 32; ++w) x ^= part[w];
        // the only write: after the preceding work on the stream has finished
        asm volatile("griddepcontrol.wait;" ::: "memory");
        sink[blockIdx.x] = x;
    }
}

}  // namespace

int read_floor_grid(const DeviceInfo &dev) { return dev.sm_count * kFloorCtasPerSm; }

cudaError_t launch_read_floor(const void *A, const void *B, int64_t bytes, void *sink,
                              const DeviceInfo &dev, cudaStream_t stream) {
    static bool attr_set[64] = {};
    if (dev.device >= 0 && dev.device < 64 && !attr_set[dev.device]) {
        const cudaError_t e = cudaFuncSetAttribute(
            read_floor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFloorSmem);
        if (e != cudaSuccess) return e;
        attr_set[dev.device] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(read_floor_grid(dev));
    cfg.blockDim = dim3(kFloorThreads);
    cfg.dynamicSmemBytes = kFloorSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, read_floor_kernel,
                                             static_cast<const uint8_t *>(A),
                                             static_cast<const uint8_t *>(B), bytes,
                                             static_cast<uint32_t *>(sink));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace swiglu
