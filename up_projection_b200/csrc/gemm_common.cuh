// gemm_common.cuh -- pieces shared by the two tcgen05 dual-GEMM kernels.
#pragma once

#include "ptx.cuh"

namespace swiglu {

namespace gemm {

// Tile raster: groups of kGroupM consecutive M tiles sweep all N tiles, so
// the ~148 tiles in flight at any time share a few X row blocks and weight
// column blocks in L2.
constexpr int kGroupM = 16;

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int &mt, int &nt) {
    const int per_group = kGroupM * num_n;
    const int grp = t / per_group;
    const int first_m = grp * kGroupM;
    const int gsize = min(num_m - first_m, kGroupM);
    const int r = t - grp * per_group;
    mt = first_m + r % gsize;
    nt = r / gsize;
}

// Bounded wait that ignores the abort flag (used while draining work that
// is already in flight).
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
    int never = 0;
    (void)dev::mbar_wait(bar, parity, reinterpret_cast<volatile int *>(&never));
}

}  // namespace gemm
}  // namespace swiglu
