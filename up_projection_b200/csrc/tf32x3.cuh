// tf32x3.cuh -- pieces shared by the 3xTF32 kernels (the fp32 forward and the
// fp32 backward GEMMs): the hi/lo split of an operand stage and the
// round-to-nearest fold of a finished accumulation chunk.
//
//   a = hi + lo,  hi = trunc_tf32(a),  lo = rna_tf32(a - hi);  a*b is formed
//   as hi*hi + hi*lo + lo*hi on the tensor cores (Markidis et al. 2018;
//   Ootomo & Yokota 2022, written from the mathematics).
//
// hi is the raw fp32 operand as TMA landed it: a kind::tf32 MMA reads only
// the top 19 bits of each 32-bit element (sign, exponent, 10 mantissa bits),
// i.e. trunc_tf32(a), so only lo has to be written.  That saves a third of
// the split's shared-memory stores, on kernels whose limit is shared-memory
// traffic (B200, LLaMA-2 13B M = 2048: forward 2.84 -> 2.46 ms, dX 2.83 ->
// 2.54 ms).  a - trunc(a) is exact (the 13 low mantissa bits), and its
// rounding to tf32 leaves |a - hi - lo| <= 2^-21 |a| (rounding hi instead
// gives 2^-22): still far inside the 1e-5 bound.  Were the tensor core to
// round or keep more of a, hi + lo would miss a by up to 2^-11 |a| and every
// fp32 parity test would fail by orders of magnitude.
//
// The tensor cores' fp32 accumulation loses up to about one unit in the last
// place of the running sum per accumulate step, an error linear in the
// reduction length; so the reduction is cut into chunks that accumulate from
// zero in TMEM, and each finished chunk is added to a running sum in TMEM with
// round-to-nearest fp32 adds on the CUDA cores.
#pragma once

#include "ptx.cuh"

namespace swiglu {
namespace tf32x3 {

__device__ __forceinline__ uint32_t tf32_rna(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// lo of 4 fp32 values (hi is the value itself, read truncated by the MMA).
__device__ __forceinline__ void split4(const uint4 &v, uint4 &lo) {
    const uint32_t *pv = &v.x;
    uint32_t *pl = &lo.x;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(pv[i]);
        const float hi = __uint_as_float(pv[i] & 0xFFFFE000u);  // trunc_tf32(a)
        pl[i] = tf32_rna(a - hi);
    }
}

// One split thread's share of a raw stage of kRawBytes at `st`: the stage
// itself serves as hi; write lo at st + kRawBytes (same layout, so the same
// descriptors address both).  All loads first, then the splits and stores,
// so the shared-memory latency is paid once per stage.
template <uint32_t kRawBytes, int kThreadsSplit>
__device__ __forceinline__ void split_stage(uint32_t st, int sidx) {
    constexpr int kVecs = kRawBytes / 16;
    constexpr int kPerThread = kVecs / kThreadsSplit;
    static_assert(kVecs % kThreadsSplit == 0, "split work must divide evenly");
    uint4 x[kPerThread];
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) x[i] = dev::lds_v4(st + 16u * (sidx + i * kThreadsSplit));
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
        uint4 lo;
        split4(x[i], lo);
        const uint32_t off = 16u * (sidx + i * kThreadsSplit);
        dev::sts_v4(st + kRawBytes + off, lo);
    }
}

// Fold chunk `q` of a tile (kCols accumulator columns of this warp's 32 TMEM
// lanes) into the running sum: run = chunk for q == 0, else
// run = rn(run + chunk).  Ends with the stores complete.
template <int kCols>
__device__ __forceinline__ void fold_chunk(uint32_t chunk_acc, uint32_t run_acc, int q) {
#pragma unroll 1
    for (int col = 0; col < kCols; col += 32) {
        uint32_t c[32], r[32];
        dev::tmem_ld_32x32b_x32(chunk_acc + col, c);
        if (q > 0) dev::tmem_ld_32x32b_x32(run_acc + col, r);
        dev::tmem_ld_wait(c);
        if (q > 0) {
            dev::tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                c[i] = __float_as_uint(__fadd_rn(__uint_as_float(r[i]), __uint_as_float(c[i])));
        }
        dev::tmem_st_32x32b_x32(run_acc + col, c);
    }
    dev::tmem_st_wait();
}

}  // namespace tf32x3
}  // namespace swiglu
