// gemm_common.cuh -- pieces shared by the two tcgen05 dual-GEMM kernels.
#pragma once

#include "ptx.cuh"

namespace swiglu {

namespace gemm {

// Tile raster: groups of `group` consecutive M tiles sweep all N tiles, so
// the ~148 tiles in flight at any time share a few row blocks of A and column
// blocks of B in L2; a group's A rows stay in L2 while B streams past them,
// so B is read from HBM once per group.
//
// The forward takes groups of 32 M tiles.  Measured on B200 at K = 4096,
// N = 14336 (ncu DRAM bytes read per launch, time): 16 M tiles: M = 4096
// 504 MB (1.88x the X + Wg + Wu bytes), M = 8192 1.01 GB (3.3x); 32: 272 MB
// (1.01x) and 552 MB (1.83x), 2.5-2.8 % faster; 64: 272 MB at M = 4096 but
// 2.42 GB at M = 8192 (the group's 67 MB of X no longer stays in L2 next to
// the output stream), 7 % slower there.  The backward GEMMs keep groups of
// 16 (with 32 their LLaMA-3 8B M = 8192 calls ran 2.6 % slower).
constexpr int kGroupMForward = 32;
constexpr int kGroupMBackward = 16;

template <int kGroupM>
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

// ---------------------------------------------------------------------------
// Static schedule of the backward GEMMs' tiles over the persistent CTAs, for
// one launch computing dX and/or dWg, dWu.  dX tiles are long (a 2N-deep
// reduction), dW tiles short (M-deep), so a CTA first takes its round-robin
// share of the dX tiles (T_dx = q G + r: CTAs below r take q + 1) and then
// fills with dW tiles in the order in which the CTAs become free:
//   phase 1: the CTAs with q dX tiles (nB = G - r of them) start dW one dX
//            tile's time earlier and take R1 = c_dx / c_dw rounds of dW tiles
//            alone: tile j * nB + b for round j, b their rank among them;
//   phase 2: from P1 = R1 * nB on, every CTA takes tile P1 + round * G + cta.
// It is an exact partition of the T_dw tiles (phase 1 covers [0, P1), phase 2
// the rest, each index once), fixed per launch (deterministic), and the dW
// tiles in flight at any time are neighbours in the raster (they share the
// operand blocks in L2).  With T_dw = 0 it is plain round-robin over dX, with
// T_dx = 0 over dW.
struct BwdSched {
    int T_dx, T_dw;   // tiles of each kind
    int q, r;         // T_dx = q * G + r
    int R1, nB, P1;   // phase 1: R1 rounds over nB CTAs, P1 = R1 * nB tiles
};

inline BwdSched make_bwd_sched(int T_dx, int T_dw, int G, long long c_dx, long long c_dw) {
    BwdSched s{};
    s.T_dx = T_dx;
    s.T_dw = T_dw;
    s.q = T_dx / G;
    s.r = T_dx % G;
    s.nB = G - s.r;
    s.R1 = (s.r > 0 && c_dw > 0) ? static_cast<int>(c_dx / c_dw) : 0;
    const long long p1 = static_cast<long long>(s.R1) * s.nB;
    s.P1 = static_cast<int>(p1 < T_dw ? p1 : T_dw);
    if (s.P1 < p1) s.R1 = (s.P1 + s.nB - 1) / s.nB;  // phase 1 cut short by T_dw
    return s;
}

enum : int { kTileDx = 0, kTileDw = 1 };

// The seq-th tile of CTA `cta` of G: returns false once the CTA is done.
// (Host-callable too, so that the partition can be checked without a GPU.)
__host__ __device__ __forceinline__ bool bwd_tile_of(const BwdSched &s, int cta, int G, int seq,
                                            int &kind, int &t) {
    const int ndx = s.q + (cta < s.r ? 1 : 0);
    if (seq < ndx) {
        kind = kTileDx;
        t = cta + seq * G;
        return true;
    }
    const int j = seq - ndx;
    long long idx;
    if (cta >= s.r && j < s.R1)
        idx = static_cast<long long>(j) * s.nB + (cta - s.r);
    else
        idx = static_cast<long long>(s.P1) +
              static_cast<long long>(cta < s.r ? j : j - s.R1) * G + cta;
    if (cta >= s.r && j < s.R1 && idx >= s.P1) return false;
    if (idx >= s.T_dw) return false;
    kind = kTileDw;
    t = static_cast<int>(idx);
    return true;
}

// Split tail of a dX-only launch (the fp32 backward): of T tiles over G
// CTAs, the r = T mod G beyond the whole waves (all T when T < G) are each
// split into `parts` runs of consecutive 256-deep chunks of their reduction,
// parts = min(G / r, chunks) so that every part has a CTA and a chunk.  The
// whole tiles [0, t0) go round-robin (make_bwd_sched(t0, 0, G, ..): t0 / G
// each); afterwards CTA `slot` < tiles * parts takes part slot mod parts of
// tail tile t0 + slot / parts.  parts = 0: no split (whole waves, or fewer
// than two parts possible).
struct DxSplit {
    int t0, tiles, parts, chunks;
};

__host__ __device__ __forceinline__ DxSplit dx_split_shape(long long T, int chunks, int G) {
    DxSplit s{0, 0, 0, chunks};
    if (T <= 0 || G < 2 || chunks < 2) return s;
    const long long r = T % G;
    if (r == 0) return s;
    long long parts = G / r;
    if (parts > chunks) parts = chunks;
    if (parts < 2) return s;
    s.t0 = static_cast<int>(T - r);
    s.tiles = static_cast<int>(r);
    s.parts = static_cast<int>(parts);
    return s;
}

// The tail tile t and its chunk range [c_begin, c_end) of part `slot`.
__host__ __device__ __forceinline__ bool dx_split_part(const DxSplit &s, int slot, int &t,
                                                       int &c_begin, int &c_end) {
    if (s.parts == 0 || slot < 0 || slot >= s.tiles * s.parts) return false;
    const int j = slot / s.parts, p = slot - j * s.parts;
    t = s.t0 + j;
    c_begin = static_cast<int>(static_cast<long long>(s.chunks) * p / s.parts);
    c_end = static_cast<int>(static_cast<long long>(s.chunks) * (p + 1) / s.parts);
    return true;
}

}  // namespace gemm
}  // namespace swiglu
