// dx_split_check.cu -- host-only check of the split tail of a dX-only fp32
// backward launch (dx_split_shape / dx_split_part with the round-robin
// schedule of the whole tiles): over every CTA's sequence, each whole tile
// [0, t0) is taken exactly once, each tail tile's 256-deep chunks
// [0, chunks) are covered by its parts exactly once with no empty part, a
// CTA takes at most one part and only after its whole tiles, the parts fit
// the grid (so the partial tiles of the workspace never exceed one per
// CTA), and a split happens exactly when some CTAs would otherwise idle in
// the last wave and two parts fit.  Sweeps tile counts, chunk counts and
// grid sizes.  Prints "ok <shapes checked>" or the first violation.
#include "../up_projection_b200/csrc/gemm_common.cuh"

#include <cstdio>
#include <vector>

int main() {
    using namespace swiglu::gemm;
    static const long long kTiles[] = {1, 2, 3, 7, 24, 37, 73, 74, 75, 147, 148, 149, 172, 221,
                                       222, 296, 320, 384, 1000, 2304};
    static const int kChunks[] = {1, 2, 3, 5, 6, 17, 108, 192, 1000};
    static const int kGrids[] = {1, 2, 3, 16, 132, 147, 148};
    long long n = 0;
    std::vector<int> whole, chunk_seen;
    for (long long T : kTiles)
        for (int C : kChunks)
            for (int G : kGrids) {
                const DxSplit s = dx_split_shape(T, C, G);
                const long long r = T % G;
                const bool expect = G >= 2 && C >= 2 && r != 0 &&
                                    (G / r < C ? G / r : C) >= 2;
                if ((s.parts > 0) != expect) {
                    std::printf("violation: split=%d expected %d (T=%lld C=%d G=%d)\n", s.parts,
                                expect ? 1 : 0, T, C, G);
                    return 1;
                }
                const long long t0 = s.parts > 0 ? s.t0 : T;
                if (s.parts > 0 && (t0 % G != 0 || t0 + s.tiles != T ||
                                    static_cast<long long>(s.tiles) * s.parts > G ||
                                    s.parts > C)) {
                    std::printf("violation: shape t0=%d tiles=%d parts=%d (T=%lld C=%d G=%d)\n",
                                s.t0, s.tiles, s.parts, T, C, G);
                    return 1;
                }
                const BwdSched sched = make_bwd_sched(static_cast<int>(t0), 0, G, C, 1);
                whole.assign(static_cast<size_t>(t0), 0);
                chunk_seen.assign(static_cast<size_t>(s.tiles) * (C > 0 ? C : 1), 0);
                for (int cta = 0; cta < G; ++cta) {
                    int seq = 0, kind = -1, t = -1;
                    while (bwd_tile_of(sched, cta, G, seq, kind, t)) {
                        if (kind != kTileDx || t < 0 || t >= t0 || t % G != cta) {
                            std::printf("violation: whole tile %d of CTA %d (T=%lld G=%d)\n", t,
                                        cta, T, G);
                            return 1;
                        }
                        ++whole[t];
                        ++seq;
                    }
                    if (s.parts > 0 && seq != sched.q) {
                        std::printf("violation: CTA %d has %d whole tiles, not %d\n", cta, seq,
                                    sched.q);
                        return 1;
                    }
                    int tt, cb, ce;
                    if (dx_split_part(s, cta, tt, cb, ce)) {
                        if (tt < s.t0 || tt >= s.t0 + s.tiles || cb < 0 || ce > C || cb >= ce) {
                            std::printf("violation: part of CTA %d: tile %d chunks [%d, %d)\n",
                                        cta, tt, cb, ce);
                            return 1;
                        }
                        for (int c = cb; c < ce; ++c)
                            ++chunk_seen[static_cast<size_t>(tt - s.t0) * C + c];
                    } else if (s.parts > 0 && cta < s.tiles * s.parts) {
                        std::printf("violation: CTA %d has no part\n", cta);
                        return 1;
                    }
                }
                for (long long t = 0; t < t0; ++t)
                    if (whole[t] != 1) {
                        std::printf("violation: whole tile %lld seen %d times (T=%lld G=%d)\n", t,
                                    whole[t], T, G);
                        return 1;
                    }
                for (size_t i = 0; i < chunk_seen.size() && s.parts > 0; ++i)
                    if (chunk_seen[i] != 1) {
                        std::printf("violation: tail tile %zu chunk %zu seen %d times\n", i / C,
                                    i % C, chunk_seen[i]);
                        return 1;
                    }
                ++n;
            }
    std::printf("ok %lld\n", n);
    return 0;
}
