// bwd_sched_check.cu -- host-only check that the backward GEMMs' static
// schedule (make_bwd_sched / bwd_tile_of) is an exact partition: over every
// CTA's tile sequence each dX tile and each dW tile appears exactly once,
// and a CTA's dX tiles all come before its dW tiles.  Sweeps tile counts,
// grid sizes and the dX / dW cost ratio, including the edge cases (no dX
// tiles, no dW tiles, more CTAs than tiles, phase 1 cut short by T_dw).
// Prints "ok <schedules checked>" or the first violation; exits non-zero.
#include "../up_projection_b200/csrc/gemm_common.cuh"

#include <cstdio>
#include <vector>

int main() {
    using namespace swiglu::gemm;
    static const int kTiles[] = {0, 1, 2, 7, 37, 147, 148, 149, 296, 320, 1000, 2304};
    static const int kGrids[] = {1, 2, 3, 16, 147, 148, 296};
    static const long long kCost[][2] = {{1, 1}, {2, 1}, {7, 2}, {1, 3}, {14336, 4096},
                                         {28672, 8192}, {100, 1}, {5, 0}};
    long long n = 0;
    std::vector<int> seen_dx, seen_dw;
    for (int T_dx : kTiles)
        for (int T_dw : kTiles)
            for (int G : kGrids)
                for (const auto &c : kCost) {
                    const BwdSched s = make_bwd_sched(T_dx, T_dw, G, c[0], c[1]);
                    seen_dx.assign(T_dx, 0);
                    seen_dw.assign(T_dw, 0);
                    for (int cta = 0; cta < G; ++cta) {
                        bool in_dw = false;
                        for (int seq = 0;; ++seq) {
                            int kind = -1, t = -1;
                            if (!bwd_tile_of(s, cta, G, seq, kind, t)) break;
                            if (seq > T_dx + T_dw) {
                                std::printf("violation: endless sequence T_dx=%d T_dw=%d G=%d\n",
                                            T_dx, T_dw, G);
                                return 1;
                            }
                            if (kind == kTileDx) {
                                if (in_dw || t < 0 || t >= T_dx) {
                                    std::printf("violation: dX tile %d of CTA %d (T_dx=%d T_dw=%d G=%d)\n",
                                                t, cta, T_dx, T_dw, G);
                                    return 1;
                                }
                                ++seen_dx[t];
                            } else if (kind == kTileDw) {
                                in_dw = true;
                                if (t < 0 || t >= T_dw) {
                                    std::printf("violation: dW tile %d of CTA %d (T_dx=%d T_dw=%d G=%d)\n",
                                                t, cta, T_dx, T_dw, G);
                                    return 1;
                                }
                                ++seen_dw[t];
                            } else {
                                std::printf("violation: tile kind %d\n", kind);
                                return 1;
                            }
                        }
                    }
                    for (int t = 0; t < T_dx; ++t)
                        if (seen_dx[t] != 1) {
                            std::printf("violation: dX tile %d seen %d times (T_dx=%d T_dw=%d G=%d c=%lld/%lld)\n",
                                        t, seen_dx[t], T_dx, T_dw, G, c[0], c[1]);
                            return 1;
                        }
                    for (int t = 0; t < T_dw; ++t)
                        if (seen_dw[t] != 1) {
                            std::printf("violation: dW tile %d seen %d times (T_dx=%d T_dw=%d G=%d c=%lld/%lld)\n",
                                        t, seen_dw[t], T_dx, T_dw, G, c[0], c[1]);
                            return 1;
                        }
                    ++n;
                }
    std::printf("ok %lld\n", n);
    return 0;
}
