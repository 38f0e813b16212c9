// decode_geometry_check.cu -- host-only check of the decode kernel's
// shared-memory geometry for every K it accepts (multiples of 8), both launch
// forms (plain; weights_stable with the two-CTAs-per-SM budget and the
// compact X layout), every M <= 8: the launch the kernel gets must fit the
// opt-in shared memory (and two CTAs per SM where the small budget is used),
// keep its TMA boxes within 256 per dimension and 16-byte aligned, keep every
// region 16-byte aligned and in order, and keep each stage's and X's
// transaction bytes below the mbarrier limit.  Prints "ok <launches
// checked>" or the first violation; exits non-zero.
#include "../up_projection_b200/csrc/decode_bf16.cu"

#include <cstdio>

namespace {

int fail(const char *what, int K, int M, int ws) {
    std::printf("violation: %s at K=%d M=%d weights_stable=%d\n", what, K, M, ws);
    return 1;
}

}  // namespace

int main() {
    using namespace swiglu;
    long long n = 0, supported = 0;
    for (int K = 8; K <= 65536; K += 8) {
        if (!decode_bf16_supported(K)) continue;
        ++supported;
        for (int ws = 0; ws < 2; ++ws)
            for (int M = 1; M <= 8; ++M) {
                // the launch's own choice of budget and X layout
                int budget = decode_budget(K, ws != 0, 8);
                Geometry g = geometry(K, budget, 8);
                int xrows = 8;
                if (ws && M < 8 && budget != kPdlSmemBudget &&
                    decode_budget(K, true, M) == kPdlSmemBudget) {
                    budget = kPdlSmemBudget;
                    xrows = M;
                    g = geometry(K, budget, M);
                }
                if (!g.ok) return fail("no geometry for a supported K", K, M, ws);
                if (g.smem > kMaxSmem) return fail("shared memory", K, M, ws);
                if (budget == kPdlSmemBudget && 2 * (g.smem + 1024) > 228 * 1024)
                    return fail("two CTAs per SM", K, M, ws);
                if (g.inner < 8 || g.inner > 256 || K % g.inner != 0 || g.kc % g.inner != 0 ||
                    g.kc / g.inner > 256)
                    return fail("TMA box", K, M, ws);
                if (g.stages < 2 || g.stages > kMaxStages) return fail("ring depth", K, M, ws);
                if (static_cast<long long>(g.slices) * g.kc < K || g.kx != g.slices * g.kc)
                    return fail("slices do not cover K", K, M, ws);
                // stage = [Wg box 8 x kc][Wu box 8 x kc]; X [xrows][kx]
                if ((32 * g.kc) % 16 != 0 || g.off_x != g.stages * 32 * g.kc ||
                    g.off_red < g.off_x + 2 * xrows * g.kx || g.off_bar < g.off_red + kRedBytes)
                    return fail("region order", K, M, ws);
                if (g.off_x % 16 != 0 || g.off_red % 16 != 0 || g.off_bar % 8 != 0 ||
                    (2 * g.kx) % 16 != 0)
                    return fail("alignment", K, M, ws);
                if (32 * g.kc >= (1 << 20) || 2 * M * K >= (1 << 20))
                    return fail("transaction bytes", K, M, ws);
                if (g.smem < g.off_bar + 8 * kNumBars + 16 + 1024)
                    return fail("barriers past the allocation", K, M, ws);
                ++n;
            }
    }
    // the largest supported K stages 8 rows of X (16 K bytes) in the opt-in limit
    if (supported < 1000 || decode_bf16_supported(65536)) {
        std::printf("violation: supported range\n");
        return 1;
    }
    std::printf("ok %lld\n", n);
    return 0;
}
