// stream_plan_check.cu -- host-only check of the batched-decode stream
// kernel's launch plans (no GPU is touched: the kernel is compiled with the
// translation unit but never launched).
//
// For every shape the route sends to the kernel, over a range of SM counts,
// the plan must satisfy the conditions the kernel relies on for memory
// safety: shared memory within the opt-in limit (and two CTAs per SM where
// the plan says so), the A operand's reads past the X box inside the
// allocation, the B operand's reads inside their stage, TMEM columns within
// the SM's share, TMA box dimensions within 256, the epilogue's staging
// chunk inside the idle ring, the MMA shapes tcgen05 accepts, and per-CTA
// unit counts of q or q + 1.  Prints "ok <plans checked>" or the first
// violation and exits non-zero.
#include "../up_projection_b200/csrc/stream_tc_bf16.cu"

#include <cstdio>

namespace {

int fail(const char *what, int M, int K, int N, int sms) {
    std::printf("violation: %s at M=%d K=%d N=%d sm_count=%d\n", what, M, K, N, sms);
    return 1;
}

int check(int M, int K, int N, int sms) {
    using namespace swiglu;
    const StreamPlan p = stream_plan(M, K, N, sms);
    const StreamGeo &g = p.geo;
    if (!g.ok) return fail("no plan for a routed shape", M, K, N, sms);
    const int units = N / 8;
    const int cps = g.ctas_per_sm;
    if (cps != 1 && cps != 2) return fail("CTAs per SM", M, K, N, sms);
    if (p.grid < 1 || p.grid > units) return fail("grid", M, K, N, sms);
    // balanced split: every CTA has q or q + 1 units, at most q1
    const int q = p.q, q1 = (units + p.grid - 1) / p.grid;
    if (q < 1 || q != units / p.grid || q1 > g.q1 || g.q1 > 16 / cps)
        return fail("units per CTA", M, K, N, sms);
    if (8 * (q + 1) > 256 || g.mpad > 256 || g.kb > 256) return fail("TMA box dimension", M, K, N, sms);
    // shared memory: the allocation, and two CTAs (1 KB reserved each) per SM
    if (g.smem > 227 * 1024) return fail("shared memory per CTA", M, K, N, sms);
    if (cps == 2 && 2 * (g.smem + 1024) > 228 * 1024) return fail("two CTAs per SM", M, K, N, sms);
    if (g.off_bar + kTail != g.smem) return fail("layout tail", M, K, N, sms);
    // stage layout: weights (2 wbytes) then the X box (mpad x kc bf16)
    if (g.stage != 2 * g.wbytes + g.mpad * g.kb * 128 || g.wbytes != g.q1 * g.kb * 1024)
        return fail("stage layout", M, K, N, sms);
    if (g.stage % 1024 != 0 || g.wbytes % 1024 != 0) return fail("1024-byte alignment", M, K, N, sms);
    // the mbarrier transaction count of one stage
    if (g.stage >= (1 << 20)) return fail("transaction bytes per stage", M, K, N, sms);
    // A operand: mma_m rows of 128 B from each k-block of the last stage's X box
    const long long a_end = static_cast<long long>(g.ring - 1) * g.stage + 2 * g.wbytes +
                            static_cast<long long>(g.kb - 1) * g.mpad * 128 + g.mma_m * 128;
    if (a_end > g.off_bar) return fail("A operand past the ring", M, K, N, sms);
    if (g.mma_m != (g.mpad <= 64 ? 64 : 128)) return fail("MMA M", M, K, N, sms);
    for (int cnt = q; cnt <= q + 1 && cnt <= g.q1; ++cnt) {
        // pair form: N = 16 cnt rows of block b inside the weight boxes
        const int n_pair = 16 * cnt;
        if (n_pair > 256 || n_pair % 16 != 0) return fail("MMA N (pair)", M, K, N, sms);
        const long long b_end_pair = static_cast<long long>(g.kb - 1) * cnt * 2048 + n_pair * 128;
        if (b_end_pair > 2LL * g.wbytes) return fail("B operand (pair)", M, K, N, sms);
        // split form: N = 8 cnt (rounded to 16 for M = 128) from each box
        const int n_split = g.mma_m == 128 ? (8 * cnt + 15) / 16 * 16 : 8 * cnt;
        if (n_split > 256 || (g.mma_m == 128 ? n_split % 16 : n_split % 8) != 0)
            return fail("MMA N (split)", M, K, N, sms);
        const long long b_end_split =
            g.wbytes + static_cast<long long>(g.kb - 1) * cnt * 1024 + n_split * 128;
        if (b_end_split > g.stage) return fail("B operand (split)", M, K, N, sms);
        // TMEM: two sets x (gate, up) regions
        if (2 * g.region < n_pair || g.region < n_split) return fail("TMEM region", M, K, N, sms);
    }
    if (g.tmem_cols < 4 * g.region || g.tmem_cols > 512 / cps ||
        (g.tmem_cols & (g.tmem_cols - 1)) != 0 || g.tmem_cols < 32)
        return fail("TMEM columns", M, K, N, sms);
    // epilogue staging: epi_units x M rows x 64 B inside the idle ring
    if (g.epi_units < 1 || g.epi_units > g.q1 ||
        static_cast<long long>(g.epi_units) * g.mpad * 64 > static_cast<long long>(g.ring) * g.stage)
        return fail("epilogue chunk", M, K, N, sms);
    if (g.slices != (g.kblocks + g.kb - 1) / g.kb || g.kblocks != K / 64)
        return fail("slices", M, K, N, sms);
    return 0;
}

}  // namespace

int main() {
    static const int kKs[] = {64, 128, 192, 256, 320, 512, 832, 1024, 1536, 2048,
                              4096, 5120, 6144, 8192, 14336, 65536};
    static const int kNs[] = {8, 16, 24, 64, 264, 520, 1032, 2368, 6912, 11008,
                              13824, 14336, 24576, 37888, 8 * 148 * 32 + 8, 8 * 148 * 16 * 3};
    static const int kSms[] = {148, 132, 80, 20, 1};
    long long n = 0;
    for (int M = 9; M <= 128; ++M)
        for (int K : kKs)
            for (int N : kNs)
                for (int sms : kSms) {
                    if (!swiglu::stream_tc_bf16_supported(M, K, N)) {
                        std::printf("violation: routed shape unsupported M=%d K=%d N=%d\n", M, K, N);
                        return 1;
                    }
                    if (check(M, K, N, sms)) return 1;
                    ++n;
                }
    // shapes the kernel must refuse
    if (swiglu::stream_tc_bf16_supported(8, 256, 512) ||
        swiglu::stream_tc_bf16_supported(129, 256, 512) ||
        swiglu::stream_tc_bf16_supported(16, 264, 512) ||
        swiglu::stream_tc_bf16_supported(16, 256, 12)) {
        std::printf("violation: an unsupported shape is accepted\n");
        return 1;
    }
    std::printf("ok %lld\n", n);
    return 0;
}
