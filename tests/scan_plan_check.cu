// Host-only check of the tensor-core scan's launch plan (segments, state
// parts, workspace).  Compiled and run by tests/test_scan_plan_cpu.py; no
// kernel is launched (without a device the SM count falls back to 148).
#include "../selective_ssm_sequence_b200/csrc/scan_tc.cu"

#include <cstdio>

namespace hm {
void count_launches(unsigned) {}
}  // namespace hm

using namespace hm;

static int fails = 0;
#define CHECK(c, ...)                                      \
    do {                                                   \
        if (!(c)) {                                        \
            if (++fails <= 20) {                           \
                printf("FAIL %s: ", #c);                   \
                printf(__VA_ARGS__);                       \
                printf("\n");                              \
            }                                              \
        }                                                  \
    } while (0)

int main() {
    int n = 0;
    for (int B : {1, 2, 3, 4, 8, 16, 64})
        for (int H : {1, 2, 4, 8, 16})
            for (int64_t L : {1, 63, 64, 65, 500, 512, 1000, 2047, 2048, 4096, 8192, 32768, 100000})
                for (int ws : {0, 1}) {
                    ScanCore c{};
                    c.B = B;
                    c.L = L;
                    c.H = H;
                    c.F = 256;
                    c.dv = 256;
                    const Plan p = make_plan(c, ws != 0);
                    const Geo &g = p.g;
                    ++n;
                    const int64_t BH = (int64_t)B * H;
                    // segments: G of seg_chunks cover the chunks, none empty
                    CHECK(g.nchunks == (int)((L + 63) / 64), "B%d H%d L%ld nchunks %d", B, H, (long)L, g.nchunks);
                    CHECK(g.G >= 1 && (int64_t)g.G * g.seg_chunks >= g.nchunks &&
                              (int64_t)(g.G - 1) * g.seg_chunks < g.nchunks,
                          "B%d H%d L%ld G %d seg %d", B, H, (long)L, g.G, g.seg_chunks);
                    // one CTA per SM: the output kernel's grid fits the GPU
                    CHECK(2 * BH * g.G <= 148 || g.G == 1, "B%d H%d L%ld grid %ld", B, H, (long)L,
                          (long)(2 * BH * g.G));
                    // parts tile the segments
                    CHECK(g.part_chunks >= 1 && g.seg_chunks % g.part_chunks == 0, "B%d H%d L%ld part %d seg %d", B, H,
                          (long)L, g.part_chunks, g.seg_chunks);
                    CHECK((int64_t)g.NP * g.part_chunks >= g.nchunks &&
                              (int64_t)(g.NP - 1) * g.part_chunks < g.nchunks,
                          "B%d H%d L%ld NP %d", B, H, (long)L, g.NP);
                    const int pps = g.seg_chunks / g.part_chunks;
                    if (ws) {
                        CHECK(g.NPc == g.NP, "B%d H%d L%ld state wanted, NPc %d NP %d", B, H, (long)L, g.NPc, g.NP);
                    } else {
                        // the computed parts reach the start of the last segment, no further
                        CHECK((int64_t)g.NPc * g.part_chunks >= (int64_t)(g.G - 1) * g.seg_chunks &&
                                  g.NPc <= (g.G - 1) * pps,
                              "B%d H%d L%ld NPc %d G %d pps %d", B, H, (long)L, g.NPc, g.G, pps);
                    }
                    // the carry stores each later segment's start once: part p = g * pps
                    for (int s = 1; s < g.G; ++s) {
                        const int p0 = s * pps;
                        CHECK(p0 <= g.NPc && p0 % pps == 0 && p0 / pps == s, "B%d H%d L%ld seg %d part %d NPc %d", B, H,
                              (long)L, s, p0, g.NPc);
                    }
                    // workspace regions: ordered, 256-byte aligned, inside the total
                    const size_t nS = (size_t)256 * 256;
                    const size_t offs[5] = {p.off_Spart, p.off_zpart, p.off_lsum, p.off_Sstart, p.off_zstart};
                    const size_t np = (size_t)(BH * g.NPc), ng = (size_t)(BH * g.G);
                    const size_t lens[5] = {4 * np * nS, 4 * np * 256, 4 * np, 4 * ng * nS, 4 * ng * 256};
                    for (int r = 0; r < 5; ++r) {
                        CHECK(offs[r] % 256 == 0, "region %d offset %zu", r, offs[r]);
                        CHECK(offs[r] + lens[r] <= p.total, "region %d past the end", r);
                        if (r > 0) CHECK(offs[r - 1] + lens[r - 1] <= offs[r], "regions %d and %d overlap", r - 1, r);
                    }
                    CHECK(scan_tc_workspace(c) >= p.total, "workspace query %zu < plan %zu", scan_tc_workspace(c),
                          p.total);
                }
    printf("%d plans, %d failures\n", n, fails);
    return fails != 0;
}
