// split_check.cu -- host-side check of the attention work split and of the
// merge's record enumeration, compiled from the kernels' own headers and run
// on the CPU (no CUDA call is made).
//
// The kept lists of all units are concatenated into W blocks; CTA c of C
// takes [c*W/C, (c+1)*W/C).  Checked by brute force over seeded cases:
//   * cta_of(x) is the CTA whose range holds x, for every x;
//   * for every unit, the CTAs c_lo..c_hi that merge_record walks cover the
//     unit's [pre, pre + cnt) exactly once, and a record is reported written
//     exactly when its CTA's range meets the unit (one record per slot) or,
//     with four records per slot, when the warp's pair (w / 2) owns one of
//     the unit's tiles in that CTA (pair p owns CTA-local tile indices of
//     parity p);
//   * slot c + unit is never shared by two (CTA, unit) pairs that both hold
//     tiles, and stays below C + units (the partial buffers' size).
// Prints "ok <cases>" and exits 0, or prints the first failure and exits 1.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "merge.cuh"

using spattn::cta_of;
using spattn::merge_record;
using spattn::MergeArgs;

static uint64_t g_rng = 0x9e3779b97f4a7c15ull;
static uint32_t rnd(uint32_t n) {   // splitmix64, reduced to [0, n)
    uint64_t z = (g_rng += 0x9e3779b97f4a7c15ull);
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    z ^= z >> 31;
    return n ? (uint32_t)(z % n) : 0;
}

#define CHECK(cond, ...)                                    \
    do {                                                    \
        if (!(cond)) {                                      \
            std::printf("FAIL %s: ", #cond);                \
            std::printf(__VA_ARGS__);                       \
            std::printf("\n");                              \
            std::exit(1);                                   \
        }                                                   \
    } while (0)

static void check_case(const std::vector<int> &counts, int C, int wslots) {
    const int units = (int)counts.size();
    int64_t W = 0;
    for (int c : counts) W += c;
    MergeArgs a{};
    a.ctas = C;
    a.wslots = wslots;
    a.pairs = wslots == 4;
    a.units = units;
    // cta_of against the ranges themselves
    for (int64_t x = 0; x < W; ++x) {
        const int c = cta_of(x, W, C);
        CHECK(c >= 0 && c < C && W * c / C <= x && x < W * (c + 1) / C, "x=%lld W=%lld C=%d c=%d", (long long)x,
              (long long)W, C, c);
    }
    std::vector<int> slot_owner((size_t)(C + units) * wslots, -1);
    int64_t pre = 0;
    for (int u = 0; u < units; ++u) {
        const int cnt = counts[u];
        if (cnt > 0) {
            const int c_lo = cta_of(pre, W, C), c_hi = cta_of(pre + cnt - 1, W, C);
            std::vector<int> covered(cnt, 0);
            for (int x = 0; x < (c_hi - c_lo + 1) * wslots; ++x) {
                const int cc = c_lo + x / wslots, w = x % wslots;
                const int64_t lo = W * cc / C, hi = W * (cc + 1) / C;
                // brute force: the unit's tiles in this CTA, and this warp's share
                int mine = 0, any = 0;
                for (int64_t y = pre; y < pre + cnt; ++y) {
                    if (y < lo || y >= hi) continue;
                    ++any;
                    if (!a.pairs || ((y - lo) & 1) == (w >> 1)) ++mine;
                    if (w == 0) ++covered[y - pre];
                }
                const int64_t r = merge_record(a, x, c_lo, u, pre, cnt, W);
                CHECK((r >= 0) == (mine > 0), "unit %d cta %d warp %d: record %lld, tiles %d (of %d)", u, cc, w,
                      (long long)r, mine, any);
                if (r >= 0) {
                    CHECK(r == ((int64_t)cc + u) * wslots + w, "record index %lld", (long long)r);
                    CHECK(r < (int64_t)(C + units) * wslots, "record %lld beyond the buffer", (long long)r);
                    CHECK(slot_owner[r] < 0, "record %lld written by units %d and %d", (long long)r, slot_owner[r],
                          u);
                    slot_owner[r] = u;
                }
            }
            for (int y = 0; y < cnt; ++y) CHECK(covered[y] == 1, "unit %d tile %d covered %d times", u, y, covered[y]);
        }
        pre += cnt;
    }
}

int main() {
    int cases = 0;
    // fixed edge cases: one unit, empty units, fewer tiles than CTAs
    const int Cs[] = {1, 2, 3, 7, 148, 160, 296, 320};
    for (int C : Cs)
        for (int ws : {1, 4}) {
            check_case({1}, C, ws);
            check_case({0, 5, 0}, C, ws);
            check_case({3, 0, 0, 1, 2}, C, ws);
            check_case({1641, 1641}, C, ws);
            cases += 4;
        }
    // seeded random mixes of unit counts (decode-sized and skewed)
    for (int it = 0; it < 1500; ++it) {
        const int units = 1 + (int)rnd(96);
        std::vector<int> counts(units);
        const int mode = (int)rnd(4);
        for (int &c : counts) {
            if (mode == 0) c = (int)rnd(4);                    // tiny, many empty
            else if (mode == 1) c = 3 + (int)rnd(310);         // decode-sized
            else if (mode == 2) c = rnd(8) == 0 ? 900 + (int)rnd(800) : (int)rnd(20);   // skewed
            else c = (int)rnd(2000);
        }
        const int C = 1 + (int)rnd(320);
        check_case(counts, C, rnd(2) ? 4 : 1);
        ++cases;
    }
    std::printf("ok %d\n", cases);
    return 0;
}
