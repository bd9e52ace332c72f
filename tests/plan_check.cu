// plan_check.cu -- host-only check of the launch plans that the RoPE and
// quantised tensor-core kernels index memory with (test infrastructure; built
// and run by tests/test_plans_cpu.py, linked against the library's objects).
//
// For many call shapes it takes la::plan_rope_sk and la::plan_rope_table as
// the library computes them and checks, by walking every CTA's range the way
// the kernels do:
//   - the reduce's stream-K plan covers every 16-token granule of every
//     (b, block, head group) exactly once, every segment holds at least one
//     token of its block, and every split-sum slot a CTA writes is below skP;
//     the slots of a unit are exactly 0 .. P-1 with P the count the combine
//     kernel derives (so it reads each slot once and nothing unwritten);
//   - the apply's plan covers every 128-token tile of every (b, block, head
//     pair) exactly once;
//   - the workspace that la_workspace_size reports holds skP slots;
//   - every cos/sin record a transform thread can read lies inside the table;
//   - magic_div's (m, s) divide exactly over the whole int range used.
// Prints "ok <cases>" or the first failure, and exits 0 only if all passed.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <tuple>
#include <vector>

#include "../block_causal_linear_b200/csrc/la_internal.cuh"
#include "../include/la.h"

namespace {

int g_fail = 0;
int g_tables = 0;   // tables that fit the kernels' layout and were checked

#define CHECK(cond, ...)                                              \
    do {                                                              \
        if (!(cond)) {                                                \
            if (!g_fail) {                                            \
                std::printf("FAIL %s:%d: %s: ", __FILE__, __LINE__, #cond); \
                std::printf(__VA_ARGS__);                             \
                std::printf("\n");                                    \
            }                                                         \
            g_fail = 1;                                               \
            return;                                                   \
        }                                                             \
    } while (0)

// The units of a plan in (b, block, unit) order with their first granule,
// enumerated directly (not through sk_locate / sk_unit_first).
struct UnitRef {
    int b, n, u;
    long long first, len;
};

std::vector<UnitRef> enumerate_units(const la::Sk &s, int B) {
    std::vector<UnitRef> out;
    long long x = 0;
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < s.nb; ++n)
            for (int u = 0; u < s.units; ++u) {
                const long long len = n < s.nb - 1 ? s.g_full : s.g_last;
                out.push_back({b, n, u, x, len});
                x += len;
            }
    return out;
}

// One stream-K plan: coverage, segment walk, slots.  `gran` tokens per granule.
void check_sk(const la::Sk &s, const la::Plan &p, int gran, int units, bool slots, const char *what) {
    const int Llast = p.N - (p.nb - 1) * p.L;
    CHECK(s.C >= 1 && s.C <= la::kSmCount, "%s: C = %d", what, s.C);
    CHECK(s.units == units && s.nb == p.nb, "%s: units %d nb %d", what, s.units, s.nb);
    CHECK(s.g_full == (p.L + gran - 1) / gran && s.g_last == (Llast + gran - 1) / gran, "%s: granules", what);
    const std::vector<UnitRef> us = enumerate_units(s, p.B);
    const long long total = us.back().first + us.back().len;
    CHECK(s.total == total, "%s: total %lld vs %lld", what, s.total, total);
    CHECK(la::sk_cta_start(s, 0) == 0 && la::sk_cta_start(s, s.C) == total, "%s: ends", what);
    for (int c = 0; c < s.C; ++c) {
        const long long a = la::sk_cta_start(s, c), e = la::sk_cta_start(s, c + 1);
        CHECK(a < e, "%s: CTA %d has an empty range", what, c);
        CHECK(la::sk_cta_of(s, a) == c && la::sk_cta_of(s, e - 1) == c, "%s: cta_of at CTA %d", what, c);
    }
    // sk_locate and sk_unit_first against the enumeration, at every unit's ends
    for (const UnitRef &r : us) {
        for (long long x : {r.first, r.first + r.len - 1}) {
            int b, n, u;
            la::sk_locate(s, x, b, n, u);
            CHECK(b == r.b && n == r.n && u == r.u, "%s: sk_locate(%lld)", what, x);
        }
        CHECK(la::sk_unit_first(s, r.b, r.n, r.u) == r.first, "%s: sk_unit_first", what);
        CHECK(la::sk_len(s, r.n) == r.len, "%s: sk_len", what);
    }
    // every CTA's walk, as the kernels take it: segments [x, min(unit end, range end))
    std::map<std::tuple<int, int, int>, std::vector<int>> written;   // unit -> slot counts
    std::vector<int> covered(total > (1 << 22) ? 0 : total, 0);
    for (int c = 0; c < s.C; ++c) {
        const long long xb = la::sk_cta_start(s, c), xe = la::sk_cta_start(s, c + 1);
        int b, n, u;
        la::sk_locate(s, xb, b, n, u);
        long long first = la::sk_unit_first(s, b, n, u), end = first + la::sk_len(s, n);
        for (long long x = xb; x < xe; x = end) {
            while (x >= end) {   // the next unit in order
                if (++u == s.units) {
                    u = 0;
                    if (++n == s.nb) {
                        n = 0;
                        ++b;
                    }
                }
                first = end;
                end = first + la::sk_len(s, n);
            }
            const long long e = end < xe ? end : xe;
            const int Ln = n < p.nb - 1 ? p.L : Llast;
            const long long tok0 = (x - first) * gran, tok1 = (e - first) * gran < Ln ? (e - first) * gran : Ln;
            CHECK(b < p.B && tok0 >= 0 && tok0 < tok1 && tok1 <= Ln, "%s: CTA %d segment [%lld, %lld) of %d", what,
                  c, tok0, tok1, Ln);
            if (!covered.empty())
                for (long long y = x; y < e; ++y) ++covered[y];
            if (slots) {
                const int slot = c - la::sk_cta_of(s, first);
                CHECK(slot >= 0 && slot < p.skP, "%s: CTA %d slot %d of %d", what, c, slot, p.skP);
                std::vector<int> &w = written[std::make_tuple(b, n, u)];
                if ((int)w.size() <= slot) w.resize(slot + 1, 0);
                ++w[slot];
            }
        }
    }
    for (size_t y = 0; y < covered.size(); ++y) CHECK(covered[y] == 1, "%s: granule %zu taken %d times", what, y, covered[y]);
    if (!slots) return;
    for (const UnitRef &r : us) {
        // the combine's slot count for this unit
        const int P = la::sk_cta_of(s, r.first + r.len - 1) - la::sk_cta_of(s, r.first) + 1;
        CHECK(P >= 1 && P <= p.skP, "%s: unit P = %d of %d", what, P, p.skP);
        const std::vector<int> &w = written[std::make_tuple(r.b, r.n, r.u)];
        CHECK((int)w.size() == P, "%s: unit (%d, %d, %d) wrote %zu slots, combine reads %d", what, r.b, r.n, r.u,
              w.size(), P);
        for (int j = 0; j < P; ++j) CHECK(w[j] == 1, "%s: slot %d written %d times", what, j, w[j]);
    }
}

void check_table(const la::Plan &p) {
    if (p.tab_bytes <= 0) return;
    ++g_tables;
    CHECK(p.tab_bytes <= 8192, "table %d bytes", p.tab_bytes);
    const long long len[3] = {p.tab_frames, p.Hg, p.Wg};
    // the positions a call's tokens take: frames 0 .. (N - 1) / (Hg Wg), rows, columns
    CHECK((long long)p.tab_frames * p.Hg * p.Wg >= p.N, "table covers %d frames", p.tab_frames);
    for (int m = 0; m < 8; ++m) {
        const int ax = p.hc_axis[m];
        CHECK(ax >= 0 && ax <= 2 && p.hc_base[m] >= 0 && p.hc_base[m] % 16 == 0 && p.hc_stride[m] % 16 == 0,
              "group %d record layout", m);
        CHECK(p.hc_base[m] + (len[ax] - 1) * p.hc_stride[m] + 16 <= p.tab_bytes, "group %d reads past the table", m);
    }
}

void check_magic() {
    const unsigned ds[] = {1, 2, 3, 5, 7, 26, 52, 80, 390, 1560, 3600, 46656, 65535, 65536, 1000003, 0x7fffffffu};
    for (unsigned d : ds) {
        unsigned long long m;
        int s;
        la::magic_div(d, m, s);
        auto q = [&](long long n) { return (long long)(((unsigned long long)n * m) >> s); };
        for (long long n = 0; n < 4096; ++n) CHECK(q(n) == n / d, "magic_div(%u) at %lld", d, n);
        for (long long k = 1; k <= 8192; ++k) {   // around multiples of d, up to 2^31 - 1
            const long long base = (long long)(((unsigned long long)k * 0x7fffffffull) / 8192 / d) * d;
            for (long long n = base - 1; n <= base + 1; ++n)
                if (n >= 0 && n <= 0x7fffffffLL) CHECK(q(n) == n / d, "magic_div(%u) at %lld", d, n);
        }
        CHECK(q(0x7fffffffLL) == 0x7fffffffLL / d, "magic_div(%u) at 2^31 - 1", d);
    }
}

}  // namespace

int main() {
    int cases = 0;
    check_magic();
    const int Bs[] = {1, 2, 4, 7};
    const int Hs[] = {4, 8, 12, 64, 128};
    const int Ns[] = {1, 15, 16, 17, 48, 100, 128, 129, 300, 1000, 2730, 8190, 10800, 15600};
    const int Ls[] = {0, 16, 48, 100, 128, 250, 1000, 2730};
    for (int B : Bs)
        for (int H : Hs)
            for (int N : Ns)
                for (int L0 : Ls) {
                    if (g_fail) break;
                    if (L0 > N) continue;
                    la::Plan p{};
                    p.B = B;
                    p.N = N;
                    p.H = H;
                    p.L = L0 > 0 && L0 < N ? L0 : N;
                    p.nb = (N + p.L - 1) / p.L;
                    la::plan_rope_sk(p);
                    check_sk(p.skr, p, 16, H / 4, true, "reduce");
                    check_sk(p.ska, p, 128, H / 2, false, "apply");
                    // the workspace sized by the C ABI holds the reduce's skP slots
                    const size_t ws = la_workspace_size(B, N, H, la::kD, L0);
                    if (!g_fail && ws < la::ws_layout(B, H, p.nb, p.skP).total) {
                        std::printf("FAIL workspace %zu < %zu for B %d N %d H %d L %d\n", ws,
                                    la::ws_layout(B, H, p.nb, p.skP).total, B, N, H, L0);
                        g_fail = 1;
                    }
                    // cos/sin tables for a few grids whose frames hold whole rows
                    const int grids[][2] = {{3, 10}, {15, 26}, {45, 80}, {30, 52}, {1, 1}, {2, 8}};
                    for (const auto &g : grids) {
                        la::Plan r = p;
                        r.rope = 1;
                        r.Hg = g[0];
                        r.Wg = g[1];
                        // feature pairs of 3D RoPE 8/12/12: 4 frame, 6 row, 6 column pairs
                        for (int i = 0; i < la::kD / 2; ++i) r.axis[i] = i < 4 ? 0 : (i < 10 ? 1 : 2);
                        la::plan_rope_table(r);
                        check_table(r);
                    }
                    if (g_fail) std::printf("  at B %d N %d H %d L %d\n", B, N, H, L0);
                    ++cases;
                }
    if (g_fail) return 1;
    std::printf("ok %d cases, %d tables\n", cases, g_tables);
    return 0;
}
