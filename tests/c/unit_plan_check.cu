// Host check of the prefill work decomposition in prefill_plan.cuh, the same
// functions the kernel's warps call (compiled here for the CPU; no GPU).
//
// For each case the launch parameters come from prefill_units() as the host
// API fills them, and every unit of the launch is planned.  Checked:
//  * the persistent blocks (min(units, SMs) of them, alternating direction
//    every round) take every unit exactly once;
//  * every (sequence, query head, query row) is computed by exactly one head
//    slot of one unit, and that head belongs to the unit's KV head
//    (contiguous groups: head h uses KV head h / G);
//  * a unit visits no key tile twice;
//  * for every row, the keys its unit's tiles contribute are exactly the
//    row's key set, each position once: the window i-W < j <= i (positions
//    from 0), plus the sink positions j < S outside the window.  What a key
//    storage contributes to row i follows from what it holds: a row of the
//    main k/v (position s0 + r) when it is in the window (or, in one-shot
//    prefill, a sink); a rolling-buffer slot s, which holds position
//    s0 - age(s) with age(s) = (s0 - s) mod W in 1..W (empty below 0), when
//    that position is in the window; a sink-buffer slot j (position j) when
//    j is outside the window;
//  * a tile the planner marks clean (the softmax applies no mask to it)
//    contributes all its keys to every row of its unit, and all of them
//    exist.
// Sources: the SWA mask of "핵심 구성요소" of the "Mistral 7B -- Sliding
// Window Attention" summary, "Pre-fill + Chunking" of the same summary (a
// chunk attends to the buffer and to itself), the rolling buffer's write
// rule slot = p mod W ("Rolling Buffer KV Cache 동작 설명"), and the attention
// sinks of the aionda.blog page (the first few positions kept).
//
// Also 160 seeded random launches (shapes, windows, sinks, packed offsets,
// buffer positions and SM counts drawn).  Prints "ok <cases> <rows>" and
// exits 0, or the first mismatch and exits 1.
#include <cstdio>
#include <cstdlib>
#include <set>
#include <utility>
#include <vector>

#include "../../sliding_window_gqa_prefill_b200/csrc/prefill_plan.cuh"

namespace {

struct Case {
    const char *name;
    int B;                  // sequences
    int N;                  // rows per sequence (chunk length in chunk mode; total packed rows if varlen)
    int Hq, Hkv, W;
    bool chunk;
    int S;                  // sinks: one-shot S, or the chunk mode's sink buffer slots
    std::vector<int> start; // chunk mode: first position of each sequence
    std::vector<int> cu;    // packed batch: B + 1 row offsets (empty: fixed length)
    bool skip_len1;
    int sms;
};

long long g_rows = 0;

bool fail(const Case &c, const char *what, long long a = 0, long long b = 0, long long d = 0) {
    std::printf("FAIL %s: %s (%lld, %lld, %lld)\n", c.name, what, a, b, d);
    return false;
}

bool check(const Case &c0) {
    // the host clamps a one-shot window to the rows (it never reaches before
    // position 0); the key sets are the same either way
    Case c = c0;
    if (!c.chunk && c.W > c.N) c.W = c.N;
    swa::PrefillParams p{};
    const bool varlen = !c.cu.empty();
    swa::prefill_units(p, c.B, c.N, c.Hq, c.Hkv, c.W, varlen, c.chunk, c.sms);
    p.start_pos = c.chunk ? c.start.data() : nullptr;
    p.cu_seqlens = varlen ? c.cu.data() : nullptr;
    p.skip_len1 = c.skip_len1 ? 1 : 0;
    p.sinks = c.chunk ? 0 : c.S;
    p.sink_buf = c.chunk ? c.S : 0;
    const int G = c.Hq / c.Hkv;

    std::vector<int> pre(c.B + 1, 0);
    int units = p.num_units;
    if (varlen) {
        if (swa::varlen_prefix(p, pre.data())) return fail(c, "malformed offsets reported");
        units = pre[c.B] * p.Hkv * p.npairs;
        if (units > p.num_units) return fail(c, "packed units above the host's bound", units, p.num_units);
    }

    // the persistent schedule: over the alternating rounds, the grid's blocks
    // take every unit exactly once
    {
        const int C = units < c.sms ? units : c.sms;
        std::vector<int> taken(units, 0);
        for (int cta = 0; cta < C; ++cta)
            for (int k = 0, u; (u = swa::unit_of(k, cta, C)) < units; ++k) ++taken[u];
        for (int u = 0; u < units; ++u)
            if (taken[u] != 1) return fail(c, "unit not taken exactly once", u, taken[u], C);
    }

    // rows per sequence
    std::vector<int> nq(c.B);
    for (int b = 0; b < c.B; ++b) nq[b] = varlen ? c.cu[b + 1] - c.cu[b] : c.N;
    // cover[(b, h, row)] = number of head slots computing it
    std::vector<std::vector<int>> cover(c.B);
    for (int b = 0; b < c.B; ++b) cover[b].assign((size_t)c.Hq * nq[b], 0);

    std::vector<int> cnt;
    for (int u = 0; u < units; ++u) {
        const swa::UnitPlan P = swa::plan_unit(p, u, pre.data());
        const int b = P.b;
        if (b < 0 || b >= c.B || P.nq != nq[b]) return fail(c, "unit sequence", u, b, P.nq);
        const int s0 = c.chunk ? c.start[b] : 0;
        // tiles: distinct, and their storage
        std::set<std::pair<int, int>> seen;
        std::vector<swa::TileRef> tiles(P.n);
        for (int j = 0; j < P.n; ++j) {
            tiles[j] = swa::tile_ref(p, P, j);
            const int kind = (!c.chunk && j < P.sink_tile) ? 0 : tiles[j].cache;
            if (!seen.insert({kind, tiles[j].row0}).second) return fail(c, "tile visited twice", u, j, tiles[j].row0);
        }
        for (int t = 0; t < 1 + P.act1; ++t) {
            const int h = p.qpair ? P.h0 : P.h0 + t;
            if (h < 0 || h >= c.Hq || h / G != P.g) return fail(c, "head of the unit's KV head", u, h, P.g);
            const int first = P.q0 + (p.qpair ? t * 128 : 0);
            if (first >= P.nq) return fail(c, "head slot with no rows", u, t, first);
            for (int i = first; i < first + 128 && i < P.nq; ++i) {
                ++cover[b][(size_t)h * nq[b] + i];
                const int a = s0 + i;                  // absolute position of the query
                cnt.assign((size_t)a + 1, 0);
                for (int j = 0; j < P.n; ++j) {
                    const swa::TileRef &T = tiles[j];
                    for (int cc = 0; cc < 128; ++cc) {
                        long long pos = -1;            // position this key holds, -1: none
                        bool in = false;
                        if (T.cache == 2) {            // sink buffer slot
                            const int slot = T.row0 + cc;
                            if (slot < c.S) {
                                pos = slot;
                                in = pos <= (long long)a - c.W;
                            }
                        } else if (T.cache == 1) {     // rolling-buffer slot
                            const int slot = T.row0 + cc;
                            if (slot < c.W) {
                                const int qs = s0 % c.W;
                                const int m = ((qs - slot) % c.W + c.W) % c.W;   // age mod W
                                const int age = m == 0 ? c.W : m;
                                pos = (long long)s0 - age;
                                if (pos < 0) pos = -1;
                                in = pos >= 0 && pos > (long long)a - c.W;
                            }
                        } else {                       // row of the main k/v
                            const int r = T.row0 + cc;
                            if (r < P.nq) {
                                pos = (long long)s0 + r;
                                in = pos <= a && (pos > (long long)a - c.W || (!c.chunk && pos < c.S));
                            }
                        }
                        if (!T.masked && (pos < 0 || !in))
                            return fail(c, "clean tile holds a key the row must not see", u, i, j);
                        if (in) {
                            if (pos < 0 || pos > a) return fail(c, "key past the query", u, i, pos);
                            if (++cnt[(size_t)pos] > 1) return fail(c, "key counted twice", u, i, pos);
                        }
                    }
                }
                // the row's key set: window plus sinks outside it
                for (long long pos = 0; pos <= a; ++pos) {
                    const bool want = pos > (long long)a - c.W || pos < c.S;
                    if (want != (cnt[(size_t)pos] == 1)) return fail(c, "key set of the row", u, i, pos);
                }
                ++g_rows;
            }
        }
    }
    for (int b = 0; b < c.B; ++b)
        for (size_t k = 0; k < cover[b].size(); ++k)
            if (cover[b][k] != (varlen && c.skip_len1 && nq[b] == 1 ? 0 : 1))
                return fail(c, "row computed other than once", b, (long long)(k / nq[b]), (long long)(k % nq[b]));
    return true;
}

}  // namespace

int main() {
    const int sms = 148;
    std::vector<Case> cases = {
        // one-shot, head pairs
        {"one-shot 8/2 ragged", 2, 1000, 8, 2, 300, false, 0, {}, {}, false, sms},
        {"one-shot 32/8 W>N", 1, 700, 32, 8, 4096, false, 0, {}, {}, false, sms},
        {"one-shot odd group 6/2 below two waves", 1, 900, 6, 2, 256, false, 0, {}, {}, false, sms},
        {"one-shot G=3 head pairs, 288 units", 1, 2304, 24, 8, 600, false, 0, {}, {}, false, sms},
        {"one-shot half-wave split 32/8", 1, 256, 32, 8, 64, false, 0, {}, {}, false, sms},
        // odd groups in one wave: one head per unit
        {"one-shot single heads G=7", 1, 512, 28, 4, 256, false, 0, {}, {}, false, sms},
        {"one-shot single heads G=3 sinks", 2, 300, 6, 2, 100, false, 4, {}, {}, false, sms},
        {"one-shot G=3 past one wave of single heads", 1, 1024, 24, 8, 383, false, 0, {}, {}, false, sms},
        {"one-shot W=1", 1, 300, 4, 2, 1, false, 0, {}, {}, false, sms},
        // windows of 128k-1 keys: a tile's first key lands on the last row's window edge
        {"one-shot W=255", 2, 1000, 8, 2, 255, false, 0, {}, {}, false, sms},
        {"one-shot W=383 sinks", 1, 1200, 6, 2, 383, false, 4, {}, {}, false, sms},
        {"qpair MHA W=383", 1, 1900, 32, 32, 383, false, 0, {}, {}, false, sms},
        {"chunk W=511", 2, 400, 8, 2, 511, true, 0, {511, 2000}, {}, false, sms},
        {"one-shot sinks S=4", 1, 900, 8, 2, 256, false, 4, {}, {}, false, sms},
        {"one-shot sinks S=130", 1, 1000, 6, 2, 300, false, 130, {}, {}, false, sms},
        // query-block pairs (odd groups, at least two waves)
        {"qpair MHA ragged pair", 1, 1900, 32, 32, 500, false, 0, {}, {}, false, sms},
        {"qpair MHA W>N", 1, 2048, 32, 32, 3000, false, 0, {}, {}, false, sms},
        {"qpair G=3", 1, 2560, 24, 8, 600, false, 0, {}, {}, false, sms},
        {"qpair G=5 ragged", 1, 1700, 40, 8, 450, false, 0, {}, {}, false, sms},
        {"qpair G=7 one-block last pair", 1, 1300, 56, 8, 700, false, 0, {}, {}, false, sms},
        {"qpair MHA sinks", 1, 1900, 32, 32, 500, false, 4, {}, {}, false, sms},
        // chunk mode
        {"chunk C<W fresh and deep", 2, 200, 8, 2, 256, true, 0, {0, 500}, {}, false, sms},
        {"chunk C=W", 1, 512, 8, 2, 512, true, 0, {1536}, {}, false, sms},
        {"chunk partial buffer", 3, 300, 4, 2, 1000, true, 0, {0, 300, 850}, {}, false, sms},
        {"chunk unaligned start", 2, 333, 8, 2, 700, true, 0, {77, 5000}, {}, false, sms},
        {"chunk sinks", 1, 256, 8, 2, 256, true, 4, {3000}, {}, false, sms},
        {"chunk sinks two tiles", 1, 300, 6, 2, 384, true, 130, {600}, {}, false, sms},
        {"chunk 4096 last-wave split", 1, 4096, 32, 8, 4096, true, 0, {12288}, {}, false, sms},
        {"chunk qpair G=3", 2, 1280, 24, 8, 1280, true, 0, {1280, 2560}, {}, false, sms},
        {"chunk qpair MHA sinks", 1, 1280, 32, 32, 1280, true, 130, {1280}, {}, false, sms},
        // pairs of query blocks split into their blocks in a short last wave
        {"chunk qpair MHA 4096 last-wave split", 1, 4096, 32, 32, 4096, true, 0, {12288}, {}, false, sms},
        {"chunk qpair ragged, split away from the one-block pairs", 1, 1000, 40, 40, 1000, true, 4, {2000}, {}, false,
         sms},
        {"chunk qpair one-block pairs in the last wave: no split", 1, 200, 300, 300, 256, true, 0, {1000}, {}, false,
         sms},
        // packed batches
        {"varlen one-shot", 6, 1000, 32, 8, 256, false, 0, {}, {0, 1, 129, 130, 700, 700, 1000}, false, sms},
        {"varlen chunk", 5, 900, 8, 2, 512, true, 0, {0, 3000, 7, 512, 100}, {0, 300, 301, 600, 600, 900}, false, sms},
        {"varlen chunk, one-row sequences to decode", 5, 900, 8, 2, 512, true, 0, {0, 3000, 7, 512, 100},
         {0, 300, 301, 600, 601, 900}, true, sms},
        // packed batches in pairs of query blocks (odd groups, two waves by the host's bound)
        {"varlen qpair MHA", 4, 2500, 32, 32, 500, false, 0, {}, {0, 700, 1300, 1301, 2500}, false, sms},
        {"varlen qpair G=3 W=383", 3, 2300, 24, 8, 383, false, 0, {}, {0, 1000, 1001, 2300}, false, sms},
        {"varlen chunk qpair G=3", 3, 2300, 24, 8, 1024, true, 0, {0, 5000, 100}, {0, 1000, 1001, 2300}, false, sms},
        {"varlen chunk qpair G=3, one-row sequences to decode", 4, 2300, 24, 8, 1024, true, 0, {0, 5000, 100, 9},
         {0, 1000, 1001, 2299, 2300}, true, sms},
    };
    for (const Case &c : cases)
        if (!check(c)) return 1;

    // seeded random launches; small SM counts make the two-wave, last-wave
    // and one-wave policies trigger at small sizes
    unsigned long long state = 0x2545F4914F6CDD1DULL;
    auto draw = [&](int lo, int hi) {               // uniform on [lo, hi]
        state ^= state << 13;
        state ^= state >> 7;
        state ^= state << 17;
        return lo + (int)(state % (unsigned long long)(hi - lo + 1));
    };
    const int sm_choices[] = {148, 33, 16, 8, 3};
    int random_cases = 0;
    for (int it = 0; it < 160; ++it) {
        Case c;
        c.name = "random";
        const int mode = draw(0, 3);                // one-shot, chunk, packed one-shot, packed chunk
        c.Hkv = draw(1, 2);
        c.Hq = c.Hkv * draw(1, 8);
        c.W = draw(1, 600);
        c.sms = sm_choices[draw(0, 4)];
        c.chunk = mode == 1 || mode == 3;
        c.skip_len1 = false;
        c.S = 0;
        if (mode == 0 || mode == 1) {
            c.B = draw(1, 2);
            c.N = c.chunk ? draw(1, c.W < 500 ? c.W : 500) : draw(1, 500);
            if (draw(0, 2) == 0) c.S = draw(1, 140);     // sinks (fixed-length calls only)
        } else {
            c.B = draw(1, 4);
            c.cu.push_back(0);
            for (int b = 0; b < c.B; ++b) {
                const int kind = draw(0, 4);
                c.cu.push_back(c.cu.back() + (kind == 0 ? 0 : kind == 1 ? 1 : draw(2, 300)));
            }
            c.N = c.cu.back();
            if (c.N == 0) continue;                 // an empty packed call is rejected by the host
            c.skip_len1 = c.chunk && draw(0, 1) == 1;
        }
        if (c.chunk)
            for (int b = 0; b < c.B; ++b) c.start.push_back(draw(0, 3) == 0 ? 0 : draw(0, 4000));
        if (!check(c)) {
            std::printf("  (random case %d: B=%d N=%d Hq=%d Hkv=%d W=%d chunk=%d S=%d sms=%d)\n", it, c.B, c.N, c.Hq,
                        c.Hkv, c.W, (int)c.chunk, c.S, c.sms);
            return 1;
        }
        ++random_cases;
    }
    std::printf("ok %zu %lld (and %d random)\n", cases.size(), g_rows, random_cases);
    return 0;
}
