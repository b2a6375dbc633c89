// Host-only check of the projection kernels' work splits, run on the CPU
// (no CUDA call is made).  It walks the same planning and walking functions
// the kernels use (work_split.cuh for the persistent prefill projection,
// run_begin / owner / next_seg for the decode projection's stream-K runs) for
// many shapes and checks, for every shape:
//   * every (tile, k-tile) unit is processed exactly once;
//   * tile coordinates are a bijection onto the M x N tile grid;
//   * a split tile's contributors are exactly the CTAs owner() names, each
//     writes one partial slot (0: its run's first segment, 1: its last), no
//     CTA writes a slot twice, and the reader's slot rule finds each partial;
//   * grid and run counts stay within their bounds.
// Prints "ok" and exits 0, or prints the first failure and exits 1.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <random>
#include <set>
#include <utility>
#include <vector>

#include "../../decoder_only_transformer_llama_b200/csrc/decode_tile.cuh"
#include "../../decoder_only_transformer_llama_b200/csrc/work_split.cuh"

using namespace llb;

#define CHECK(cond, ...)                                  \
    do {                                                  \
        if (!(cond)) {                                    \
            std::printf("FAIL %s:%d: ", __FILE__, __LINE__); \
            std::printf(__VA_ARGS__);                     \
            std::printf("\n");                            \
            std::exit(1);                                 \
        }                                                 \
    } while (0)

struct Piece {
    int cta, slot, ks, ke;
};

// Contributors of split tiles must match owner(); each writes its own slot.
static void check_split_tiles(const std::map<int, std::vector<Piece>>& pieces, int KT, int W, int P, int first_tile,
                              const char* what) {
    for (const auto& kv : pieces) {
        const int tl = kv.first - first_tile;   // index among the split-eligible tiles
        const int ub = tl * KT;
        const int cf = owner(ub, W, P), cl = owner(ub + KT - 1, W, P);
        std::set<int> ctas;
        int covered = 0;
        for (const Piece& p : kv.second) {
            ctas.insert(p.cta);
            covered += p.ke - p.ks;
            const int read_slot = run_begin(p.cta, W, P) >= ub ? 0 : 1;
            CHECK(read_slot == p.slot, "%s tile %d cta %d: written slot %d, read slot %d", what, kv.first, p.cta,
                  p.slot, read_slot);
        }
        CHECK(covered == KT, "%s tile %d: pieces cover %d of %d k-tiles", what, kv.first, covered, KT);
        CHECK(static_cast<int>(ctas.size()) == cl - cf + 1, "%s tile %d: %zu contributors, owner() says %d", what,
              kv.first, ctas.size(), cl - cf + 1);
        CHECK(*ctas.begin() == cf && *ctas.rbegin() == cl, "%s tile %d: contributors %d..%d, owner() %d..%d", what,
              kv.first, *ctas.begin(), *ctas.rbegin(), cf, cl);
    }
}

static void check_prefill(int TM, int TN, int KT, int P, bool can_split) {
    TcPlan p;
    p.TM = TM;
    p.TN = TN;
    p.KT = KT;
    const int T = TM * TN;
    int grid = 0;
    plan_tc(T, KT, P, can_split, &p, &grid);
    CHECK(grid >= 1 && grid <= P && grid <= T * KT, "prefill grid %d (T=%d KT=%d P=%d)", grid, T, KT, P);
    CHECK(p.dp + p.sk == T, "prefill dp %d + sk %d != T %d", p.dp, p.sk, T);
    CHECK(p.dp % grid == 0 || p.sk == 0, "prefill: %d whole tiles are not whole waves of %d", p.dp, grid);
    if (p.sk > 0) CHECK(p.psk >= 1 && p.psk <= grid && p.psk <= 4 * p.sk, "prefill psk %d", p.psk);
    std::vector<int> cover(static_cast<size_t>(T) * KT, 0);
    std::map<int, std::vector<Piece>> pieces;
    std::set<std::pair<int, int>> slots;
    const int Wsk = p.sk * KT;
    for (int c = 0; c < grid; ++c) {
        WorkIt w = work_begin(p, c, grid);
        Item it;
        const int u0 = c < p.psk ? run_begin(c, Wsk, p.psk) : 0;
        while (work_next(w, p, grid, it)) {
            CHECK(it.tile >= 0 && it.tile < T && 0 <= it.ks && it.ks < it.ke && it.ke <= KT, "prefill item %d [%d,%d)",
                  it.tile, it.ks, it.ke);
            for (int k = it.ks; k < it.ke; ++k) ++cover[static_cast<size_t>(it.tile) * KT + k];
            if (it.ks == 0 && it.ke == KT) continue;
            CHECK(it.tile >= p.dp, "prefill: split item in the whole-tile range (tile %d)", it.tile);
            const int ub = (it.tile - p.dp) * KT;
            const int slot = (ub + it.ks == u0) ? 0 : 1;
            CHECK(slots.insert({c, slot}).second, "prefill cta %d writes slot %d twice", c, slot);
            pieces[it.tile].push_back({c, slot, it.ks, it.ke});
        }
    }
    for (size_t i = 0; i < cover.size(); ++i)
        CHECK(cover[i] == 1, "prefill unit (tile %zu, k %zu) processed %d times (TM=%d TN=%d KT=%d P=%d)", i / KT,
              i % KT, cover[i], TM, TN, KT, P);
    if (p.sk > 0) check_split_tiles(pieces, KT, Wsk, p.psk, p.dp, "prefill");
    std::set<std::pair<int, int>> coords;
    for (int t = 0; t < T; ++t) {
        int tm, tn;
        tile_coords(t, p, tm, tn);
        CHECK(tm >= 0 && tm < TM && tn >= 0 && tn < TN, "tile %d -> (%d, %d)", t, tm, tn);
        CHECK(coords.insert({tm, tn}).second, "tile coordinates (%d, %d) reached twice", tm, tn);
    }
}

// Decode projection: the split tile's finisher is split_finisher() (its first
// contributor); its segment must be the LAST of its run (so it is processed
// after the CTA's other work) and every other contributor's segment the FIRST
// of its run, so each CTA publishes at most one partial, and the finisher
// collects exactly the other contributors' partials.
static void check_decode(int T, int KT, int sms) {
    const int W = T * KT;
    const int P = W < sms ? W : sms;   // the decode launcher's grid
    std::vector<int> cover(static_cast<size_t>(W), 0);
    std::map<int, std::vector<int>> published;   // tile -> CTAs that published a partial of it
    std::map<int, int> finished;                 // tile -> finishing CTA
    std::vector<int> n_pub(static_cast<size_t>(P), 0);
    for (int c = 0; c < P; ++c) {
        const int u0 = run_begin(c, W, P), u1 = run_begin(c + 1, W, P);
        CHECK(u1 > u0, "decode cta %d has an empty run (W=%d P=%d)", c, W, P);
        int u = u0;
        Seg sg;
        while (next_seg(u, u1, KT, sg)) {
            for (int k = sg.ks; k < sg.ke; ++k) ++cover[static_cast<size_t>(sg.tile) * KT + k];
            const int tb = sg.tile * KT;
            const int cf = split_finisher(sg.tile, KT, W, P), cl = owner(tb + KT - 1, W, P);
            if (cl == cf) {
                CHECK(sg.ks == 0 && sg.ke == KT, "decode tile %d owned by one cta but cut", sg.tile);
                continue;
            }
            if (c == cf) {
                CHECK(tb + sg.ke == u1, "decode tile %d: finisher cta %d's segment is not its run's last", sg.tile, c);
                CHECK(sg.ks == 0, "decode tile %d: finisher cta %d does not hold the first unit", sg.tile, c);
                CHECK(finished.insert({sg.tile, c}).second, "decode tile %d finished twice", sg.tile);
            } else {
                CHECK(tb + sg.ks == u0, "decode tile %d: cta %d's published segment is not its run's first", sg.tile, c);
                published[sg.tile].push_back(c);
                CHECK(++n_pub[static_cast<size_t>(c)] == 1, "decode cta %d publishes two partials", c);
            }
        }
    }
    for (size_t i = 0; i < cover.size(); ++i)
        CHECK(cover[i] == 1, "decode unit %zu processed %d times (T=%d KT=%d)", i, cover[i], T, KT);
    for (const auto& kv : published) {
        const int t = kv.first, tb = t * KT;
        const int cf = owner(tb, W, P), cl = owner(tb + KT - 1, W, P);
        CHECK(finished.count(t) == 1 && finished[t] == cf, "decode tile %d has no finisher", t);
        CHECK(static_cast<int>(kv.second.size()) == cl - cf, "decode tile %d: %zu partials, the finisher waits for %d",
              t, kv.second.size(), cl - cf);
        for (size_t i = 0; i < kv.second.size(); ++i)
            CHECK(kv.second[i] == cf + 1 + static_cast<int>(i), "decode tile %d: partial of cta %d out of order", t,
                  kv.second[i]);
    }
    for (const auto& kv : finished)
        CHECK(published.count(kv.first) == 1, "decode tile %d finished with no partials to collect", kv.first);
}

int main() {
    // the shapes of the workloads (7B, 13B, 70B slice, small models) ...
    const int sms[] = {148, 132, 256, 7, 1};
    for (int s : sms) {
        for (int TM : {1, 2, 16, 58, 128})
            for (int TN : {1, 2, 16, 20, 40, 48, 86, 108, 224})
                for (int KT : {1, 4, 64, 80, 128, 172, 216, 448}) check_prefill(TM, TN, KT, s, true);
        for (int T : {1, 2, 32, 40, 96, 120, 172, 216, 250, 448})
            for (int KT : {1, 4, 64, 80, 128, 172, 216, 448}) check_decode(T, KT, s);
    }
    check_prefill(16, 48, 64, 148, false);
    // ... and random ones
    std::mt19937 rng(12345);
    for (int i = 0; i < 3000; ++i) {
        const int TM = 1 + static_cast<int>(rng() % 140), TN = 1 + static_cast<int>(rng() % 240);
        const int KT = 1 + static_cast<int>(rng() % 450), P = sms[rng() % 5];
        check_prefill(TM, TN, KT, P, (rng() & 7) != 0);
        check_decode(1 + static_cast<int>(rng() % 600), KT, P);
    }
    std::printf("ok\n");
    return 0;
}
