// Work split of the persistent prefill projection (gemm_tc.cu): which tiles
// and k-ranges each CTA takes.  Host and device code: the launcher plans on
// the host, every warp role of the kernel walks the same list on the device,
// and a host-only checker (tests) walks it exhaustively.
#pragma once

#include <algorithm>

#include "common.cuh"

namespace llb {

constexpr int kGroupM = 16;   // M-tiles per rasterisation group

// Work list of one CTA: (c < psk) its stream-K run over the last sk tiles
// first, then whole tiles c, c+P, ... below dp.  Split tiles come first so
// that their fixups (partials published, the last arrival adding them up)
// overlap the MMAs of the CTA's whole tiles instead of ending the launch.
struct TcPlan {
    int TM, TN, KT;
    int dp, sk, psk;
};
struct Item {
    int tile, ks, ke;
};
struct WorkIt {
    int next_dp, u, u1;
};

__host__ __device__ __forceinline__ WorkIt work_begin(const TcPlan& p, int c, int P) {
    WorkIt w;
    w.next_dp = c;
    const int W = p.sk * p.KT;
    w.u = c < p.psk ? run_begin(c, W, p.psk) : 0;
    w.u1 = c < p.psk ? run_begin(c + 1, W, p.psk) : 0;
    return w;
}

__host__ __device__ __forceinline__ bool work_next(WorkIt& w, const TcPlan& p, int P, Item& it) {
    if (w.u < w.u1) {
        const int tl = w.u / p.KT;
        it.tile = p.dp + tl;
        it.ks = w.u - tl * p.KT;
        it.ke = p.KT < it.ks + (w.u1 - w.u) ? p.KT : it.ks + (w.u1 - w.u);
        w.u += it.ke - it.ks;
        return true;
    }
    if (w.next_dp < p.dp) {
        it.tile = w.next_dp;
        it.ks = 0;
        it.ke = p.KT;
        w.next_dp += P;
        return true;
    }
    return false;
}

// Tile t -> (M-tile, N-tile): groups of kGroupM M-tiles, N-major inside a group.
__host__ __device__ __forceinline__ void tile_coords(int t, const TcPlan& p, int& tm, int& tn) {
    const int per_group = kGroupM * p.TN;
    const int g = t / per_group;
    const int rem = t - g * per_group;
    const int gm = kGroupM < p.TM - g * kGroupM ? kGroupM : p.TM - g * kGroupM;
    tn = rem / gm;
    tm = g * kGroupM + (rem - tn * gm);
}

// Work split of one prefill projection over P persistent CTAs: whole tiles
// round-robin for every full wave, and a stream-K run over a partial last
// wave unless it is nearly full (>= 85 % of the CTAs) or there is no workspace
// for split tiles.  A split tile is cut at most 4 ways (finishing it reads the
// other pieces' 128 KB partials back).
inline void plan_tc(int T, int KT, int P, bool can_split, TcPlan* p, int* grid) {
    p->dp = T;
    p->sk = 0;
    p->psk = 0;
    *grid = T < P ? T : P;
    if (!can_split || T % P == 0 || KT < 2) return;
    const int full = T / P, R = T % P;
    if (full >= 1 && R * 100 >= 85 * P) return;
    p->dp = full * P;
    p->sk = R;
    long long psk = std::min<long long>(std::min<long long>(P, 4LL * R), static_cast<long long>(R) * KT);
    if (static_cast<long long>(R) * KT * psk >= (1LL << 31)) {   // keep unit arithmetic in int
        p->dp = T;
        p->sk = 0;
        return;
    }
    p->psk = static_cast<int>(psk);
    *grid = full >= 1 ? P : p->psk;
}

}  // namespace llb
