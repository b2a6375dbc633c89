// Pieces of the decode-shaped projection kernel (gemm_decode.cu): the walk
// over a run of stream-K units, the epilogue of a finished 128-row weight
// tile, and the epilogue warps' loop over a run's segments.
#pragma once

#include "common.cuh"
#include "epilogue.cuh"
#include "model.h"

namespace llb {

constexpr int kABytes = 128 * 128;  // 128 weight rows x 64 16-bit values: one A-operand ring stage

struct Seg {
    int tile, ks, ke;
};

// A tile whose k-range is split between the runs of CTAs cf .. cl (cf < cl) is
// finished by cf, the CTA holding its first unit: cf's run ends inside the
// tile (a run that held the whole tile would not split it), so that segment
// is the LAST of cf's run, while every other contributor's run starts inside
// the tile, so its segment is the FIRST of its run.  Each CTA therefore
// publishes at most one partial (its first segment, when it does not start at
// a tile boundary), early in its run, and the finisher, at the end of its
// own run, only has to collect them: it never publishes or counts itself.
__host__ __device__ __forceinline__ int split_finisher(int tile, int KT, int W, int P) {
    return owner(tile * KT, W, P);
}

// Next segment (one tile's k-range) of a run of units; false past the end.
__host__ __device__ __forceinline__ bool next_seg(int& u, int u1, int KT, Seg& s) {
    if (u >= u1) return false;
    s.tile = u / KT;
    s.ks = u - s.tile * KT;
    s.ke = KT < s.ks + (u1 - u) ? KT : s.ks + (u1 - u);
    u += s.ke - s.ks;
    return true;
}

// The inputs of a tile's epilogue that do not depend on its accumulator,
// loaded while its MMAs still run: the RoPE factors of each token column
// (QKV: from the row's position), or the old residual values and the next
// norm's weight (residual modes).
template <int BN>
struct EpiPre {
    float2 cs[BN];
    float xo[BN];
    float wn;
};

template <int BN>
__device__ __forceinline__ void prefetch_tile(EpiPre<BN>& pre, int t, int r, int nb, int N, const Epi& ep,
                                              const NormIO& nio, const int (&posv)[BN]) {
    const int n = t * 128 + r;
    const bool row_ok = n < N;
    if (ep.mode == EPI_QKV) {
        const bool is_q = n < ep.nq;
        const int cc = n - ep.nq;
        const bool rot = is_q || cc < ep.nkvc;
        const int d = is_q ? n % ep.hd : cc % ep.hd;
#pragma unroll
        for (int b = 0; b < BN; ++b) {
            const bool okp = row_ok && rot && posv[b] >= 0 && posv[b] < ep.max_seq;
            pre.cs[b] = okp ? ep.rope[static_cast<long long>(posv[b]) * (ep.hd / 2) + (d >> 1)] : make_float2(1.f, 0.f);
        }
    } else if (ep.mode == EPI_RESID_F32) {
        pre.wn = (row_ok && nio.ssq_out) ? nio.w_next[n] : 0.f;
#pragma unroll
        for (int b = 0; b < BN; ++b)
            pre.xo[b] = (row_ok && b < nb) ? ep.out[static_cast<long long>(b) * ep.ldo + n] : 0.f;
    }
}

// Epilogue of one finished 128-row weight tile t: v[b] = acc[row r of the
// tile, token column b] for the nb real token columns.  All 128 epilogue
// threads of the CTA call it together (the residual + sum-of-squares mode
// synchronises them on named barrier 2).  `pre` (or null: loaded here) holds
// the inputs prefetch_tile loaded; `posv` the token columns' positions.
template <int BN, typename T>
__device__ __forceinline__ void finish_tile(float (&v)[BN], int t, int r, int lane, int q, int epi_tid, int nb,
                                            int N, int n_tiles, const Epi& ep, const NormIO& nio, bool scale_in,
                                            const float* rs, float* red, const EpiPre<BN>* pre = nullptr,
                                            const int* posv_in = nullptr) {
    if (scale_in) {
#pragma unroll
        for (int b = 0; b < BN; ++b) v[b] *= (b < nb) ? rs[b] : 0.f;
    }
    const int n = t * 128 + r;
    const bool row_ok = n < N;
    if (ep.mode == EPI_SWIGLU) {
        // rows are interleaved in blocks of 16: lanes 0-15 of a warp hold
        // w1 rows, lanes 16-31 the matching w3 rows
#pragma unroll
        for (int b = 0; b < BN; ++b) {
            if (b >= nb) break;   // uniform over the CTA
            const float up = __shfl_xor_sync(0xffffffffu, v[b], 16);
            if (lane < 16 && row_ok && b < nb) {
                const int h = (n >> 5) * 16 + (n & 15);
                static_cast<T*>(ep.g)[static_cast<long long>(b) * ep.H + h] =
                    from_f32<T>(silu_f(v[b]) * up);
            }
        }
    } else if (ep.mode == EPI_QKV) {
        const bool even = (lane & 1) == 0;
        const bool is_q = n < ep.nq;
        int cc = n - ep.nq;
        T* cache = static_cast<T*>(ep.kc);
        const bool is_k = !is_q && cc < ep.nkvc;
        if (!is_q && !is_k) { cc -= ep.nkvc; cache = static_cast<T*>(ep.vc); }
        const int d = is_q ? n % ep.hd : cc % ep.hd;
        const int head = is_q ? 0 : cc / ep.hd;
        // per group of 16 columns: all positions and RoPE factors first
        // (independent loads), then the rotations and stores
#pragma unroll
        for (int b0 = 0; b0 < BN; b0 += 16) {
            int posv[16];
            float2 cs[16];
            if (pre) {
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    posv[u] = posv_in[b0 + u];
                    cs[u] = pre->cs[b0 + u];
                }
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) posv[u] = (b0 + u < nb) ? ep.tok_pos[b0 + u] : -1;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const bool okp = row_ok && posv[u] >= 0 && posv[u] < ep.max_seq && (is_q || is_k);
                    cs[u] = okp ? ep.rope[static_cast<long long>(posv[u]) * (ep.hd / 2) + (d >> 1)]
                                : make_float2(1.f, 0.f);
                }
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int b = b0 + u;
                if (b >= nb) break;   // uniform over the CTA
                const float partner = __shfl_xor_sync(0xffffffffu, v[b], 1);
                const int pos = posv[u];
                if (!row_ok || b >= nb || pos < 0 || pos >= ep.max_seq) continue;
                const float re = even ? v[b] : partner, im = even ? partner : v[b];
                const float rot = even ? re * cs[u].x - im * cs[u].y : re * cs[u].y + im * cs[u].x;
                if (is_q) {
                    static_cast<T*>(ep.q)[static_cast<long long>(b) * ep.nq + n] = from_f32<T>(rot);
                } else {
                    const int row = ep.tok_row ? ep.tok_row[b] : b;
                    cache[static_cast<long long>(row) * ep.kv_row_stride +
                          (static_cast<long long>(head) * ep.max_seq + pos) * ep.hd + d] =
                        from_f32<T>(is_k ? rot : v[b]);
                }
            }
        }
    } else if (ep.mode == EPI_RESID_F32 && nio.ssq_out) {
        // residual add, plus this tile's share of sum(x^2) for the next RMSNorm;
        // the old x values of a 16-column group are loaded together
        const float wn = pre ? pre->wn : (row_ok ? nio.w_next[n] : 0.f);
        float xo[16];   // v[b] becomes x^2 of column b below
#pragma unroll
        for (int b = 0; b < BN; ++b) {
            if (b >= nb) break;   // uniform over the CTA
            if ((b & 15) == 0) {
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    xo[u] = pre ? pre->xo[b + u]
                                : ((row_ok && b + u < nb) ? ep.out[static_cast<long long>(b + u) * ep.ldo + n] : 0.f);
            }
            float sq = 0.f;
            if (row_ok) {
                const float nv = xo[b & 15] + v[b];
                ep.out[static_cast<long long>(b) * ep.ldo + n] = nv;
                static_cast<T*>(nio.y_out)[static_cast<long long>(b) * ep.ldo + n] = from_f32<T>(nv * wn);
                sq = nv * nv;
            }
            v[b] = sq;
        }
        // the warp's column sums of x^2, 32 columns at a time, by a
        // transposing butterfly: after it lane l holds column c0 + l's sum
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 32) {
            if (c0 >= nb) break;   // uniform over the CTA
            float a[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) a[i] = (c0 + i < BN && c0 + i < nb) ? v[c0 + i] : 0.f;
#pragma unroll
            for (int step = 16, h = 16; step >= 1; step >>= 1, h >>= 1) {
                const bool upper = (lane & step) != 0;
#pragma unroll
                for (int i = 0; i < h; ++i) {
                    const float send = upper ? a[i] : a[i + h];
                    const float keep = upper ? a[i + h] : a[i];
                    a[i] = keep + __shfl_xor_sync(0xffffffffu, send, step);
                }
            }
            if (c0 + lane < nb) red[q * 64 + c0 + lane] = a[0];
        }
        named_sync(2, 128);
        if (epi_tid < nb)
            nio.ssq_out[epi_tid * n_tiles + t] = ((red[epi_tid] + red[64 + epi_tid]) + red[128 + epi_tid]) +
                                           red[192 + epi_tid];
        named_sync(2, 128);
    } else if (ep.mode == EPI_LOGITS_ARGMAX) {
        // logits (when kept) and this tile's share of each token column's
        // greedy pick: the warp's largest key, folded into best[b]
#pragma unroll
        for (int b = 0; b < BN; ++b) {
            if (b < nb) {   // uniform over the CTA
                unsigned long long key = 0;
                if (row_ok) {
                    if (ep.out) ep.out[static_cast<long long>(b) * ep.ldo + n] = v[b];
                    key = argmax_key(v[b], n);
                }
                key = warp_max_u64(key);
                if (lane == 0 && key) atomicMax(&ep.best[b], key);
            }
        }
    } else if (row_ok) {
        if (ep.mode == EPI_RESID_F32) {
#pragma unroll
            for (int b0 = 0; b0 < BN; b0 += 16) {
                float xo[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    xo[u] = pre ? pre->xo[b0 + u]
                                : ((b0 + u < nb) ? ep.out[static_cast<long long>(b0 + u) * ep.ldo + n] : 0.f);
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (b0 + u < nb) ep.out[static_cast<long long>(b0 + u) * ep.ldo + n] = xo[u] + v[b0 + u];
            }
        } else {
#pragma unroll
            for (int b = 0; b < BN; ++b)
                if (b < nb) ep.out[static_cast<long long>(b) * ep.ldo + n] = v[b];
        }
    }
}

// The epilogue warps' loop over the segments of one CTA's stream-K run of a
// decode projection: wait for each segment's accumulator (TMEM buffer j % 2,
// 64 columns apart; tmem_lane = TMEM base + this warp's lane quarter), read
// it, hand the buffer back to the MMA warp, then finish the tile, or publish
// this CTA's partial of a split tile it does not finish (and count it), or --
// as the split tile's finisher (split_finisher) -- wait until every other
// contributor has counted its partial, add them after its own in CTA order
// (deterministic) and finish the tile.  Runs are run_begin(c, W, P) ..
// run_begin(c + 1, W, P) over W = n_tiles * KT units; partials are one
// 128 x BN fp32 block per CTA.
template <int BN, typename T>
__device__ __forceinline__ void decode_epilogue_loop(uint32_t tmem_lane, uint64_t* tfull, uint64_t* tempty, int* flag,
                                                     float* part, int* counters, int c, int P, int u0, int u1,
                                                     int KT, int N, int M, const Epi& ep, const NormIO& nio,
                                                     bool scale_in, const float* rs, float* red, int r, int lane,
                                                     int q, int epi_tid, uint64_t wlim) {
    const int n_tiles = (N + 127) / 128;
    const int W = n_tiles * KT;
    int u = u0;
    Seg sg;
    int j = 0;
    const int nb = M < BN ? M : BN;
    // narrow steps load each finished tile's epilogue inputs while its MMAs run
    constexpr bool kPre = BN <= 32;
    int posv[BN];
#pragma unroll
    for (int b = 0; b < BN; ++b) posv[b] = (kPre && ep.mode == EPI_QKV && b < nb) ? ep.tok_pos[b] : -1;
    while (next_seg(u, u1, KT, sg)) {
        const int acc = j & 1;
        const int t = sg.tile;
        const int tb = t * KT;
        const int cf = split_finisher(t, KT, W, P), cl = owner(tb + KT - 1, W, P);
        EpiPre<BN> pre;
        if (kPre && !(cl > cf && c != cf)) prefetch_tile<BN>(pre, t, r, nb, N, ep, nio, posv);
        const bool ok_wait = mbar_wait(&tfull[acc], (j >> 1) & 1, wlim);
        tc_fence_after();
        float v[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 16; ++cc)
            tmem_ld_32x32b_x16(tmem_lane + acc * 64 + cc * 16, v + cc * 16);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        ++j;
        if (named_any(1, 128, !ok_wait || *reinterpret_cast<volatile int*>(&flag[0]) != 0)) {
            if (epi_tid == 0) report_status(ep.status, LLAMA_ERR_DEVICE_TIMEOUT);
            break;
        }
        if (cl > cf && c != cf) {
            // a split tile this CTA does not finish (its run's first segment):
            // publish the partial and count it
            float* my = part + (static_cast<long long>(c) * 128 + r) * BN;
#pragma unroll
            for (int b = 0; b < BN; b += 4)
                if (b < nb) *reinterpret_cast<float4*>(my + b) = make_float4(v[b], v[b + 1], v[b + 2], v[b + 3]);
            __threadfence();
            named_sync(1, 128);
            if (epi_tid == 0) atomicAdd(&counters[t], 1);
            continue;
        }
        if (cl > cf) {
            // the finisher (its run's last segment): the other cl - cf
            // contributors published theirs early in their runs
            if (epi_tid == 0) {
                const int need = cl - cf;
                const volatile int* cnt = counters + t;
                bool okc = *cnt >= need;
                if (!okc) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!(okc = *cnt >= need) && globaltimer_ns() - t0 <= wlim) {
                    }
                }
                flag[1] = okc ? 1 : 0;
            }
            named_sync(1, 128);
            if (!flag[1]) {
                if (epi_tid == 0) {
                    report_status(ep.status, LLAMA_ERR_DEVICE_TIMEOUT);
                    atomicExch(&flag[0], 1);
                }
                break;
            }
            __threadfence();
            // partials after this CTA's own, in CTA order.  Up to 4 token
            // columns: one float4 per contributor, 8 contributors per batch of
            // independent loads (each batch is an L2 round trip under full
            // HBM load); wider: see below.
            if (nb <= 4) {
                for (int cb = cf + 1; cb <= cl; cb += 8) {
                    float4 f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (cb + e <= cl)
                            f[e] = __ldcg(reinterpret_cast<const float4*>(part + (static_cast<long long>(cb + e) * 128 + r) * BN));
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (cb + e <= cl) {
                            v[0] += f[e].x;
                            v[1] += f[e].y;
                            v[2] += f[e].z;
                            v[3] += f[e].w;
                        }
                    }
                }
            }
            if (nb > 4) {
                // the real columns of one contributor's row per load group;
                // up to 32 columns, the next contributor's loads are issued
                // before this one's are added (two groups in flight)
                auto load = [&](float4 (&f)[BN / 4], int cc) {
                    const float4* pp = reinterpret_cast<const float4*>(part + (static_cast<long long>(cc) * 128 + r) * BN);
#pragma unroll
                    for (int qq = 0; qq < BN / 4; ++qq)
                        if (4 * qq < nb) f[qq] = __ldcg(pp + qq);
                };
                auto add = [&](const float4 (&f)[BN / 4]) {
#pragma unroll
                    for (int qq = 0; qq < BN / 4; ++qq) {
                        if (4 * qq < nb) {
                            v[4 * qq] += f[qq].x;
                            v[4 * qq + 1] += f[qq].y;
                            v[4 * qq + 2] += f[qq].z;
                            v[4 * qq + 3] += f[qq].w;
                        }
                    }
                };
                if constexpr (BN <= 32) {
                    float4 fa[BN / 4], fb[BN / 4];
                    load(fa, cf + 1);
                    for (int cb = cf + 1; cb <= cl; cb += 2) {
                        if (cb + 1 <= cl) load(fb, cb + 1);
                        add(fa);
                        if (cb + 2 <= cl) load(fa, cb + 2);
                        if (cb + 1 <= cl) add(fb);
                    }
                } else {
                    for (int cb = cf + 1; cb <= cl; ++cb) {
                        float4 f[BN / 4];
                        load(f, cb);
                        add(f);
                    }
                }
            }
            if (epi_tid == 0) counters[t] = 0;
        }
        finish_tile<BN, T>(v, t, r, lane, q, epi_tid, nb, N, n_tiles, ep, nio, scale_in, rs, red, kPre ? &pre : nullptr,
                           posv);
    }
}

}  // namespace llb
