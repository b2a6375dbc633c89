// 16-bit (bf16 or fp16) projections on the 5th-generation tensor cores (tcgen05), fed by TMA,
// accumulating in TMEM, with the fused epilogues of the forward pass
// (Admin Guide §8.4: wq/wk/wv + RoPE + KV-cache append, wo + residual,
// w1/w3 + silu*mul, w2 + residual, output projection).
//
// This file holds the prefill-shaped kernel (many token rows); decode-shaped
// projections (<= 64 rows) run in gemm_decode.cu.
//
// D[i, j] = sum_k A[i, k] * B[j, k]; A = activations [tokens, K], B = weights
// [N, K], both K-major 16-bit read through 128-byte-swizzled TMA boxes of 64
// K-elements.  D is cut into 128 x 256 tiles, ordered in groups of 16 tiles
// along M (all N-tiles of one group before the next group), so that the
// tiles in flight at any time share a few hundred KB of A and B in L2.
//
// The kernel is persistent: one CTA per SM walks a fixed list of work items.
// The first `dp` tiles (all full waves) go round-robin, one whole tile per
// item: the CTAs of a wave walk K in step, so the A and B tiles in flight at
// any moment share a few MB of L2.  The `sk` tiles of a partial last wave form
// one flat run of sk * K/64 k-tile units cut into psk equal contiguous runs
// (stream-K, at most 4 runs per tile), so the SMs end together; each CTA
// takes its stream-K run before its whole tiles.  A tile split between CTAs
// is finished by the contributor that arrives last at the tile's counter: it
// adds the fp32 partials in CTA order (deterministic) and applies the
// epilogue while its MMAs go on with the whole tiles; no CTA ever waits for
// another.
//
// Warp roles (320 threads):
//   warp 0 lane 0  TMA producer (4-deep ring of 128x64 A + 256x64 B tiles)
//   warp 1 lane 0  MMA issuer (tcgen05.mma kind::f16, M=128, N=256, K=16)
//   warp 1         TMEM owner: two 256-column accumulators, so the MMAs of
//                  one item run while the epilogue drains the previous one
//   warps 2-9      epilogue: warp w reads TMEM lanes 32*(w%4)..+31 = token rows,
//                  warps 2-5 the tile's first 128 columns, warps 6-9 the other
//                  128 (twice the epilogue's loads and stores in flight); each
//                  warp owns 4 KB of shared memory for staging fp32 outputs
// Shared memory: the operand ring, then the epilogue staging (8 x 4 KB),
// then the barriers.  Every wait is bounded; no TMA multicast.
#include "common.cuh"
#include "epilogue.cuh"
#include "model.h"
#include "work_split.cuh"

#include <algorithm>
#include <cudaTypedefs.h>

namespace llb {

namespace {

constexpr int kEpiThreads = 256;             // eight epilogue warps: two per TMEM lane quarter
constexpr int kThreadsTc = 64 + kEpiThreads;
constexpr int kBN = 256;                     // tile width along N (weight rows)
constexpr int kStagesTc = 4;
constexpr int kA_BYTES = 128 * 128;          // 128 rows x 64 16-bit values
constexpr int kB_BYTES = kBN * 128;
constexpr int kStageBytes = kA_BYTES + kB_BYTES;
constexpr int kPartFloats = 128 * kBN;       // one fp32 partial tile
constexpr int kStgBytes = (kEpiThreads / 32) * 32 * 32 * 4;   // epilogue staging: 32 x 32 fp32 per warp

// A tile's epilogue inputs that do not depend on its accumulator, taken
// while its MMAs run: 1/rms of token row m (the consumer side of a fused
// RMSNorm over K features, from the row's per-128-feature sums of squares)
// and, for a residual epilogue, the 128 residual features n0.. of row m that
// this warp will add into, pulled into L2.
__device__ __forceinline__ void epi_tile_inputs(const Epi& ep, const NormIO& nio, int m, bool row_ok, int n0, int rowsB,
                                                int K, float& rs) {
    if (!row_ok) return;
    if (nio.ssq_in) rs = rsqrtf(row_ssq(nio.ssq_in + static_cast<long long>(m) * nio.n_in, nio.n_in) /
                                    static_cast<float>(K) + nio.eps);
    if (ep.mode == EPI_RESID_F32 && n0 < rowsB && (ep.ldo % 4) == 0) {
        const int nf = rowsB - n0 < 128 ? rowsB - n0 : 128;
        bulk_prefetch_l2(ep.out + static_cast<long long>(m) * ep.ldo + n0, static_cast<uint32_t>((nf * 4 + 15) & ~15));
    }
}

// Epilogue of one 32 x 32 block of a tile: token rows m0..m0+31 (one warp's
// TMEM lane quarter; lane = row as tcgen05.ld delivers it) x output features
// n0..n0+31, after the consumer side of a fused RMSNorm (scale by the row's
// 1/rms).  The 16-bit outputs (q/k/v with RoPE, silu(w1 x) * w3 x) are
// written straight from the lane's row: 64 or 32 contiguous bytes each.  The
// fp32 outputs (residual add, stores) go through the warp's 4 KB of shared
// memory so that every global access is row-contiguous: phase 1 writes the
// lane's row as float4s whose slot is XOR-swizzled by the row (conflict-free
// both ways), phase 2 has lane = (row rr of a group of 4, float4 column f):
// 4 rows x 128 bytes per warp access instead of 32 rows x 16 bytes.  `sq`
// accumulates the lane's row's sum of x^2 for the next RMSNorm; it is written
// when the chunk closes a 128-feature block.
template <typename E>
__device__ __forceinline__ void epi_block(const Epi& ep, const NormIO& nio, int m0, int n0, int rowsA, int rowsB,
                                          float rs, float (&v)[32], float4* stg, int lane, float& sq) {
    if (n0 >= rowsB) return;   // the same for the whole warp
    if (nio.ssq_in) {
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] *= rs;
    }
    const int sw = lane & 7;
    const int mrow = m0 + lane;
    if (ep.mode == EPI_SWIGLU) {
        // lane = token row: each 32-column chunk holds 16 w1 outputs, then the
        // same 16 w3 outputs; 32 bytes of g per row
        if (mrow >= rowsA) return;
        float g16[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) g16[t] = __fdividef(v[t], 1.f + __expf(-v[t])) * v[16 + t];
        uint4* d4 = reinterpret_cast<uint4*>(static_cast<E*>(ep.g) + static_cast<long long>(mrow) * ep.H + (n0 / 32) * 16);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            uint4 u;
            u.x = pack2<E>(g16[8 * q + 0], g16[8 * q + 1]);
            u.y = pack2<E>(g16[8 * q + 2], g16[8 * q + 3]);
            u.z = pack2<E>(g16[8 * q + 4], g16[8 * q + 5]);
            u.w = pack2<E>(g16[8 * q + 6], g16[8 * q + 7]);
            d4[q] = u;
        }
        return;
    }
    if (ep.mode == EPI_QKV) {
        // lane = token row: RoPE on q and k, 64 bytes to q or to the cache
        // (the chunk lies inside one head of q, k or v: hd is a multiple of 32)
        if (mrow >= rowsA) return;
        const int pos = ep.tok_pos[mrow];
        if (pos < 0 || pos >= ep.max_seq) return;
        E* dst;
        bool rot = true;
        int d0;
        if (n0 < ep.nq) {
            d0 = n0 % ep.hd;
            dst = static_cast<E*>(ep.q) + static_cast<long long>(mrow) * ep.nq + n0;
        } else {
            int cc = n0 - ep.nq;
            E* cache = static_cast<E*>(ep.kc);
            if (cc >= ep.nkvc) {
                cc -= ep.nkvc;
                cache = static_cast<E*>(ep.vc);
                rot = false;
            }
            const int head = cc / ep.hd;
            d0 = cc % ep.hd;
            const int row = ep.tok_row ? ep.tok_row[mrow] : mrow;
            dst = cache + static_cast<long long>(row) * ep.kv_row_stride +
                  (static_cast<long long>(head) * ep.max_seq + pos) * ep.hd + d0;
        }
        if (rot) {
            // (cos, sin) of rotation pairs d0/2 .. d0/2 + 15, two per float4
            const float4* cs4 = reinterpret_cast<const float4*>(ep.rope + static_cast<long long>(pos) * (ep.hd / 2) + (d0 >> 1));
#pragma unroll
            for (int t = 0; t < 32; t += 4) {
                const float4 cs = cs4[t >> 2];
                const float a0 = v[t] * cs.x - v[t + 1] * cs.y, b0 = v[t] * cs.y + v[t + 1] * cs.x;
                const float a1 = v[t + 2] * cs.z - v[t + 3] * cs.w, b1 = v[t + 2] * cs.w + v[t + 3] * cs.z;
                v[t] = a0;
                v[t + 1] = b0;
                v[t + 2] = a1;
                v[t + 3] = b1;
            }
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack2<E>(v[8 * q + 0], v[8 * q + 1]);
            u.y = pack2<E>(v[8 * q + 2], v[8 * q + 3]);
            u.z = pack2<E>(v[8 * q + 4], v[8 * q + 5]);
            u.w = pack2<E>(v[8 * q + 6], v[8 * q + 7]);
            d4[q] = u;
        }
        return;
    }
    // fp32 outputs: staged
#pragma unroll
    for (int qq = 0; qq < 8; ++qq)
        stg[lane * 8 + (qq ^ sw)] = make_float4(v[4 * qq], v[4 * qq + 1], v[4 * qq + 2], v[4 * qq + 3]);
    __syncwarp();
    const int f = lane & 7;
    const int n = n0 + 4 * f;
    if (nio.ssq_out) {
        // x += acc; y = x * w_next in E (rowsB % 128 == 0, ldo == rowsB); x
        // back into the staging slots, then lane = row again for its sum of x^2
        const float4 w = *reinterpret_cast<const float4*>(nio.w_next + n);
        float4 p[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int m = m0 + it * 4 + (lane >> 3);
            p[it] = m < rowsA ? *reinterpret_cast<const float4*>(ep.out + static_cast<long long>(m) * ep.ldo + n)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + (lane >> 3);
            const int m = m0 + rr;
            float4& slot = stg[rr * 8 + (f ^ (rr & 7))];
            const float4 x = slot;
            const float4 o = make_float4(p[it].x + x.x, p[it].y + x.y, p[it].z + x.z, p[it].w + x.w);
            slot = o;
            if (m < rowsA) {
                *reinterpret_cast<float4*>(ep.out + static_cast<long long>(m) * ep.ldo + n) = o;
                uint2 u;
                u.x = pack2<E>(o.x * w.x, o.y * w.y);
                u.y = pack2<E>(o.z * w.z, o.w * w.w);
                *reinterpret_cast<uint2*>(static_cast<E*>(nio.y_out) + static_cast<long long>(m) * ep.ldo + n) = u;
            }
        }
        __syncwarp();
#pragma unroll
        for (int qq = 0; qq < 8; ++qq) {
            const float4 o = stg[lane * 8 + (qq ^ sw)];
            sq += o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
        }
        if (((n0 + 32) & 127) == 0 || n0 + 32 >= rowsB) {
            const int m = m0 + lane;
            if (m < rowsA) nio.ssq_out[static_cast<long long>(m) * ((rowsB + 127) / 128) + n0 / 128] = sq;
            sq = 0.f;
        }
    } else {
        // fp32 store, or residual add (x += acc)
        const bool resid = ep.mode == EPI_RESID_F32;
        const bool vec = n + 4 <= rowsB && (ep.ldo % 4) == 0;
        float4 p[8];
        if (resid) {
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int m = m0 + it * 4 + (lane >> 3);
                p[it] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (m < rowsA && vec) p[it] = *reinterpret_cast<const float4*>(ep.out + static_cast<long long>(m) * ep.ldo + n);
            }
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + (lane >> 3);
            const int m = m0 + rr;
            float4 x = stg[rr * 8 + (f ^ (rr & 7))];
            float* o = ep.out + static_cast<long long>(m) * ep.ldo + n;
            if (m < rowsA && vec) {
                if (resid) x = make_float4(p[it].x + x.x, p[it].y + x.y, p[it].z + x.z, p[it].w + x.w);
                *reinterpret_cast<float4*>(o) = x;
            } else if (m < rowsA) {
                if (n < rowsB) o[0] = resid ? o[0] + x.x : x.x;
                if (n + 1 < rowsB) o[1] = resid ? o[1] + x.y : x.y;
                if (n + 2 < rowsB) o[2] = resid ? o[2] + x.z : x.z;
                if (n + 3 < rowsB) o[3] = resid ? o[3] + x.w : x.w;
            }
        }
    }
    __syncwarp();
}

}  // namespace

template <typename E>
__global__ void __launch_bounds__(kThreadsTc, 1)
linear_tcp_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                  int rowsA, int rowsB, TcPlan plan, Epi ep, float* __restrict__ part, int* __restrict__ counters,
                  NormIO nio) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float4* stg_all = reinterpret_cast<float4*>(smem + kStagesTc * kStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStagesTc * kStageBytes + kStgBytes);
    uint64_t* empty = full + kStagesTc;
    uint64_t* tfull = empty + kStagesTc;   // [2]
    uint64_t* tempty = tfull + 2;          // [2]
    uint64_t* mdone = tempty + 2;          // the MMA issuer's last commit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
    int* flag = reinterpret_cast<int*>(tmem_slot + 1);   // [0] abort, [1] arrival broadcast

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, c = blockIdx.x;
    const int KT = plan.KT;
    const uint64_t wlim = ep.wait_ns > 0 ? static_cast<uint64_t>(ep.wait_ns) : kWaitLimitNs;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesTc; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], kEpiThreads); }
        mbar_init(mdone, 1);
        flag[0] = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapA);
        tma_prefetch_desc(&mapB);
    }
    if (warp == 1) { tmem_alloc(tmem_slot, 2 * kBN); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int issued = 0, stall = -1;   // producer: stages [0, issued) were issued, all but `stall`
    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        stall = c == 0 ? ep.stall - 1 : -1;   // tests of the timeout path only
        WorkIt w = work_begin(plan, c, P);
        Item it;
        int i = 0;
        bool abort = false;
        while (!abort && work_next(w, plan, P, it)) {
            int tm, tn;
            tile_coords(it.tile, plan, tm, tn);
            for (int k = it.ks; k < it.ke; ++k, ++i) {
                const int s = i % kStagesTc;
                if (!mbar_wait(&empty[s], ((i / kStagesTc) & 1) ^ 1, wlim)) { atomicExch(&flag[0], 1); abort = true; break; }
                if (i != stall) {
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    uint8_t* st = smem + s * kStageBytes;
                    tma_load_2d(st, &mapA, k * 64, tm * 128, &full[s]);
                    tma_load_2d(st + kA_BYTES, &mapB, k * 64, tn * kBN, &full[s]);
                }
                issued = i + 1;
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        const uint32_t idesc = idesc_16_f32<E>(128, kBN);
        WorkIt w = work_begin(plan, c, P);
        Item it;
        int i = 0, j = 0;
        bool abort = false;
        while (!abort && work_next(w, plan, P, it)) {
            const int acc = j & 1;
            if (!mbar_wait(&tempty[acc], ((j >> 1) & 1) ^ 1, wlim)) { atomicExch(&flag[0], 1); break; }
            tc_fence_after();
            const uint32_t d = tmem + acc * kBN;
            for (int k = it.ks; k < it.ke; ++k, ++i) {
                const int s = i % kStagesTc;
                if (!mbar_wait(&full[s], (i / kStagesTc) & 1, wlim)) { atomicExch(&flag[0], 1); abort = true; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * kStageBytes);
                const uint32_t b0 = a0 + kA_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_16(d, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                                (k > it.ks || kk > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            tc_commit(&tfull[acc]);
            ++j;
        }
        // every MMA issued here has finished before TMEM is freed
        tc_commit(mdone);
        if (!mbar_wait(mdone, 0, wlim)) atomicExch(&flag[0], 1);
    } else if (warp >= 2) {
        // ---------------- epilogue: thread = token row of the tile, TMEM columns = features
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const int epi_tid = threadIdx.x - 64;
        float4* stg = stg_all + (warp - 2) * 256;   // this warp's 32 x 32 fp32 staging block
        const int c_lo = ((warp - 2) >> 2) * 4;   // warps 2-5: 32-column chunks 0-3, warps 6-9: chunks 4-7
        const int Wsk = plan.sk * KT;
        const int Psk = plan.psk;
        const int u0 = c < Psk ? run_begin(c, Wsk, Psk) : 0;
        WorkIt w = work_begin(plan, c, P);
        Item it;
        int j = 0;
        while (work_next(w, plan, P, it)) {
            const int acc = j & 1;
            int tm, tn;
            tile_coords(it.tile, plan, tm, tn);
            const int m = tm * 128 + r;
            const bool row_ok = m < rowsA;
            const uint32_t tb = tmem + lane_base + acc * kBN;
            const int nbase = tn * kBN;
            float rs = 1.f, sq = 0.f;
            epi_tile_inputs(ep, nio, m, row_ok, nbase + c_lo * 32, rowsB, KT * 64, rs);
            // one thread waits for the accumulator; the named barrier releases the others
            const bool ok_wait = epi_tid != 0 || mbar_wait(&tfull[acc], (j >> 1) & 1, wlim);
            if (named_any(1, kEpiThreads, !ok_wait || *reinterpret_cast<volatile int*>(&flag[0]) != 0)) {
                if (epi_tid == 0) report_status(ep.status, LLAMA_ERR_DEVICE_TIMEOUT);
                break;
            }
            tc_fence_after();
            ++j;
            // a split tile: publish this CTA's partial (feature-major, coalesced
            // over rows); only the last contributor to arrive goes on
            const bool whole = it.ks == 0 && it.ke == KT;
            const int tl = it.tile - plan.dp;
            const int ub = tl * KT;
            const int cf = whole ? c : owner(ub, Wsk, Psk), cl = whole ? c : owner(ub + KT - 1, Wsk, Psk);
            if (!whole) {
                const int slot = (ub + it.ks == u0) ? 0 : 1;   // the run's first segment, or its last
                float* my = part + (static_cast<long long>(c) * 2 + slot) * kPartFloats + r;
#pragma unroll 1
                for (int cc = c_lo; cc < c_lo + 4; ++cc) {
                    float v[32];
                    tmem_ld_32x32b_x32(tb + cc * 32, v);
                    tc_wait_ld();
#pragma unroll
                    for (int t = 0; t < 32; ++t) my[(cc * 32 + t) * 128] = v[t];
                }
                __threadfence();
                named_sync(1, kEpiThreads);
                if (epi_tid == 0) flag[1] = atomicAdd(&counters[tl], 1);
                named_sync(1, kEpiThreads);
                if (flag[1] != cl - cf) {   // not the last contributor
                    tc_fence_before();
                    mbar_arrive(&tempty[acc]);
                    continue;
                }
                __threadfence();
            }
            if (!whole) {
                // the last contributor: its accumulator is in its published
                // partial as well, so the MMAs get it back now
                tc_fence_before();
                mbar_arrive(&tempty[acc]);
            }
            // TMEM, or the contributors' partials summed in CTA order
            // -> epilogue, 32 features at a time
#pragma unroll 1
            for (int cc = c_lo; cc < c_lo + 4; ++cc) {
                float v[32];
                if (whole) {
                    tmem_ld_32x32b_x32(tb + cc * 32, v);
                    tc_wait_ld();
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) v[t] = 0.f;
                    for (int cb = cf; cb <= cl; ++cb) {
                        const int sl = run_begin(cb, Wsk, Psk) >= ub ? 0 : 1;
                        const float* pp = part + (static_cast<long long>(cb) * 2 + sl) * kPartFloats + r;
                        float f[32];
#pragma unroll
                        for (int t = 0; t < 32; ++t) f[t] = pp[(cc * 32 + t) * 128];
#pragma unroll
                        for (int t = 0; t < 32; ++t) v[t] += f[t];
                    }
                }
                epi_block<E>(ep, nio, m - lane, nbase + cc * 32, rowsA, rowsB, rs, v, stg, lane, sq);
            }
            if (whole) {
                tc_fence_before();
                mbar_arrive(&tempty[acc]);
            } else if (epi_tid == 0) {
                counters[tl] = 0;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&flag[0]) != 0) {
        // the CTA gave up: the copies it still has in flight land before it
        // exits (the newest stage of each ring slot; a skipped one is not waited for)
        for (int s = 0; s < kStagesTc; ++s) {
            if (issued <= s) continue;
            int jn = s + ((issued - 1 - s) / kStagesTc) * kStagesTc;
            if (jn == stall) jn -= kStagesTc;
            if (jn >= 0) mbar_wait(&full[s], (jn / kStagesTc) & 1, wlim);
        }
    }
    if (warp == 1) tmem_dealloc(tmem, 2 * kBN);
    if (threadIdx.x == 0) tl_stamp(ep.tl);
}

// ---------------------------------------------------------------- CTA-pair kernel
// The same projection with 256 x 256 tiles on a pair of SMs (a cluster of two
// CTAs, cta_group::2).  CTA rank r of a pair holds token rows r*128..+127 of
// the tile (the A half) and weight rows r*128..+127 (the B half); the rank-0
// CTA issues M=256, N=256 MMAs that read both CTAs' halves from their shared
// memory, and each CTA's tensor memory receives its 128 token rows over all
// 256 features, so each CTA runs the same epilogue as the one-SM kernel on
// its half.  Per 64-deep k-block an SM receives 32 KB of operands instead of
// 48 KB for the same MMA work, and a 6-stage ring covers 6 k-blocks of
// latency instead of 4.
//
// Handshakes (every wait bounded):
//   full[s]    rank 0: both CTAs' TMA copies of stage s landed (each CTA's
//              copies complete on rank 0's barrier; rank 0 expects both)
//   empty[s]   each CTA: the MMAs reading stage s are done (rank 0 commits to
//              its own and to the peer's barrier)
//   tfull[a]   each CTA: accumulator a is complete (both commits likewise)
//   tempty[a]  rank 0: both CTAs' epilogues drained accumulator a (count 2)
// A CTA that gives up cannot wait on rank 0's barrier for its own copies, so
// on that path rank 1 lets kDrainNs pass before it leaves (a copy lands within
// microseconds) and rank 0 waits for the stages it expected.
// A split tile is reduced per half: counters[2 * tile + r], partials of CTA
// (2 * pair + r).  No TMA multicast.
constexpr int kPairTile = 256;
constexpr int kStagesPair = 6;
constexpr int kPairHalfBytes = 128 * 128;            // 128 rows x 64 16-bit values
constexpr int kPairStageBytes = 2 * kPairHalfBytes;  // A half + B half
constexpr uint64_t kDrainNs = 100000;                // rank 1's wait for its copies on the give-up path

template <typename E>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsTc, 1)
linear_tcp_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                       int rowsA, int rowsB, TcPlan plan, Epi ep, float* __restrict__ part,
                       int* __restrict__ counters, NormIO nio) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float4* stg_all = reinterpret_cast<float4*>(smem + kStagesPair * kPairStageBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStagesPair * kPairStageBytes + kStgBytes);
    uint64_t* empty = full + kStagesPair;
    uint64_t* tfull = empty + kStagesPair;   // [2]
    uint64_t* tempty = tfull + 2;            // [2]
    uint64_t* mdone = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
    int* flag = reinterpret_cast<int*>(tmem_slot + 1);   // [0] abort, [1] arrival broadcast

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t peer = rank ^ 1u;
    const int P = gridDim.x >> 1, c = blockIdx.x >> 1;   // pairs
    const int KT = plan.KT;
    const uint64_t wlim = ep.wait_ns > 0 ? static_cast<uint64_t>(ep.wait_ns) : kWaitLimitNs;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesPair; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 2); }
        mbar_init(mdone, 1);
        flag[0] = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapA);
        tma_prefetch_desc(&mapB);
    }
    if (warp == 1) { tmem_alloc_pair(tmem_slot, 2 * kPairTile); tmem_relinquish_pair(); }
    tc_fence_before();
    cluster_sync();   // both CTAs' barriers initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int issued = 0, stall = -1;   // producer: stages [0, issued) were issued, all but `stall`
    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer (both CTAs): this CTA's A and B halves
        stall = blockIdx.x == 0 ? ep.stall - 1 : -1;   // tests of the timeout path only (rank 0 of pair 0)
        WorkIt w = work_begin(plan, c, P);
        Item it;
        int i = 0;
        bool abort = false;
        while (!abort && work_next(w, plan, P, it)) {
            int tm, tn;
            tile_coords(it.tile, plan, tm, tn);
            for (int k = it.ks; k < it.ke; ++k, ++i) {
                const int s = i % kStagesPair;
                if (!mbar_wait(&empty[s], ((i / kStagesPair) & 1) ^ 1, wlim)) { atomicExch(&flag[0], 1); abort = true; break; }
                if (i != stall) {
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kPairStageBytes);
                    uint8_t* st = smem + s * kPairStageBytes;
                    const uint32_t fb = cluster_addr(&full[s], 0);
                    tma_load_2d_pair(st, &mapA, k * 64, tm * kPairTile + static_cast<int>(rank) * 128, fb);
                    tma_load_2d_pair(st + kPairHalfBytes, &mapB, k * 64,
                                     tn * kPairTile + static_cast<int>(rank) * 128, fb);
                }
                issued = i + 1;
            }
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ---------------- MMA issuer (rank 0)
        const uint32_t idesc = idesc_16_f32<E>(kPairTile, kPairTile);
        WorkIt w = work_begin(plan, c, P);
        Item it;
        int i = 0, j = 0;
        bool abort = false;
        while (!abort && work_next(w, plan, P, it)) {
            const int acc = j & 1;
            if (!mbar_wait_cluster(&tempty[acc], ((j >> 1) & 1) ^ 1, wlim)) { atomicExch(&flag[0], 1); break; }
            tc_fence_after();
            const uint32_t d = tmem + acc * kPairTile;
            for (int k = it.ks; k < it.ke; ++k, ++i) {
                const int s = i % kStagesPair;
                const uint32_t par = (i / kStagesPair) & 1;
                if (!mbar_wait(&full[s], par, wlim)) {
                    atomicExch(&flag[0], 1);
                    abort = true;
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * kPairStageBytes);
                const uint32_t b0 = a0 + kPairHalfBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_16_pair(d, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                                   (k > it.ks || kk > 0) ? 1u : 0u);
                tc_commit_pair(smem_u32(&empty[s]));
                tc_commit_pair(cluster_addr(&empty[s], peer));
            }
            tc_commit_pair(smem_u32(&tfull[acc]));
            tc_commit_pair(cluster_addr(&tfull[acc], peer));
            ++j;
        }
        // every pair MMA issued here has finished before either CTA frees its
        // tensor memory or shared memory
        tc_commit_pair(smem_u32(mdone));
        if (!mbar_wait(mdone, 0, wlim)) atomicExch(&flag[0], 1);
    } else if (warp >= 2) {
        // ---------------- epilogue (both CTAs): thread = token row of this CTA's half
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const int epi_tid = threadIdx.x - 64;
        float4* stg = stg_all + (warp - 2) * 256;   // this warp's 32 x 32 fp32 staging block
        const int c_lo = ((warp - 2) >> 2) * 4;   // warps 2-5: 32-column chunks 0-3, warps 6-9: chunks 4-7
        const int Wsk = plan.sk * KT;
        const int Psk = plan.psk;
        const int u0 = c < Psk ? run_begin(c, Wsk, Psk) : 0;
        const uint32_t tempty_rank0 = cluster_addr(tempty, 0);   // tempty[0] of rank 0; [1] is 8 bytes on
        WorkIt w = work_begin(plan, c, P);
        Item it;
        int j = 0;
        // hand accumulator `a` back to rank 0's MMA issuer: one arrive per CTA
        auto release = [&](int a) {
            tc_fence_before();
            named_sync(1, kEpiThreads);
            if (epi_tid == 0) mbar_arrive_cluster(tempty_rank0 + 8u * static_cast<uint32_t>(a));
        };
        while (work_next(w, plan, P, it)) {
            const int acc = j & 1;
            int tm, tn;
            tile_coords(it.tile, plan, tm, tn);
            const int m = tm * kPairTile + static_cast<int>(rank) * 128 + r;
            const bool row_ok = m < rowsA;
            const uint32_t tb = tmem + lane_base + acc * kPairTile;
            const int nbase = tn * kPairTile;
            float rs = 1.f, sq = 0.f;
            epi_tile_inputs(ep, nio, m, row_ok, nbase + c_lo * 32, rowsB, KT * 64, rs);
            // one thread waits for the accumulator; the named barrier releases the others
            const bool ok_wait = epi_tid != 0 || mbar_wait(&tfull[acc], (j >> 1) & 1, wlim);
            if (named_any(1, kEpiThreads, !ok_wait || *reinterpret_cast<volatile int*>(&flag[0]) != 0)) {
                if (epi_tid == 0) report_status(ep.status, LLAMA_ERR_DEVICE_TIMEOUT);
                break;
            }
            tc_fence_after();
            ++j;
            // a split tile: this CTA's half of it, reduced among the same halves
            // of the tile's other pairs (last arrival finishes, in pair order)
            const bool whole = it.ks == 0 && it.ke == KT;
            const int tl = it.tile - plan.dp;
            const int ub = tl * KT;
            const int cf = whole ? c : owner(ub, Wsk, Psk), cl = whole ? c : owner(ub + KT - 1, Wsk, Psk);
            const int cnt_idx = 2 * tl + static_cast<int>(rank);
            if (!whole) {
                const int slot = (ub + it.ks == u0) ? 0 : 1;
                float* my =
                    part + (static_cast<long long>(2 * c + static_cast<int>(rank)) * 2 + slot) * kPartFloats + r;
#pragma unroll 1
                for (int cc = c_lo; cc < c_lo + 4; ++cc) {
                    float v[32];
                    tmem_ld_32x32b_x32(tb + cc * 32, v);
                    tc_wait_ld();
#pragma unroll
                    for (int t = 0; t < 32; ++t) my[(cc * 32 + t) * 128] = v[t];
                }
                __threadfence();
                named_sync(1, kEpiThreads);
                if (epi_tid == 0) flag[1] = atomicAdd(&counters[cnt_idx], 1);
                named_sync(1, kEpiThreads);
                if (flag[1] != cl - cf) {
                    release(acc);
                    continue;
                }
                __threadfence();
            }
            if (!whole) release(acc);   // the last contributor's accumulator is in its partial too
#pragma unroll 1
            for (int cc = c_lo; cc < c_lo + 4; ++cc) {
                float v[32];
                if (whole) {
                    tmem_ld_32x32b_x32(tb + cc * 32, v);
                    tc_wait_ld();
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) v[t] = 0.f;
                    for (int cb = cf; cb <= cl; ++cb) {
                        const int sl = run_begin(cb, Wsk, Psk) >= ub ? 0 : 1;
                        const float* pp = part +
                            (static_cast<long long>(2 * cb + static_cast<int>(rank)) * 2 + sl) * kPartFloats + r;
                        float f[32];
#pragma unroll
                        for (int t = 0; t < 32; ++t) f[t] = pp[(cc * 32 + t) * 128];
#pragma unroll
                        for (int t = 0; t < 32; ++t) v[t] += f[t];
                    }
                }
                epi_block<E>(ep, nio, m - lane, nbase + cc * 32, rowsA, rowsB, rs, v, stg, lane, sq);
            }
            if (whole) release(acc);
            else if (epi_tid == 0) counters[cnt_idx] = 0;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&flag[0]) != 0) {
        // the CTA gave up: its copies still in flight land before it exits
        if (rank == 0) {
            // the newest stage of each ring slot (a stage the peer never
            // issued does not complete: that wait gives up after kDrainNs)
            for (int s = 0; s < kStagesPair; ++s) {
                if (issued <= s) continue;
                int jn = s + ((issued - 1 - s) / kStagesPair) * kStagesPair;
                if (jn == stall) jn -= kStagesPair;
                if (jn >= 0) mbar_wait(&full[s], (jn / kStagesPair) & 1, kDrainNs);
            }
        } else {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < kDrainNs) {
            }
        }
    }
    // neither CTA leaves while the other may still signal its barriers or
    // (rank 0's MMAs, waited for above) read its shared memory
    cluster_sync();
    if (warp == 1) tmem_dealloc_pair(tmem, 2 * kPairTile);
    if (threadIdx.x == 0) tl_stamp(ep.tl);
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int encode_kmajor_16(CUtensorMap* map, const void* base, int rows, int cols, int box_rows, int dtype) {
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || fn == nullptr || q != cudaDriverEntryPointSuccess) {
            set_error("cuTensorMapEncodeTiled unavailable");
            return LLAMA_ERR_CUDA;
        }
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (cols * 2) % 16) {
        set_error("TMA operand must be 16-byte aligned with rows a multiple of 16 bytes");
        return LLAMA_ERR_INVALID_ARG;
    }
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = dtype == LLAMA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) rows=%d cols=%d box=%d", static_cast<int>(r), rows,
                  cols, box_rows);
        return LLAMA_ERR_CUDA;
    }
    return LLAMA_OK;
}

static int g_sms_tc = 0;

template <typename E>
static int launch_tcp(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, const Epi& ep, float* part,
                      int* counters, cudaStream_t st, const NormIO& nio) {
    if (M <= 0 || N <= 0) return LLAMA_OK;
    constexpr int smem = 1024 + kStagesTc * kStageBytes + kStgBytes + (2 * kStagesTc + 5) * 8 + 16;
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(linear_tcp_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(linear_tcp_kernel)");
        attr_set = true;
    }
    if (g_sms_tc == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms_tc, cudaDevAttrMultiProcessorCount, dev);
        if (g_sms_tc <= 0) g_sms_tc = 148;
        if (g_sms_tc > kMaxPrefillCtas) g_sms_tc = kMaxPrefillCtas;
    }
    TcPlan plan;
    plan.TM = (M + 127) / 128;
    plan.TN = (N + kBN - 1) / kBN;
    plan.KT = (K + 63) / 64;
    const long long T = static_cast<long long>(plan.TM) * plan.TN;
    if (T >= (1LL << 30)) { set_error("prefill projection too large (%lld tiles)", T); return LLAMA_ERR_INVALID_ARG; }
    int grid = 0;
    plan_tc(static_cast<int>(T), plan.KT, g_sms_tc, part != nullptr && counters != nullptr, &plan, &grid);
    if (plan.sk > kMaxTiles) { set_error("internal: %d split tiles exceed the counters", plan.sk); return LLAMA_ERR_INVALID_ARG; }
    linear_tcp_kernel<E><<<grid, kThreadsTc, smem, st>>>(mapA->a128, mapW->b, M, N, plan, ep, part, counters, nio);
    LLB_CHECK_LAUNCH("linear_tcp_kernel");
    return LLAMA_OK;
}

// When a projection runs on CTA pairs: at least 256 token rows (fewer would
// leave most of a 256-row pair tile empty) and a weight matrix larger than
// 4096 x 4096.  Measured on the 7B prefill (4 x 512 tokens, interleaved runs,
// medians): pairs take w1/w3 (22016 x 4096) from 9.8 to 9.3 ms and w2
// (4096 x 11008) from 6.1 to 5.7 ms per prefill, wq/wk/wv (12288 x 4096) is
// even, and wo (4096 x 4096) goes from 3.4 to 3.9 ms, so it keeps one SM per
// tile.
constexpr int kPairMinRows = 256;
constexpr long long kPairMinWeights = 4096LL * 4096;

template <typename E>
static int launch_tcp_pair(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, const Epi& ep, float* part,
                           int* counters, cudaStream_t st, const NormIO& nio) {
    constexpr int smem = 1024 + kStagesPair * kPairStageBytes + kStgBytes + (2 * kStagesPair + 5) * 8 + 16;
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    auto kern = linear_tcp_pair_kernel<E>;
    static int pairs = 0;   // clusters of two that are resident at once
    if (pairs == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(linear_tcp_pair_kernel)");
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kMaxPrefillCtas);
        cfg.blockDim = dim3(kThreadsTc);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(linear_tcp_pair_kernel)");
        if (n < 1) { set_error("linear_tcp_pair_kernel: no CTA pair fits on this GPU"); return LLAMA_ERR_CUDA; }
        pairs = n < kMaxPrefillCtas / 2 ? n : kMaxPrefillCtas / 2;
    }
    TcPlan plan;
    plan.TM = (M + kPairTile - 1) / kPairTile;
    plan.TN = (N + kPairTile - 1) / kPairTile;
    plan.KT = (K + 63) / 64;
    const long long T = static_cast<long long>(plan.TM) * plan.TN;
    if (T >= (1LL << 30)) { set_error("prefill projection too large (%lld tiles)", T); return LLAMA_ERR_INVALID_ARG; }
    int grid = 0;
    plan_tc(static_cast<int>(T), plan.KT, pairs, part != nullptr && counters != nullptr, &plan, &grid);
    if (2 * plan.sk > kMaxTiles) {
        set_error("internal: %d split tile halves exceed the counters", 2 * plan.sk);
        return LLAMA_ERR_INVALID_ARG;
    }
    kern<<<2 * grid, kThreadsTc, smem, st>>>(mapA->a128, mapW->a128, M, N, plan, ep, part, counters, nio);
    LLB_CHECK_LAUNCH("linear_tcp_pair_kernel");
    return LLAMA_OK;
}

int linear16_tc(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, int dtype, const Epi& ep, float* part,
                int* counters, cudaStream_t st, const NormIO* nio_in) {
    NormIO nio = {};
    if (nio_in) nio = *nio_in;
    if (nio.ssq_out && (N % 128 || !nio.y_out || !nio.w_next || ep.mode != EPI_RESID_F32 || ep.ldo != N)) {
        set_error("fused RMSNorm producer needs a residual epilogue over whole rows, N %% 128 == 0, y_out and w_next");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (nio.ssq_in && K % 64) { set_error("fused RMSNorm consumer needs K %% 64 == 0"); return LLAMA_ERR_INVALID_ARG; }
    if (M <= 0 || N <= 0) return LLAMA_OK;
    if (M >= kPairMinRows && static_cast<long long>(N) * K > kPairMinWeights) {
        if (dtype == LLAMA_F16) return launch_tcp_pair<f16>(mapA, mapW, M, N, K, ep, part, counters, st, nio);
        if (dtype == LLAMA_BF16) return launch_tcp_pair<bf16>(mapA, mapW, M, N, K, ep, part, counters, st, nio);
    }
    if (dtype == LLAMA_F16) return launch_tcp<f16>(mapA, mapW, M, N, K, ep, part, counters, st, nio);
    if (dtype == LLAMA_BF16) return launch_tcp<bf16>(mapA, mapW, M, N, K, ep, part, counters, st, nio);
    set_error("16-bit projection: dtype must be LLAMA_BF16 or LLAMA_F16");
    return LLAMA_ERR_INVALID_ARG;
}

int linear16(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, int dtype, const Epi& ep, float* part,
             size_t part_bytes, int* counters, cudaStream_t st, bool pdl, const NormIO* nio) {
    if (M <= 64) return linear16_decode(mapA, mapW, M, N, K, dtype, ep, part, part_bytes, counters, st, pdl, nio);
    return linear16_tc(mapA, mapW, M, N, K, dtype, ep, part, counters, st, nio);
}

}  // namespace llb
