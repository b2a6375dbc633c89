// Decode-shaped bf16 projections (few token rows) on tcgen05: a persistent,
// stream-K, weight-streaming kernel.
//
// acc[n, b] = sum_k W[n, k] * X[b, k] for b < M <= 64 token rows.  The weight
// W is the 128-row MMA operand (M=128, N=BN=16..64 token columns, K=16).
// The N/128 weight tiles x K/64 k-tiles form one flat list of work units;
// each of the P persistent CTAs (one per SM) takes an equal contiguous run
// of it, so every SM streams the same number of bytes whatever the matrix
// shape.  A tile whose k-range is split between CTAs is finished by the CTA
// that arrives last at the tile's counter: it adds the fp32 partials in CTA
// order (deterministic) and applies the epilogue.  A tile covered by one CTA
// goes straight from TMEM to the epilogue.
//
// Warp roles (192 threads): warp 0 = TMA producer (STAGES-deep ring), warp 1
// = MMA issuer and TMEM owner, warps 2-5 = epilogue (TMEM lanes 0-127).
//
// Fused RMSNorm (Admin Guide §8.4, RMSNorm before wq/wk/wv, before w1/w3 and
// before the output projection), see NormIO: a residual epilogue here also
// writes the next projection's operand bf16(x * w_next) and per-tile sums of
// x^2; a consuming projection scales accumulator column b by r_b.
// A deep ring (about 200 KB of weight tiles in flight per SM) keeps HBM
// busy; the next projection's CTAs launch early (programmatic dependent
// launch) and start streaming as soon as this kernel's CTAs leave their SMs.
// (Extra L2 prefetches of weight tiles that are bulk-loaded soon after were
// measured to lower the streaming rate, so there are none.)  Two TMEM accumulators let the MMA of the next segment overlap the epilogue
// of the previous one.  With programmatic dependent launch, weight tiles are
// requested before the previous kernel has finished; the activation tiles
// and every global read of the epilogue wait for it (griddepcontrol.wait).
// Every wait is bounded; no TMA multicast.
#include "common.cuh"
#include "epilogue.cuh"
#include "model.h"

namespace llb {

namespace {
constexpr int kThreads = 192;
constexpr int kAccStride = 64;      // TMEM columns per accumulator buffer
constexpr int kTmemCols = 128;      // two accumulator buffers
constexpr int kABytes = 128 * 128;  // 128 weight rows x 64 bf16

struct Seg {
    int tile, ks, ke;
};

// Next segment (one tile's k-range) of a run of units; false past the end.
__device__ __forceinline__ bool next_seg(int& u, int u1, int KT, Seg& s) {
    if (u >= u1) return false;
    s.tile = u / KT;
    s.ks = u - s.tile * KT;
    s.ke = min(KT, s.ks + (u1 - u));
    u += s.ke - s.ks;
    return true;
}
}  // namespace

// Epilogue of one finished 128-row weight tile t: v[b] = acc[row r of the
// tile, token column b] for the nb real token columns.  All 128 epilogue
// threads of the CTA call it together (the residual + sum-of-squares mode
// synchronises them on named barrier 2).
template <int BN>
__device__ __forceinline__ void finish_tile(float (&v)[BN], int t, int r, int lane, int q, int epi_tid, int nb,
                                            int N, int T, const Epi& ep, const NormIO& nio, bool scale_in,
                                            const float* rs, float* red) {
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
            const float up = __shfl_xor_sync(0xffffffffu, v[b], 16);
            if (lane < 16 && row_ok && b < nb) {
                const int h = (n >> 5) * 16 + (n & 15);
                static_cast<bf16*>(ep.g)[static_cast<long long>(b) * ep.H + h] =
                    __float2bfloat16_rn(silu_f(v[b]) * up);
            }
        }
    } else if (ep.mode == EPI_QKV) {
        const bool even = (lane & 1) == 0;
        const bool is_q = n < ep.nq;
        int cc = n - ep.nq;
        bf16* cache = static_cast<bf16*>(ep.kc);
        const bool is_k = !is_q && cc < ep.nkvc;
        if (!is_q && !is_k) { cc -= ep.nkvc; cache = static_cast<bf16*>(ep.vc); }
        const int d = is_q ? n % ep.hd : cc % ep.hd;
        const int head = is_q ? 0 : cc / ep.hd;
        // per group of 16 columns: all positions and RoPE factors first
        // (independent loads), then the rotations and stores
#pragma unroll
        for (int b0 = 0; b0 < BN; b0 += 16) {
            int posv[16];
            float2 cs[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) posv[u] = (b0 + u < nb) ? ep.tok_pos[b0 + u] : -1;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const bool okp = row_ok && posv[u] >= 0 && posv[u] < ep.max_seq && (is_q || is_k);
                cs[u] = okp ? ep.rope[static_cast<long long>(posv[u]) * (ep.hd / 2) + (d >> 1)]
                            : make_float2(1.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int b = b0 + u;
                const float partner = __shfl_xor_sync(0xffffffffu, v[b], 1);
                const int pos = posv[u];
                if (!row_ok || b >= nb || pos < 0 || pos >= ep.max_seq) continue;
                const float re = even ? v[b] : partner, im = even ? partner : v[b];
                const float rot = even ? re * cs[u].x - im * cs[u].y : re * cs[u].y + im * cs[u].x;
                if (is_q) {
                    static_cast<bf16*>(ep.q)[static_cast<long long>(b) * ep.nq + n] = __float2bfloat16_rn(rot);
                } else {
                    const int row = ep.tok_row ? ep.tok_row[b] : b;
                    cache[static_cast<long long>(row) * ep.kv_row_stride +
                          (static_cast<long long>(head) * ep.max_seq + pos) * ep.hd + d] =
                        __float2bfloat16_rn(is_k ? rot : v[b]);
                }
            }
        }
    } else if (ep.mode == EPI_RESID_F32 && nio.ssq_out) {
        // residual add, plus this tile's share of sum(x^2) for the next RMSNorm;
        // the old x values of a 16-column group are loaded together
        const float wn = row_ok ? nio.w_next[n] : 0.f;
        float xo[16];
#pragma unroll
        for (int b = 0; b < BN; ++b) {
            if ((b & 15) == 0) {
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    xo[u] = (row_ok && b + u < nb) ? ep.out[static_cast<long long>(b + u) * ep.ldo + n] : 0.f;
            }
            float sq = 0.f;
            if (row_ok && b < nb) {
                const float nv = xo[b & 15] + v[b];
                ep.out[static_cast<long long>(b) * ep.ldo + n] = nv;
                static_cast<bf16*>(nio.y_out)[static_cast<long long>(b) * ep.ldo + n] = __float2bfloat16_rn(nv * wn);
                sq = nv * nv;
            }
            sq = warp_sum(sq);
            if (lane == 0) red[q * 64 + b] = sq;
        }
        named_sync(2, 128);
        if (epi_tid < nb)
            nio.ssq_out[epi_tid * T + t] = ((red[epi_tid] + red[64 + epi_tid]) + red[128 + epi_tid]) +
                                           red[192 + epi_tid];
        named_sync(2, 128);
    } else if (row_ok) {
        if (ep.mode == EPI_RESID_F32) {
#pragma unroll
            for (int b0 = 0; b0 < BN; b0 += 16) {
                float xo[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    xo[u] = (b0 + u < nb) ? ep.out[static_cast<long long>(b0 + u) * ep.ldo + n] : 0.f;
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

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
linear_decode_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapX,
                     int N, int M, int K, Epi ep, float* __restrict__ part, int* __restrict__ counters, NormIO nio) {
    constexpr int B_BYTES = BN * 128;
    constexpr int STAGE = kABytes + B_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;    // [2]
    uint64_t* tempty = tfull + 2;        // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    int* flag = reinterpret_cast<int*>(tmem_slot + 1);   // [0] abort, [1] fixup broadcast
    float* rs = reinterpret_cast<float*>(flag + 4);      // [64] RMSNorm factors of the token rows
    float* red = rs + 64;                                // [4][64] epilogue sums of squares
    const bool scale_in = nio.ssq_in != nullptr;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, c = blockIdx.x;
    const int T = (N + 127) / 128, KT = (K + 63) / 64;
    const int W = T * KT;
    const int u0 = run_begin(c, W, P), u1 = run_begin(c + 1, W, P);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 128); }
        flag[0] = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapW);
        tma_prefetch_desc(&mapX);
    }
    if (warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger();

    if (warp == 0 && lane == 0) {
        // ---------------- producer: one weight tile + the matching activation
        // tiles per ring slot, walking this CTA's units in order.  Weight
        // tiles of the first slots are requested before the previous kernel
        // has finished; activation tiles only after it has.
        const int nunits = u1 - u0;
        const int npre = nunits < STAGES ? nunits : STAGES;
        int t0 = u0 / KT, k0 = u0 - t0 * KT;          // walk (tile, k) without divisions
        int tt = t0, kk = k0;
        for (int i = 0; i < npre; ++i) {
            mbar_arrive_expect_tx(&full[i], STAGE);
            tma_load_2d(smem + i * STAGE, &mapW, kk * 64, tt * 128, &full[i]);
            if (++kk == KT) { kk = 0; ++tt; }
        }
        pdl_wait();
        tt = t0;
        kk = k0;
        for (int i = 0; i < npre; ++i) {
#pragma unroll
            for (int rr = 0; rr < BN / 16; ++rr)
                tma_load_2d(smem + i * STAGE + kABytes + rr * 2048, &mapX, kk * 64, rr * 16, &full[i]);
            if (++kk == KT) { kk = 0; ++tt; }
        }
        for (int i = npre; i < nunits; ++i) {
            const int s = i % STAGES;
            if (!mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1)) { atomicExch(&flag[0], 1); break; }
            uint8_t* st = smem + s * STAGE;
            mbar_arrive_expect_tx(&full[s], STAGE);
            tma_load_2d(st, &mapW, kk * 64, tt * 128, &full[s]);
#pragma unroll
            for (int rr = 0; rr < BN / 16; ++rr) tma_load_2d(st + kABytes + rr * 2048, &mapX, kk * 64, rr * 16, &full[s]);
            if (++kk == KT) { kk = 0; ++tt; }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        const uint32_t idesc = idesc_bf16_f32(128, BN);
        int u = u0;
        Seg sg;
        int i = 0, j = 0;
        bool abort = false;
        while (!abort && next_seg(u, u1, KT, sg)) {
            const int acc = j & 1;
            if (!mbar_wait(&tempty[acc], ((j >> 1) & 1) ^ 1)) { atomicExch(&flag[0], 1); break; }
            tc_fence_after();
            const uint32_t d = tmem + acc * kAccStride;
            for (int k = sg.ks; k < sg.ke; ++k, ++i) {
                const int s = i % STAGES;
                if (!mbar_wait(&full[s], (i / STAGES) & 1)) { atomicExch(&flag[0], 1); abort = true; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * STAGE);
                const uint32_t b0 = a0 + kABytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_bf16(d, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                                (k > sg.ks || kk > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            tc_commit(&tfull[acc]);
            ++j;
        }
    } else if (warp >= 2) {
        // ---------------- epilogue (warp w reads TMEM lanes 32*(w%4) .. +31)
        pdl_wait();
        const int q = warp & 3;
        const int r = q * 32 + lane;           // row within the 128-row tile
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const int epi_tid = threadIdx.x - 64;    // 0 .. 127
        if (scale_in && epi_tid < M) {
            // RMSNorm factor of token row epi_tid (fused RMSNorm, consumer side)
            float ss = 0.f;
            for (int t2 = 0; t2 < nio.n_in; ++t2) ss += nio.ssq_in[epi_tid * nio.n_in + t2];
            rs[epi_tid] = rsqrtf(ss / static_cast<float>(K) + nio.eps);
        }
        named_sync(1, 128);
        int u = u0;
        Seg sg;
        int j = 0;
        const int nb = M < BN ? M : BN;
        while (next_seg(u, u1, KT, sg)) {
            const int acc = j & 1;
            const bool ok_wait = mbar_wait(&tfull[acc], (j >> 1) & 1);
            tc_fence_after();
            float v[BN];
#pragma unroll
            for (int cc = 0; cc < BN / 16; ++cc)
                tmem_ld_32x32b_x16(tmem + lane_base + acc * kAccStride + cc * 16, v + cc * 16);
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            ++j;
            if (named_any(1, 128, !ok_wait || *reinterpret_cast<volatile int*>(&flag[0]) != 0)) {
                if (epi_tid == 0) report_status(ep.status, LLAMA_ERR_DEVICE_TIMEOUT);
                break;
            }
            const int t = sg.tile;
            const int tb = t * KT;
            const int cf = owner(tb, W, P), cl = owner(tb + KT - 1, W, P);
            if (cl > cf) {
                // split tile: publish this CTA's partial, the last arrival reduces
                const int slot = (tb + sg.ks == u0) ? 0 : 1;   // the run's first segment, or its last
                float* my = part + ((static_cast<long long>(c) * 2 + slot) * 128 + r) * BN;
#pragma unroll
                for (int b = 0; b < BN; b += 4)
                    *reinterpret_cast<float4*>(my + b) = make_float4(v[b], v[b + 1], v[b + 2], v[b + 3]);
                __threadfence();
                named_sync(1, 128);
                if (epi_tid == 0) flag[1] = atomicAdd(&counters[t], 1);
                named_sync(1, 128);
                const int arrived = flag[1];
                if (arrived != cl - cf) continue;      // not the last contributor
                __threadfence();
#pragma unroll
                for (int b = 0; b < BN; ++b) v[b] = 0.f;
                // partials in CTA order, CB contributors per batch of independent loads
                constexpr int CB = BN <= 16 ? 4 : (BN <= 32 ? 2 : 1);
                for (int cb = cf; cb <= cl; cb += CB) {
                    float4 f[CB][BN / 4];
#pragma unroll
                    for (int e = 0; e < CB; ++e) {
                        const int cc = cb + e;
                        if (cc <= cl) {
                            const int sl = run_begin(cc, W, P) >= tb ? 0 : 1;   // slot 0: first segment, 1: last
                            const float4* pp = reinterpret_cast<const float4*>(
                                part + ((static_cast<long long>(cc) * 2 + sl) * 128 + r) * BN);
#pragma unroll
                            for (int qq = 0; qq < BN / 4; ++qq) f[e][qq] = pp[qq];
                        }
                    }
#pragma unroll
                    for (int e = 0; e < CB; ++e) {
                        if (cb + e <= cl) {
#pragma unroll
                            for (int qq = 0; qq < BN / 4; ++qq) {
                                v[4 * qq] += f[e][qq].x;
                                v[4 * qq + 1] += f[e][qq].y;
                                v[4 * qq + 2] += f[e][qq].z;
                                v[4 * qq + 3] += f[e][qq].w;
                            }
                        }
                    }
                }
                if (epi_tid == 0) counters[t] = 0;
            }
            finish_tile<BN>(v, t, r, lane, q, epi_tid, nb, N, T, ep, nio, scale_in, rs, red);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}


// ---------------------------------------------------------------- host side
static int g_sms = 0;

template <int BN, int STAGES>
static int launch_decode(const CUtensorMap& w, const CUtensorMap& x, int N, int M, int K, const Epi& ep,
                         float* part, int* counters, int max_ctas, cudaStream_t st, bool pdl, const NormIO& nio) {
    constexpr int smem = 1024 + STAGES * (kABytes + BN * 128) + (2 * STAGES + 4) * 8 + 32 + 5 * 64 * 4;
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    auto kern = linear_decode_kernel<BN, STAGES>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(linear_decode_kernel)");
        attr = true;
    }
    const long long units = static_cast<long long>((N + 127) / 128) * ((K + 63) / 64);
    if (units > (1 << 22)) { set_error("decode projection too large (%lld work units)", units); return LLAMA_ERR_INVALID_ARG; }
    int P = max_ctas;
    if (units < P) P = static_cast<int>(units);
    cudaError_t e = launch_k(kern, dim3(P), dim3(kThreads), smem, st, pdl, w, x, N, M, K, ep, part, counters, nio);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "linear_decode_kernel");
    return LLAMA_OK;
}

int linear_bf16_decode(const TmaMaps* mapX, const TmaMaps* mapW, int M, int N, int K, const Epi& ep, float* part,
                       size_t part_bytes, int* counters, cudaStream_t st, bool pdl, const NormIO* nio_in) {
    if (M <= 0 || N <= 0) return LLAMA_OK;
    NormIO nio = {};
    if (nio_in) nio = *nio_in;
    if (nio.ssq_out && (N % 128 || !nio.y_out || !nio.w_next || ep.mode != EPI_RESID_F32)) {
        set_error("fused RMSNorm producer needs a residual epilogue, N %% 128 == 0, y_out and w_next");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (M > 64) { set_error("decode projection takes at most 64 token rows"); return LLAMA_ERR_INVALID_ARG; }
    {
        // split partials: two 128 x BN fp32 blocks per persistent CTA
        const int bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 48 ? 48 : 64;
        const size_t need = static_cast<size_t>(kMaxDecodeCtas) * 2 * 128 * bn * 4;
        if (!part || !counters || part_bytes < need) {
            set_error("decode projection needs %zu bytes of split partials and the tile counters", need);
            return LLAMA_ERR_CAPACITY;
        }
    }
    if (g_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_sms <= 0) g_sms = 148;
        if (g_sms > kMaxDecodeCtas) g_sms = kMaxDecodeCtas;
    }
    if (M <= 16) return launch_decode<16, 12>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
    if (M <= 32) return launch_decode<32, 11>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
    if (M <= 48) return launch_decode<48, 10>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
    return launch_decode<64, 9>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
}

}  // namespace llb
