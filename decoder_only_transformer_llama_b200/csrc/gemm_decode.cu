// Decode-shaped 16-bit (bf16 or fp16) projections (few token rows) on tcgen05: a persistent,
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
// writes the next projection's operand, x * w_next rounded to the model's 16-bit
// type, and per-tile sums of
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
#include "decode_tile.cuh"

namespace llb {

namespace {
constexpr int kThreads = 192;
constexpr int kAccStride = 64;      // TMEM columns per accumulator buffer
constexpr int kTmemCols = 128;      // two accumulator buffers
constexpr int kMinUnitsPerCta = 4;   // 64 KB of weights
constexpr int kMaxSplit = 8;         // CTAs sharing one weight tile, at most
}  // namespace

template <int BN, int STAGES, typename E>
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
    uint64_t* mdone = tempty + 2;        // the MMA issuer's last commit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
    int* flag = reinterpret_cast<int*>(tmem_slot + 1);   // [0] abort, [1] fixup broadcast
    float* rs = reinterpret_cast<float*>(flag + 4);      // [64] RMSNorm factors of the token rows
    float* red = rs + 64;                                // [4][64] epilogue sums of squares
    const bool scale_in = nio.ssq_in != nullptr;
    const uint64_t wlim = ep.wait_ns > 0 ? static_cast<uint64_t>(ep.wait_ns) : kWaitLimitNs;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, c = blockIdx.x;
    const int T = (N + 127) / 128, KT = (K + 63) / 64;
    const int W = T * KT;
    const int u0 = run_begin(c, W, P), u1 = run_begin(c + 1, W, P);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 128); }
        mbar_init(mdone, 1);
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

    int issued = 0, stall = -1;   // producer: ring stages [0, issued) were issued, all but `stall`
    if (warp == 0 && lane == 0) {
        // ---------------- producer: one weight tile + the matching activation
        // tiles per ring slot, walking this CTA's units in order.  Weight
        // tiles of the first slots are requested before the previous kernel
        // has finished; activation tiles only after it has.
        const int nunits = u1 - u0;
        const int npre = nunits < STAGES ? nunits : STAGES;
        stall = c == 0 ? ep.stall - 1 : -1;   // tests of the timeout path only
        const uint64_t pol_w = l2_policy_evict_first();   // weights are read once per step
        int t0 = u0 / KT, k0 = u0 - t0 * KT;          // walk (tile, k) without divisions
        int tt = t0, kk = k0;
        for (int i = 0; i < npre; ++i) {
            if (i != stall) {
                mbar_arrive_expect_tx(&full[i], STAGE);
                tma_load_2d_hint(smem + i * STAGE, &mapW, kk * 64, tt * 128, &full[i], pol_w);
            }
            if (++kk == KT) { kk = 0; ++tt; }
        }
        pdl_wait();
        tt = t0;
        kk = k0;
        for (int i = 0; i < npre; ++i) {
            if (i != stall) {
#pragma unroll
                for (int rr = 0; rr < BN / 16; ++rr)
                    tma_load_2d(smem + i * STAGE + kABytes + rr * 2048, &mapX, kk * 64, rr * 16, &full[i]);
            }
            if (++kk == KT) { kk = 0; ++tt; }
        }
        issued = npre;
        for (int i = npre; i < nunits; ++i) {
            const int s = i % STAGES;
            if (!mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, wlim)) { atomicExch(&flag[0], 1); break; }
            if (i != stall) {
                uint8_t* st = smem + s * STAGE;
                mbar_arrive_expect_tx(&full[s], STAGE);
                tma_load_2d_hint(st, &mapW, kk * 64, tt * 128, &full[s], pol_w);
#pragma unroll
                for (int rr = 0; rr < BN / 16; ++rr)
                    tma_load_2d(st + kABytes + rr * 2048, &mapX, kk * 64, rr * 16, &full[s]);
            }
            issued = i + 1;
            if (++kk == KT) { kk = 0; ++tt; }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        const uint32_t idesc = idesc_16_f32<E>(128, BN);
        int u = u0;
        Seg sg;
        int i = 0, j = 0;
        bool abort = false;
        while (!abort && next_seg(u, u1, KT, sg)) {
            const int acc = j & 1;
            if (!mbar_wait(&tempty[acc], ((j >> 1) & 1) ^ 1, wlim)) { atomicExch(&flag[0], 1); break; }
            tc_fence_after();
            const uint32_t d = tmem + acc * kAccStride;
            for (int k = sg.ks; k < sg.ke; ++k, ++i) {
                const int s = i % STAGES;
                if (!mbar_wait(&full[s], (i / STAGES) & 1, wlim)) { atomicExch(&flag[0], 1); abort = true; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * STAGE);
                const uint32_t b0 = a0 + kABytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_16(d, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                                (k > sg.ks || kk > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            tc_commit(&tfull[acc]);
            ++j;
        }
        // every MMA issued here has finished before TMEM is freed (on a normal
        // run the epilogue has already waited for them)
        tc_commit(mdone);
        if (!mbar_wait(mdone, 0, wlim)) atomicExch(&flag[0], 1);
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
            ss = row_ssq(nio.ssq_in + epi_tid * nio.n_in, nio.n_in);
            rs[epi_tid] = rsqrtf(ss / static_cast<float>(K) + nio.eps);
        }
        named_sync(1, 128);
        decode_epilogue_loop<BN, E>(tmem + lane_base, tfull, tempty, flag, part, counters, c, P, u0, u1, KT, N, M, ep,
                                 nio, scale_in, rs, red, r, lane, q, epi_tid, wlim);
        if (ep.mode == EPI_LOGITS_ARGMAX) __threadfence();   // this CTA's keys before its finish count
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (warp == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&flag[0]) != 0) {
        // the CTA gave up: the copies it still has in flight land before it
        // exits (the newest stage of each ring slot; a skipped one is not waited for)
        for (int s = 0; s < STAGES; ++s) {
            if (issued <= s) continue;
            int j = s + ((issued - 1 - s) / STAGES) * STAGES;
            if (j == stall) j -= STAGES;
            if (j >= 0) mbar_wait(&full[s], (j / STAGES) & 1, wlim);
        }
    }
    if (ep.mode == EPI_LOGITS_ARGMAX && ep.done && warp == 0) {
        // greedy pick: the CTA that finishes last reads every row's key
        int last = 0;
        if (lane == 0) last = atomicAdd(ep.done, 1) == static_cast<int>(gridDim.x) - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
            __threadfence();
            for (int b = lane; b < M; b += 32) {
                const int id = argmax_key_id(atomicExch(&ep.best[b], 0ull));
                if (ep.next) ep.next[b] = id;
                if (ep.tok_adv) ep.tok_adv[b] = id;
                if (ep.pos_adv) ep.pos_adv[b] += 1;
            }
            if (lane == 0) atomicExch(ep.done, 0);
        }
    }
    if (threadIdx.x == 0) tl_stamp(ep.tl);
}


// ---------------------------------------------------------------- host side
static int g_sms = 0;

template <int BN, int STAGES, typename E>
static int launch_decode(const CUtensorMap& w, const CUtensorMap& x, int N, int M, int K, const Epi& ep,
                         float* part, int* counters, int max_ctas, cudaStream_t st, bool pdl, const NormIO& nio) {
    constexpr int smem = 1024 + STAGES * (kABytes + BN * 128) + (2 * STAGES + 5) * 8 + 32 + 5 * 64 * 4;
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    auto kern = linear_decode_kernel<BN, STAGES, E>;
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
    // at least kMinUnitsPerCta units per CTA and at most kMaxSplit CTAs per
    // weight tile: a small projection spread over every SM would split each
    // tile among dozens of CTAs, and its finisher would add as many partials
    int P = max_ctas;
    const long long p_units = (units + kMinUnitsPerCta - 1) / kMinUnitsPerCta;
    const long long p_tiles = static_cast<long long>(kMaxSplit) * ((N + 127) / 128);
    if (p_units < P) P = static_cast<int>(p_units);
    if (p_tiles < P) P = static_cast<int>(p_tiles);
    cudaError_t e = launch_k(kern, dim3(P), dim3(kThreads), smem, st, pdl, w, x, N, M, K, ep, part, counters, nio);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "linear_decode_kernel");
    return LLAMA_OK;
}

// Token-row count -> MMA width (BN) and ring depth.
template <typename E>
static int decode_by_rows(const TmaMaps* mapX, const TmaMaps* mapW, int M, int N, int K, const Epi& ep, float* part,
                          int* counters, cudaStream_t st, bool pdl, const NormIO& nio) {
    if (M <= 16) return launch_decode<16, 12, E>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
    if (M <= 32) return launch_decode<32, 11, E>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
    if (M <= 48) return launch_decode<48, 10, E>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
    return launch_decode<64, 9, E>(mapW->a128, mapX->b, N, M, K, ep, part, counters, g_sms, st, pdl, nio);
}

int linear16_decode(const TmaMaps* mapX, const TmaMaps* mapW, int M, int N, int K, int dtype, const Epi& ep, float* part,
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
    if (dtype == LLAMA_F16) return decode_by_rows<f16>(mapX, mapW, M, N, K, ep, part, counters, st, pdl, nio);
    if (dtype == LLAMA_BF16) return decode_by_rows<bf16>(mapX, mapW, M, N, K, ep, part, counters, st, pdl, nio);
    set_error("16-bit projection: dtype must be LLAMA_BF16 or LLAMA_F16");
    return LLAMA_ERR_INVALID_ARG;
}

}  // namespace llb
