// Causal grouped-query attention over the KV cache (Admin Guide §8.4,
// Attention steps 5-7 and the mask NOTE; repeat_kv from the source tour):
//   o_h = softmax_j( q_h . K[j][h / n_rep] / sqrt(hd) ) V[j][h / n_rep],
//   keys j = 0 .. position of the query (the cached prefix plus the causal part
//   of this call's tokens).  The -inf mask is realised as a key-range bound.
//
// Decode (one query per row): split-KV.  Each KV head is read once for its
// whole query group; split partials are merged by the last split to finish.
//
// Prefill of fp32 models: one CTA per (64-query tile, head, row), online
// softmax over 64-key tiles staged in shared memory (fp32 CUDA-core
// arithmetic).  16-bit models use the tensor-core kernel of attention_prefill_tc.cu.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "model.h"

namespace llb {

// ---------------------------------------------------------------- vector loads
template <typename T, int N> struct Vec;
template <> struct Vec<float, 1> { static __device__ __forceinline__ void load(const float* p, float* o) { o[0] = p[0]; } };
template <> struct Vec<float, 2> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        const float2 v = *reinterpret_cast<const float2*>(p); o[0] = v.x; o[1] = v.y;
    }
};
template <> struct Vec<float, 4> {
    static __device__ __forceinline__ void load(const float* p, float* o) {
        const float4 v = *reinterpret_cast<const float4*>(p); o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
template <> struct Vec<bf16, 1> { static __device__ __forceinline__ void load(const bf16* p, float* o) { o[0] = __bfloat162float(p[0]); } };
template <> struct Vec<bf16, 2> {
    static __device__ __forceinline__ void load(const bf16* p, float* o) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p)); o[0] = f.x; o[1] = f.y;
    }
};
template <> struct Vec<bf16, 4> {
    static __device__ __forceinline__ void load(const bf16* p, float* o) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    }
};
template <> struct Vec<f16, 1> { static __device__ __forceinline__ void load(const f16* p, float* o) { o[0] = __half2float(p[0]); } };
template <> struct Vec<f16, 2> {
    static __device__ __forceinline__ void load(const f16* p, float* o) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(p)); o[0] = f.x; o[1] = f.y;
    }
};
template <> struct Vec<f16, 4> {
    static __device__ __forceinline__ void load(const f16* p, float* o) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    }
};

// ---------------------------------------------------------------- decode
// Flash-decoding over the cache as one persistent, balanced pass.  The work
// is a flat list of units, one unit = 64 consecutive key positions of one
// (row b, KV head g) pair, pairs in (b, g) order; pair (b, g) has
// ceil((pos[b] + 1) / 64) units.  Each of the P CTAs (as many as fit on the
// GPU at once) takes an equal contiguous run of the list, so every CTA reads
// the same number of cache bytes whatever the mix of context lengths, and all
// CTAs run in one wave.  A run is cut into segments at pair boundaries.
//
// Each unit's K and V blocks are contiguous in the cache (the positions of one
// head are adjacent) and are fetched by bulk async copies into a three-deep
// shared-memory ring that runs across segments.  Warp w scores keys
// 16w .. 16w+15 of a unit, eight at a time, for all n_rep query heads of the
// group; lane l holds head dims [l*EPL, (l+1)*EPL) and the eight partial dot
// products are summed across the warp by a transposing butterfly (one full
// sum per lane, then broadcast).  Online softmax state (max, sum, o) is kept
// per warp and merged across the 4 warps at the end of a segment.
//
// A segment that covers its whole pair writes the output row directly.  A pair
// split between CTAs is finished by its first contributor, whose segment is
// the last of its run; every other contributor's segment is the first of its
// run: it writes its unnormalised (o, max, sum) and counts it at the pair's
// counter early in its run, and the finisher, at the end of its run, waits
// (bounded) for that count, then merges its own state with the published
// ones in CTA order (deterministic).  Only a finisher waits, and only for
// other CTAs' first segments, which never wait.
// Fewest cache units (64-key blocks) a CTA's run holds when there are fewer
// than that many per CTA of the grid: short runs split every pair across many
// CTAs, and each split adds a merge to the pair's finisher.
constexpr int kMinUnitsPerCta = 2;
__device__ __forceinline__ int attn_ctas(long long W, int grid) {
    const long long p = (W + kMinUnitsPerCta - 1) / kMinUnitsPerCta;
    return static_cast<int>(p < grid ? p : grid);
}

__device__ __forceinline__ long long run_begin64(long long c, long long W, long long P) { return c * W / P; }
__device__ __forceinline__ int owner64(long long u, long long W, long long P) {
    return static_cast<int>(((u + 1) * P - 1) / W);
}

// ---------------------------------------------------------------- decode units on the tensor cores
// (mma.sync m16n8k16, bf16 or fp16 in, fp32 accumulate: a decode unit is a
// 16-row problem, too small for tcgen05's 128-row tiles)
namespace {
__device__ __forceinline__ void dec_ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void dec_ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// c += A B with A rows 8..15 zero (a1 = a3 = 0).
template <typename T>
__device__ __forceinline__ void dec_mma(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    if constexpr (std::is_same<T, bf16>::value) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
    }
}
// Shared-memory address of key `key`, dims d..d+7 of a 64-key block stored as
// two 128-byte-swizzled TMA boxes (dims 0-63, then 64-127; 8 KB each).
__device__ __forceinline__ uint32_t dec_swz(uint32_t base, int key, int d) {
    return base + static_cast<uint32_t>((d >> 6) * 8192 + key * 128 + ((((d & 63) >> 3) ^ (key & 7)) << 4));
}
}  // namespace

// Ring slots (64-key K+V units) per decode-attention CTA (six for one CTA per
// SM measured the same as three on the 70B-shaped slice).
constexpr int kDecodeSlots = 3;

// One 64-key unit for warp `warp` (keys 16*warp .. 16*warp+15 of it, n valid):
// S = Q K^T for the group's query heads, online softmax per head (m, l), and
// O += P V, all as m16n8k16 fragments; lane (g = lane/4, t = lane%4) holds
// head g's scores of keys 8nt + 2t, +1 and O columns 8nd + 2t, +1.
template <typename T, int NREP>
__device__ __forceinline__ void tc_unit(const T* sK, const T* sV, int warp, int lane, int n, float scale,
                                        const uint32_t (&qa)[8][2], float& m_run, float& l_run,
                                        float (&oacc)[16][4]) {
    const int mi = lane >> 3, rr = lane & 7, t = lane & 3;
    const uint32_t kb = smem_u32(sK), vb = smem_u32(sV);
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        // matrices: keys 0-7 / dims 0-7, keys 0-7 / dims 8-15, keys 8-15 / dims 0-7, keys 8-15 / dims 8-15
        uint32_t b00, b01, b10, b11;
        dec_ldsm_x4(dec_swz(kb, 16 * warp + ((mi >> 1) << 3) + rr, 16 * ks + ((mi & 1) << 3)), b00, b01, b10, b11);
        dec_mma<T>(sc[0], qa[ks][0], qa[ks][1], b00, b01);
        dec_mma<T>(sc[1], qa[ks][0], qa[ks][1], b10, b11);
    }
    float s4[4] = {sc[0][0] * scale, sc[0][1] * scale, sc[1][0] * scale, sc[1][1] * scale};
    const int k0 = 16 * warp + 2 * t;
    if (k0 >= n) s4[0] = -INFINITY;
    if (k0 + 1 >= n) s4[1] = -INFINITY;
    if (k0 + 8 >= n) s4[2] = -INFINITY;
    if (k0 + 9 >= n) s4[3] = -INFINITY;
    float mx = fmaxf(fmaxf(s4[0], s4[1]), fmaxf(s4[2], s4[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mnew = fmaxf(m_run, mx);          // finite: key 16*warp is valid
    const float corr = __expf(m_run - mnew);      // 0 while m_run is -inf
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = __expf(s4[e] - mnew);
    float rs = (p[0] + p[1]) + (p[2] + p[3]);
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l_run = l_run * corr + rs;
    m_run = mnew;
    const uint32_t pa0 = pack2<T>(p[0], p[1]), pa2 = pack2<T>(p[2], p[3]);
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
        oacc[nd][0] *= corr;
        oacc[nd][1] *= corr;
    }
#pragma unroll
    for (int np = 0; np < 8; ++np) {
        // transposed: keys 0-7 / dims 16np.., keys 8-15 / dims 16np.., keys 0-7 / dims 16np+8.., keys 8-15 / dims 16np+8..
        uint32_t v00, v01, v10, v11;
        dec_ldsm_x4_t(dec_swz(vb, 16 * warp + ((mi & 1) << 3) + rr, 16 * np + ((mi >> 1) << 3)), v00, v01, v10, v11);
        dec_mma<T>(oacc[2 * np], pa0, pa2, v00, v01);
        dec_mma<T>(oacc[2 * np + 1], pa0, pa2, v10, v11);
    }
}

template <typename T, int HD, int NREP, bool TC>
__global__ void __launch_bounds__(128)
attn_decode_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                   const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                   long long row_base, const int32_t* __restrict__ pos, int B, int nkv, int nq, int S,
                   long long row_stride, float* __restrict__ part_o, float* __restrict__ part_ml,
                   int* __restrict__ counters, T* __restrict__ out, int* status, unsigned long long* tl,
                   long long wait_ns, int stall) {
    constexpr int EPL = HD / 32;   // head dims per lane
    constexpr int ROW = HD * static_cast<int>(sizeof(T));
    constexpr int CH_BYTES = kChunk * ROW;
    constexpr int NSLOT = kDecodeSlots;
    static_assert(!TC || (HD == 128 && sizeof(T) == 2), "tensor-core units: 16-bit cache, head_dim 128");
    extern __shared__ __align__(128) uint8_t dsm_raw[];
    // ring slots 1024-byte aligned (128-byte swizzled TMA boxes on the tensor-core path)
    uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar[NSLOT];
    __shared__ float s_m[4][NREP], s_l[4][NREP];
    __shared__ float s_o[4][NREP][HD];
    __shared__ int s_cum[kMaxRows + 1];   // units before row b, in units of one pair's chunks
    __shared__ int s_nch[kMaxRows];       // chunks of each pair of row b (0: row skipped)
    __shared__ int s_pos[kMaxRows];       // position of row b's query
    __shared__ int s_wsum[4];
    __shared__ int s_last;
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- chunks per row and their prefix sums (rows in order, 2 per thread)
    int my_pos[2] = {-1, -1};
    auto make_plan = [&]() {
        int v[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int b = 2 * threadIdx.x + e;
            int n = 0;
            if (b < B) {
                const int p = __ldcg(pos + b);   // L2: read again after the grid dependency resolves
                my_pos[e] = p;
                if (p >= 0 && p < S) n = (p + kChunk) / kChunk;
                s_nch[b] = n;
                s_pos[b] = p;
            }
            v[e] = n;
        }
        const int t = v[0] + v[1];
        int incl = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int before = incl - t;
        for (int w = 0; w < warp; ++w) before += s_wsum[w];
        const int b0 = 2 * threadIdx.x;
        if (threadIdx.x == 0) s_cum[0] = 0;
        if (b0 + 1 <= B) s_cum[b0 + 1] = before + v[0];
        if (b0 + 2 <= B) s_cum[b0 + 2] = before + t;
        __syncthreads();
    };
    // cursor over (row, kv head, chunk) starting at unit u
    struct Cur { int b, g, j; };
    auto cur_at = [&](long long u) {
        int lo = 0, hi = B - 1;                  // largest b with s_cum[b] * nkv <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (static_cast<long long>(s_cum[mid]) * nkv <= u) lo = mid; else hi = mid - 1;
        }
        Cur r;
        r.b = lo;
        const long long rem = u - static_cast<long long>(s_cum[lo]) * nkv;
        r.g = static_cast<int>(rem / s_nch[lo]);
        r.j = static_cast<int>(rem - static_cast<long long>(r.g) * s_nch[lo]);
        return r;
    };
    auto advance = [&](Cur& r) {
        if (++r.j < s_nch[r.b]) return;
        r.j = 0;
        if (++r.g < nkv) return;
        r.g = 0;
        do { ++r.b; } while (r.b < B && s_nch[r.b] == 0);
    };
    auto head_off = [&](const Cur& r) {
        return static_cast<long long>(r.b) * row_stride + static_cast<long long>(r.g) * S * HD;
    };
    const uint64_t wlim = wait_ns > 0 ? static_cast<uint64_t>(wait_ns) : kWaitLimitNs;
    const int stall_i = blockIdx.x == 0 ? stall : -1;   // tests of the timeout path only
    Cur icur = {0, 0, 0};                        // issue cursor (thread 0)
    const uint64_t pol_kv = l2_policy_evict_first();   // read once per step
    auto issue = [&](int i) {                    // i-th unit of this run into ring slot i % NSLOT
        const int ctx = s_pos[icur.b] + 1;
        const int j0 = icur.j * kChunk;
        const int n = min(kChunk, ctx - j0);
        uint8_t* slot = dsm + (i % NSLOT) * 2 * CH_BYTES;
        const long long ho = head_off(icur);
        if (i != stall_i) {
            if constexpr (TC) {
                // four 64-key x 64-dim boxes (K and V, dims 0-63 and 64-127), whole
                // boxes even past the valid keys (masked in the scores)
                const int row = static_cast<int>(row_base + (static_cast<long long>(icur.b) * nkv + icur.g) * S + j0);
                mbar_arrive_expect_tx(&bar[i % NSLOT], 2u * CH_BYTES);
                tma_load_2d_hint(slot, &mapK, 0, row, &bar[i % NSLOT], pol_kv);
                tma_load_2d_hint(slot + CH_BYTES / 2, &mapK, 64, row, &bar[i % NSLOT], pol_kv);
                tma_load_2d_hint(slot + CH_BYTES, &mapV, 0, row, &bar[i % NSLOT], pol_kv);
                tma_load_2d_hint(slot + CH_BYTES + CH_BYTES / 2, &mapV, 64, row, &bar[i % NSLOT], pol_kv);
            } else {
                mbar_arrive_expect_tx(&bar[i % NSLOT], 2u * n * ROW);
                bulk_load_hint(slot, kc + ho + static_cast<long long>(j0) * HD, n * ROW, &bar[i % NSLOT], pol_kv);
                bulk_load_hint(slot + CH_BYTES, vc + ho + static_cast<long long>(j0) * HD, n * ROW, &bar[i % NSLOT],
                               pol_kv);
            }
        }
        advance(icur);
    };

    if (threadIdx.x == 0) {
        for (int k = 0; k < NSLOT; ++k) mbar_init(&bar[k], 1);
        fence_mbar_init();
    }
    // Before the previous kernel (which writes this step's K/V row and q) has
    // finished: plan with the positions as they read now, and start the
    // copies of this CTA's first units whose keys all lie before their row's
    // new position.  Those cache entries are final: positions that already
    // read as this step's were advanced by a kernel that ran after every
    // earlier kernel had completed (each kernel of the chain waits for its
    // predecessor before it writes), and the copies of the units holding a
    // new position start only after the grid dependency.  After it has
    // resolved, the positions are read again; if any changed, the early
    // copies are drained, the ring re-armed and the plan redone.
    make_plan();
    int n_early = 0;                             // thread 0: units issued before the dependency
    {
        const long long W0 = static_cast<long long>(s_cum[B]) * nkv;
        const int P0 = attn_ctas(W0, gridDim.x);
        if (threadIdx.x == 0 && blockIdx.x < P0) {
            const long long v0 = run_begin64(blockIdx.x, W0, P0), v1 = run_begin64(blockIdx.x + 1, W0, P0);
            icur = cur_at(v0);
            while (n_early < NSLOT && v0 + n_early < v1) {
                const int j0 = icur.j * kChunk;
                if (j0 + kChunk > s_pos[icur.b]) break;   // holds the new position: wait for its writer
                issue(n_early++);
            }
        }
    }
    pdl_wait();
    {
        bool changed = false;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int b = 2 * threadIdx.x + e;
            if (b < B) {
                const int p = __ldcg(pos + b);
                changed |= p != my_pos[e];
                if ((p < 0 || p >= S) && blockIdx.x == 0) report_status(status, LLAMA_ERR_CAPACITY);
            }
        }
        if (__syncthreads_or(changed)) {
            if (threadIdx.x == 0) {
                for (int k = 0; k < n_early; ++k)
                    if (k != stall_i) mbar_wait(&bar[k], 0, wlim);
                for (int k = 0; k < NSLOT; ++k) {
                    mbar_inval(&bar[k]);
                    mbar_init(&bar[k], 1);
                }
                fence_mbar_init();
                n_early = 0;
            }
            make_plan();
        }
    }
    const long long W = static_cast<long long>(s_cum[B]) * nkv;
    const int P = attn_ctas(W, gridDim.x), c = blockIdx.x;
    if (c >= P) {
        if (threadIdx.x == 0) tl_stamp(tl);
        return;
    }
    const long long u0 = run_begin64(c, W, P), u1 = run_begin64(c + 1, W, P);
    const int len = static_cast<int>(u1 - u0);
    if (threadIdx.x == 0) {
        if (n_early == 0) icur = cur_at(u0);
        for (int k = n_early; k < NSLOT && k < len; ++k) issue(k);
    }
    const float scale = rsqrtf(static_cast<float>(HD));
    Cur cur = cur_at(u0);
    float qv[NREP][EPL];
    float mx[NREP], sl[NREP], o[NREP][EPL];
    // tensor-core path (TC): per warp, rows g = lane / 4 of the m16n8k16
    // fragments are the group's query heads (rows >= NREP stay zero)
    const int tg = lane >> 2, tt = lane & 3;
    uint32_t qa[TC ? 8 : 1][2];          // Q A-fragments per 16-dim step: dims 2tt.., 2tt+8..
    float m_run = -INFINITY, l_run = 0.f;
    float oacc[TC ? 16 : 1][4];          // O rows tg (and tg+8, unused), dims 8nd + 2tt, +1
    auto start_pair = [&]() {
        if constexpr (TC) {
            const T* qrow = q + static_cast<long long>(cur.b) * nq + (cur.g * NREP + tg) * HD;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qa[ks][0] = tg < NREP ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tt) : 0u;
                qa[ks][1] = tg < NREP ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tt + 8) : 0u;
            }
            m_run = -INFINITY;
            l_run = 0.f;
#pragma unroll
            for (int nd = 0; nd < 16; ++nd)
#pragma unroll
                for (int e = 0; e < 4; ++e) oacc[nd][e] = 0.f;
            return;
        }
#pragma unroll
        for (int r = 0; r < NREP; ++r) {
            Vec<T, EPL>::load(q + static_cast<long long>(cur.b) * nq + (cur.g * NREP + r) * HD + lane * EPL, qv[r]);
#pragma unroll
            for (int e = 0; e < EPL; ++e) qv[r][e] *= scale;
            mx[r] = -INFINITY;
            sl[r] = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[r][e] = 0.f;
        }
    };
    start_pair();
    __syncthreads();   // barriers initialised
    bool ok = true;
    int fail_i = 0;
    int seg_j0 = cur.j, seg_i0 = 0;
    for (int i = 0; i < len; ++i) {
        // every thread of the CTA takes the same branch, even if the wait ran
        // out at slightly different times in different threads
        ok = __syncthreads_and(mbar_wait(&bar[i % NSLOT], (i / NSLOT) & 1, wlim));
        if (!ok) { fail_i = i; break; }
        const T* sK = reinterpret_cast<const T*>(dsm + (i % NSLOT) * 2 * CH_BYTES);
        const T* sV = reinterpret_cast<const T*>(dsm + (i % NSLOT) * 2 * CH_BYTES + CH_BYTES);
        const int ctx = s_pos[cur.b] + 1;
        const int n = min(kChunk, ctx - cur.j * kChunk);
        if constexpr (TC) {
            if (16 * warp < n) tc_unit<T, NREP>(sK, sV, warp, lane, n, scale, qa, m_run, l_run, oacc);
        } else {
#pragma unroll 1
        for (int jb = warp * 16; jb < min(n, warp * 16 + 16); jb += 8) {
            // eight keys: this lane's partial dot products ...
            float kv[8][EPL];
#pragma unroll
            for (int u = 0; u < 8; ++u) Vec<T, EPL>::load(sK + min(jb + u, n - 1) * HD + lane * EPL, kv[u]);
#pragma unroll
            for (int r = 0; r < NREP; ++r) {
                float d[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    d[u] = 0.f;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) d[u] = fmaf(qv[r][e], kv[u][e], d[u]);
                }
                // ... summed by a transposing butterfly: after it, lane l holds the
                // full dot of key 4*b4 + 2*b3 + b2 (b4, b3, b2 = bits 4, 3, 2 of l)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const bool hi = lane & 16;
                    const float send = hi ? d[u] : d[u + 4];
                    d[u] = (hi ? d[u + 4] : d[u]) + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const bool hi = lane & 8;
                    const float send = hi ? d[u] : d[u + 2];
                    d[u] = (hi ? d[u + 2] : d[u]) + __shfl_xor_sync(0xffffffffu, send, 8);
                }
                {
                    const bool hi = lane & 4;
                    const float send = hi ? d[0] : d[1];
                    d[0] = (hi ? d[1] : d[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                d[0] += __shfl_xor_sync(0xffffffffu, d[0], 2);
                d[0] += __shfl_xor_sync(0xffffffffu, d[0], 1);
                float sc[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    sc[u] = __shfl_sync(0xffffffffu, d[0], ((u >> 2) << 4) | (((u >> 1) & 1) << 3) | ((u & 1) << 2));
                    if (jb + u >= n) sc[u] = -INFINITY;
                }
                float mnew = mx[r];
#pragma unroll
                for (int u = 0; u < 8; ++u) mnew = fmaxf(mnew, sc[u]);
                const float corr = __expf(mx[r] - mnew);
                float pj[8], ps = 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) { pj[u] = __expf(sc[u] - mnew); ps += pj[u]; }
                sl[r] = sl[r] * corr + ps;
#pragma unroll
                for (int e = 0; e < EPL; ++e) o[r][e] *= corr;
                mx[r] = mnew;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float vv[EPL];
                    Vec<T, EPL>::load(sV + min(jb + u, n - 1) * HD + lane * EPL, vv);
#pragma unroll
                    for (int e = 0; e < EPL; ++e) o[r][e] = fmaf(pj[u], vv[e], o[r][e]);
                }
            }
        }
        }
        __syncthreads();                               // ring slot i % NSLOT is free again
        if (threadIdx.x == 0 && i + NSLOT < len) issue(i + NSLOT);
        const int nch = s_nch[cur.b];
        if (cur.j + 1 < nch && i + 1 < len) { advance(cur); continue; }

        // ---- end of a segment: merge the 4 warps, then write the row or a partial
        const bool whole = seg_j0 == 0 && cur.j + 1 == nch;
        if constexpr (TC) {
            if (tg < NREP) {
                if (tt == 0) { s_m[warp][tg] = m_run; s_l[warp][tg] = l_run; }
#pragma unroll
                for (int nd = 0; nd < 16; ++nd) {
                    s_o[warp][tg][8 * nd + 2 * tt] = oacc[nd][0];
                    s_o[warp][tg][8 * nd + 2 * tt + 1] = oacc[nd][1];
                }
            }
        } else {
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < NREP; ++r) { s_m[warp][r] = mx[r]; s_l[warp][r] = sl[r]; }
            }
#pragma unroll
            for (int r = 0; r < NREP; ++r)
#pragma unroll
                for (int e = 0; e < EPL; ++e) s_o[warp][r][lane * EPL + e] = o[r][e];
        }
        __syncthreads();
        const long long pair_u0 = static_cast<long long>(s_cum[cur.b]) * nkv + static_cast<long long>(cur.g) * nch;
        const int slot_id = c * 2 + (seg_i0 == 0 ? 0 : 1);
        // A pair split between runs is finished by its first contributor cf:
        // that segment is the last of cf's run (its run ends inside the pair),
        // while every other contributor's run starts inside the pair, so its
        // segment is the first of its run and is published early.
        const int cf = whole ? c : owner64(pair_u0, W, P), cl = whole ? c : owner64(pair_u0 + nch - 1, W, P);
        const bool finisher = !whole && c == cf;
        const int cnt_idx = cur.b * nkv + cur.g;
        if (finisher) {
            if (threadIdx.x == 0) {
                const int need = cl - cf;
                const volatile int* cnt = counters + cnt_idx;
                bool okc = *cnt >= need;
                if (!okc) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!(okc = *cnt >= need) && globaltimer_ns() - t0 <= wlim) {
                    }
                }
                s_last = okc ? 1 : 0;
            }
            __syncthreads();
            if (!s_last) {       // units up to i were consumed; i + 1 .. i + NSLOT may be in flight
                ok = false;
                fail_i = i + 1;
                break;
            }
            __threadfence();
        }
        for (int idx = threadIdx.x; idx < NREP * HD; idx += blockDim.x) {
            const int r = idx / HD, d = idx % HD;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w][r]);
            float L = 0.f, acc = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float f = (s_m[w][r] == -INFINITY) ? 0.f : __expf(s_m[w][r] - M);
                L += s_l[w][r] * f;
                acc += s_o[w][r][d] * f;
            }
            const int h = cur.g * NREP + r;
            if (whole) {
                out[static_cast<long long>(cur.b) * nq + h * HD + d] = from_f32<T>(acc / L);
            } else if (!finisher) {
                part_o[(static_cast<long long>(slot_id) * NREP + r) * HD + d] = acc;
                if (d == 0) {
                    part_ml[(static_cast<long long>(slot_id) * NREP + r) * 2] = M;
                    part_ml[(static_cast<long long>(slot_id) * NREP + r) * 2 + 1] = L;
                }
            } else {
                // merge this CTA's (M, L, acc) with the published ones, in CTA
                // order.  Every other contributor published its first segment
                // (slot 0).  Up to kMergeBatch contributors' values are loaded
                // together (one L2 round trip under full HBM load), more in a
                // pass for the maxima and one per contributor after it.
                constexpr int kMergeBatch = 8;
                const int ncon = cl - cf;
                float Mt = M, Lt = 0.f, at = 0.f;
                if (ncon <= kMergeBatch) {
                    float mm[kMergeBatch], ll[kMergeBatch], oo[kMergeBatch];
#pragma unroll
                    for (int e = 0; e < kMergeBatch; ++e) {
                        if (e < ncon) {
                            const long long base = static_cast<long long>((cf + 1 + e) * 2) * NREP + r;
                            mm[e] = __ldcg(part_ml + base * 2);
                            ll[e] = __ldcg(part_ml + base * 2 + 1);
                            oo[e] = __ldcg(part_o + base * HD + d);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < kMergeBatch; ++e)
                        if (e < ncon) Mt = fmaxf(Mt, mm[e]);
                    const float f0 = (M == -INFINITY) ? 0.f : __expf(M - Mt);
                    Lt += L * f0;
                    at += acc * f0;
#pragma unroll
                    for (int e = 0; e < kMergeBatch; ++e) {
                        if (e < ncon) {
                            const float f = (mm[e] == -INFINITY) ? 0.f : __expf(mm[e] - Mt);
                            Lt += ll[e] * f;
                            at += oo[e] * f;
                        }
                    }
                } else {
                    for (int cc = cf + 1; cc <= cl; ++cc)
                        Mt = fmaxf(Mt, __ldcg(part_ml + (static_cast<long long>(cc * 2) * NREP + r) * 2));
                    const float f0 = (M == -INFINITY) ? 0.f : __expf(M - Mt);
                    Lt += L * f0;
                    at += acc * f0;
                    for (int cc = cf + 1; cc <= cl; ++cc) {
                        const long long base = static_cast<long long>(cc * 2) * NREP + r;
                        const float mm = __ldcg(part_ml + base * 2);
                        const float f = (mm == -INFINITY) ? 0.f : __expf(mm - Mt);
                        Lt += __ldcg(part_ml + base * 2 + 1) * f;
                        at += __ldcg(part_o + base * HD + d) * f;
                    }
                }
                out[static_cast<long long>(cur.b) * nq + h * HD + d] = from_f32<T>(at / Lt);
            }
        }
        if (!whole && !finisher) {
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) atomicAdd(&counters[cnt_idx], 1);
        }
        if (finisher && threadIdx.x == 0) counters[cnt_idx] = 0;
        __syncthreads();   // s_m / s_o / s_last reused by the next segment
        if (i + 1 < len) {
            advance(cur);
            seg_j0 = cur.j;
            seg_i0 = i + 1;
            start_pair();
        }
    }
    if (!ok && threadIdx.x == 0) {
        report_status(status, LLAMA_ERR_DEVICE_TIMEOUT);
        // units [fail_i, fail_i + NSLOT) were issued and not consumed: their
        // copies land before the CTA exits (a skipped unit is not waited for)
        for (int j = fail_i; j < len && j < fail_i + NSLOT; ++j)
            if (j != stall_i) mbar_wait(&bar[j % NSLOT], (j / NSLOT) & 1, wlim);
    }
    __syncthreads();
    if (threadIdx.x == 0) tl_stamp(tl);
}

static int g_attn_sms = 0;

template <typename T, int HD, int NREP, bool TC>
static int decode_go(const Model* m, int layer, const int32_t* pos, int B, cudaStream_t st, bool pdl,
                     unsigned long long* tl, long long wait_ns, int stall) {
    const T* kc = static_cast<const T*>(m->kc) + layer * m->kv_layer_elems;
    const T* vc = static_cast<const T*>(m->vc) + layer * m->kv_layer_elems;
    auto kern = attn_decode_kernel<T, HD, NREP, TC>;
    // the ring's K+V chunks, 1024-byte aligned
    const int smem = kDecodeSlots * 2 * kChunk * HD * static_cast<int>(sizeof(T)) + 1024;
    // first cache row of this layer in the [L * Bmax * nkv * S][hd] tensor maps
    const long long row_base = static_cast<long long>(layer) * m->Bmax * m->nkv * m->S;
    static int per_sm = 0;
    if (per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 128, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_decode_kernel)");
        if (per_sm < 1) per_sm = 1;
    }
    if (g_attn_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_attn_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_attn_sms <= 0) g_attn_sms = 148;
    }
    if (B > kMaxRows) { set_error("decode attention takes at most %d rows", kMaxRows); return LLAMA_ERR_INVALID_ARG; }
    // one resident wave; never more CTAs than units (at least one unit per row and KV head)
    long long P = static_cast<long long>(g_attn_sms) * per_sm;
    P = std::min<long long>(P, kMaxAttnCtas);
    P = std::min<long long>(P, static_cast<long long>(B) * m->nkv * m->n_splits);
    P = std::max<long long>(P, 1);
    cudaError_t e = launch_k(kern, dim3(static_cast<unsigned>(P)), dim3(128), smem, st, pdl, static_cast<const T*>(m->q),
                             kc, vc, m->m_kdec, m->m_vdec, row_base, pos, B, m->nkv, m->nq, m->S, m->kv_row_elems,
                             m->part_o, m->part_ml, m->attn_cnt, static_cast<T*>(m->attn), m->status, tl, wait_ns,
                             stall);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "attn_decode_kernel");
    return LLAMA_OK;
}

template <typename T, int HD>
static int decode_rep(const Model* m, int layer, const int32_t* pos, int B, cudaStream_t st, bool pdl,
                      unsigned long long* tl, long long wait_ns, int stall) {
    // 16-bit caches with head_dim 128 and their tensor maps: units on the tensor cores
    constexpr bool kTcOk = HD == 128 && sizeof(T) == 2;
    if (kTcOk && m->has_dec_maps) {
        switch (m->n_rep) {
            case 1: return decode_go<T, HD, 1, kTcOk>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
            case 2: return decode_go<T, HD, 2, kTcOk>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
            case 4: return decode_go<T, HD, 4, kTcOk>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
            case 8: return decode_go<T, HD, 8, kTcOk>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
        }
    }
    switch (m->n_rep) {
        case 1: return decode_go<T, HD, 1, false>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
        case 2: return decode_go<T, HD, 2, false>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
        case 4: return decode_go<T, HD, 4, false>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
        case 8: return decode_go<T, HD, 8, false>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
    }
    set_error("n_heads / n_kv_heads = %d unsupported (1, 2, 4, 8)", m->n_rep);
    return LLAMA_ERR_INVALID_ARG;
}

template <typename T>
static int decode_hd(const Model* m, int layer, const int32_t* pos, int B, cudaStream_t st, bool pdl,
                     unsigned long long* tl, long long wait_ns, int stall) {
    switch (m->hd) {
        case 32: return decode_rep<T, 32>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
        case 64: return decode_rep<T, 64>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
        case 128: return decode_rep<T, 128>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
    }
    set_error("head_dim %d unsupported", m->hd);
    return LLAMA_ERR_INVALID_ARG;
}

int launch_attention_decode(const Model* m, int layer, const int32_t* pos, int B, cudaStream_t st, bool pdl,
                            unsigned long long* tl, long long wait_ns, int stall) {
    if (m->dtype == LLAMA_BF16) return decode_hd<bf16>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
    if (m->dtype == LLAMA_F16) return decode_hd<f16>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
    return decode_hd<float>(m, layer, pos, B, st, pdl, tl, wait_ns, stall);
}

// ---------------------------------------------------------------- prefill
namespace {
constexpr int PQ = 64;    // queries per CTA
constexpr int PK = 64;    // keys per tile
}

template <typename T, int HD>
__global__ void __launch_bounds__(256)
attn_prefill_kernel(RowTable rt, const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                    int nq, int n_rep, int S, long long row_stride, T* __restrict__ out) {
    extern __shared__ float sm[];
    float* Qs = sm;                        // [PQ][HD+1]
    float* Ks = Qs + PQ * (HD + 1);        // [PK][HD+1]
    float* Vs = Ks + PK * (HD + 1);        // [PK][HD]
    float* Ps = Vs + PK * HD;              // [PQ][PK+1]
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int len = rt.cu[b + 1] - rt.cu[b];
    const int t0 = qt * PQ;
    if (t0 >= len) return;
    const int nqt = min(PQ, len - t0);
    const int g = h / n_rep;
    const long long tok0 = rt.cu[b] + t0;
    const int tid = threadIdx.x, qi = tid >> 2, sub = tid & 3;
    constexpr int DPT = HD / 4;            // output dims per thread: sub, sub+4, sub+8, ...
    const float scale = rsqrtf(static_cast<float>(HD));

    for (int i = tid; i < PQ * HD; i += 256) {
        const int r = i / HD, d = i % HD;
        Qs[r * (HD + 1) + d] = r < nqt ? to_f32(q[(tok0 + r) * nq + h * HD + d]) * scale : 0.f;
    }
    const T* kb = kc + static_cast<long long>(b) * row_stride + static_cast<long long>(g) * S * HD;
    const T* vb = vc + static_cast<long long>(b) * row_stride + static_cast<long long>(g) * S * HD;
    const int my_pos = rt.start_pos + t0 + qi;       // absolute position of this thread's query
    const int kend = rt.start_pos + t0 + nqt;        // keys [0, kend) are needed by the tile

    float m_run = -INFINITY, l_run = 0.f;
    float o[DPT];
#pragma unroll
    for (int e = 0; e < DPT; ++e) o[e] = 0.f;

    for (int k0 = 0; k0 < kend; k0 += PK) {
        __syncthreads();
        const int nk = min(PK, kend - k0);
        for (int i = tid; i < PK * HD; i += 256) {
            const int r = i / HD, d = i % HD;
            const bool in = r < nk;
            Ks[r * (HD + 1) + d] = in ? to_f32(kb[static_cast<long long>(k0 + r) * HD + d]) : 0.f;
            Vs[r * HD + d] = in ? to_f32(vb[static_cast<long long>(k0 + r) * HD + d]) : 0.f;
        }
        __syncthreads();
        float sc[PK / 4];
        float tmax = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < PK / 4; ++jj) {
            const int j = sub + 4 * jj;
            float d = 0.f;
#pragma unroll 8
            for (int e = 0; e < HD; ++e) d = fmaf(Qs[qi * (HD + 1) + e], Ks[j * (HD + 1) + e], d);
            const bool vis = (j < nk) && (k0 + j <= my_pos) && (qi < nqt);
            sc[jj] = vis ? d : -INFINITY;
            tmax = fmaxf(tmax, sc[jj]);
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float mnew = fmaxf(m_run, tmax);
        const float corr = (m_run == -INFINITY) ? 0.f : __expf(m_run - mnew);
        float psum = 0.f;
#pragma unroll
        for (int jj = 0; jj < PK / 4; ++jj) {
            const float pj = (sc[jj] == -INFINITY) ? 0.f : __expf(sc[jj] - mnew);
            Ps[qi * (PK + 1) + sub + 4 * jj] = pj;
            psum += pj;
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 1);
        psum += __shfl_xor_sync(0xffffffffu, psum, 2);
        l_run = l_run * corr + psum;
        m_run = mnew;
        __syncwarp();
#pragma unroll
        for (int e = 0; e < DPT; ++e) o[e] *= corr;
        for (int j = 0; j < nk; ++j) {
            const float pj = Ps[qi * (PK + 1) + j];
#pragma unroll
            for (int e = 0; e < DPT; ++e) o[e] = fmaf(pj, Vs[j * HD + sub + 4 * e], o[e]);
        }
    }
    if (qi < nqt) {
        const float inv = 1.f / l_run;
        T* dst = out + (tok0 + qi) * nq + h * HD + sub;
#pragma unroll
        for (int e = 0; e < DPT; ++e) dst[4 * e] = from_f32<T>(o[e] * inv);
    }
}

template <typename T, int HD>
static int prefill_go(const Model* m, int layer, const RowTable& rt, cudaStream_t st) {
    const int smem = (PQ * (HD + 1) + PK * (HD + 1) + PK * HD + PQ * (PK + 1)) * 4;
    auto kern = attn_prefill_kernel<T, HD>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_prefill_kernel)");
        attr = true;
    }
    int maxlen = 0;
    for (int b = 0; b < rt.B; ++b) maxlen = max(maxlen, rt.cu[b + 1] - rt.cu[b]);
    dim3 grid((maxlen + PQ - 1) / PQ, m->nh, rt.B);
    const T* kc = static_cast<const T*>(m->kc) + layer * m->kv_layer_elems;
    const T* vc = static_cast<const T*>(m->vc) + layer * m->kv_layer_elems;
    kern<<<grid, 256, smem, st>>>(rt, static_cast<const T*>(m->q), kc, vc, m->nq, m->n_rep, m->S,
                                  m->kv_row_elems, static_cast<T*>(m->attn));
    LLB_CHECK_LAUNCH("attn_prefill_kernel");
    return LLAMA_OK;
}

template <typename T>
static int prefill_hd(const Model* m, int layer, const RowTable& rt, cudaStream_t st) {
    switch (m->hd) {
        case 32: return prefill_go<T, 32>(m, layer, rt, st);
        case 64: return prefill_go<T, 64>(m, layer, rt, st);
        case 128: return prefill_go<T, 128>(m, layer, rt, st);
    }
    set_error("head_dim %d unsupported", m->hd);
    return LLAMA_ERR_INVALID_ARG;
}

int launch_attention_prefill(const Model* m, int layer, const RowTable& rt, cudaStream_t st) {
    // 16-bit models run a tensor-core kernel (tcgen05 with TMEM accumulators
    // for head_dim 128, mma.sync for 32 and 64); fp32 models the CUDA-core one (no TF32)
    if (attention_prefill_tmem_ok(m)) return launch_attention_prefill_tmem(m, layer, rt, st);
    if (m->dtype != LLAMA_F32) return launch_attention_prefill_tc(m, layer, rt, st);
    return prefill_hd<float>(m, layer, rt, st);
}

}  // namespace llb
