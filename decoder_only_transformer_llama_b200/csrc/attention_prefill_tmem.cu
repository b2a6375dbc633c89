// Causal GQA prefill attention for 16-bit models with head_dim 128 on the
// 5th-generation tensor cores (Admin Guide §8.4, Attention steps 5-7 and the
// mask NOTE; repeat_kv from the source tour):
//   o_h = softmax(q_h K_g^T / sqrt(128)) V_g over keys 0 .. position of the query,
//   g = h / n_rep.
//
// One CTA = 128 queries of one (batch row, query head): the 128 TMEM lanes.
// Key/value tiles of 128 positions arrive by TMA (this GPU's memory only, no
// multicast) into a two-deep ring; both products run on tcgen05:
//   S_j = Q K_j^T   (M 128 queries, N 128 keys, K 128 head dims; K-major operands)
//                   into one of two 128-column TMEM buffers, so S_{j+1} is
//                   computed while the softmax of S_j runs;
//   O  += P_j V_j   (M 128 queries, N 128 head dims, K 128 keys): P_j from
//                   shared memory (K-major), V_j read MN-major straight from
//                   its TMA tile; O stays in TMEM for the whole row of tiles.
// Softmax warps own one query row per thread (its TMEM lane): they read the
// scores with tcgen05.ld, apply the causal mask (key <= query position; the
// -inf of the reference's mask), and keep the running maximum m and sum l in
// registers, in the log2 domain.  The maximum that P is taken against is
// moved only when a tile raises it by more than 8 (a factor 256): then O is
// rescaled in TMEM (load, multiply, store) before the next P V product;
// otherwise P = 2^(s - m) <= 256 against the kept maximum.  Both l and O use
// the same maximum, so the final O / l is the exact softmax average.
//
// Warp roles (192 threads): warp 0 lane 0 TMA producer; warp 1 lane 0 MMA
// issuer and TMEM owner (512 columns: S0, S1, O); warps 2-5 softmax and the
// epilogue (warp w reads TMEM lanes 32 * (w % 4) .. +31).  Every wait is
// bounded.
#include "common.cuh"
#include "model.h"

namespace llb {

namespace {
constexpr int kTq = 128;                    // queries per CTA
constexpr int kTk = 128;                    // keys per tile
constexpr int kHd = 128;                    // head dim handled here
constexpr int kBox = 128 * 128;             // one [128 rows][64 values] 16-bit box, 128-byte rows
constexpr int kTile = 2 * kBox;             // a [128][128] tile as two boxes (columns 0-63, 64-127)
constexpr int kThreads = 192;
// shared memory: Q | K[2] | V[2] | P | barriers
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;
constexpr int kOffV = kOffK + 2 * kTile;
constexpr int kOffP = kOffV + 2 * kTile;
constexpr int kOffBar = kOffP + kTile;
constexpr int kSmem = 1024 + kOffBar + 16 * 8 + 16;
}  // namespace

template <typename E>
__global__ void __launch_bounds__(kThreads, 1)
attn_prefill_tmem_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                         const __grid_constant__ CUtensorMap mapV, RowTable rt, int kv_row_base, int nkv, int S,
                         int nq, int n_rep, E* __restrict__ out, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bar + 0;
    uint64_t* kv_full = bar + 1;     // [2]
    uint64_t* kv_empty = bar + 3;    // [2]
    uint64_t* s_full = bar + 5;      // [2]
    uint64_t* s_empty = bar + 7;     // [2]
    uint64_t* p_full = bar + 9;
    uint64_t* p_empty = bar + 10;
    uint64_t* mdone = bar + 11;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 12);
    int* flag = reinterpret_cast<int*>(bar + 13);

    const int nqt_tiles = gridDim.x;
    const int qt = nqt_tiles - 1 - static_cast<int>(blockIdx.x);   // longest query tiles first
    const int h = blockIdx.y, b = blockIdx.z;
    const int len = rt.cu[b + 1] - rt.cu[b];
    const int t0 = qt * kTq;
    if (t0 >= len) return;                   // the whole CTA, before any barrier or TMEM
    const int nqt = min(kTq, len - t0);
    const int g = h / n_rep;
    const int tok0 = rt.cu[b] + t0;
    const int p0 = rt.start_pos + t0;        // position of query row 0
    const int kend = p0 + nqt;               // keys [0, kend) are visible to some row
    const int nkt = (kend + kTk - 1) / kTk;
    const int kv_row0 = kv_row_base + (b * nkv + g) * S;   // cache row of key 0 of this (row, KV head)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 128);
        }
        mbar_init(p_full, 128);
        mbar_init(p_empty, 1);
        mbar_init(mdone, 1);
        flag[0] = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapQ);
        tma_prefetch_desc(&mapK);
        tma_prefetch_desc(&mapV);
    }
    if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;        // columns: S0 [0,128), S1 [128,256), O [256,384)

    int issued = 0;                          // producer: K/V tiles [0, issued) were issued
    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        mbar_arrive_expect_tx(q_full, kTile);
        tma_load_2d(smem + kOffQ, &mapQ, h * kHd, tok0, q_full);
        tma_load_2d(smem + kOffQ + kBox, &mapQ, h * kHd + 64, tok0, q_full);
        for (int j = 0; j < nkt; ++j) {
            const int s = j & 1;
            if (!mbar_wait(&kv_empty[s], ((j >> 1) & 1) ^ 1)) { atomicExch(&flag[0], 1); break; }
            mbar_arrive_expect_tx(&kv_full[s], 2 * kTile);
            const int row = kv_row0 + j * kTk;
            tma_load_2d(smem + kOffK + s * kTile, &mapK, 0, row, &kv_full[s]);
            tma_load_2d(smem + kOffK + s * kTile + kBox, &mapK, 64, row, &kv_full[s]);
            tma_load_2d(smem + kOffV + s * kTile, &mapV, 0, row, &kv_full[s]);
            tma_load_2d(smem + kOffV + s * kTile + kBox, &mapV, 64, row, &kv_full[s]);
            issued = j + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        const uint32_t idesc_s = idesc_16_f32<E>(kTq, kTk);
        const uint32_t idesc_o = idesc_16_f32_bmn<E>(kTq, kHd);
        const uint32_t sQ = smem_u32(smem + kOffQ), sK = smem_u32(smem + kOffK), sV = smem_u32(smem + kOffV),
                       sP = smem_u32(smem + kOffP);
        bool ok = mbar_wait(q_full, 0);
        auto issue_s = [&](int j) -> bool {
            const int s = j & 1;
            if (!mbar_wait(&kv_full[s], (j >> 1) & 1)) return false;
            if (!mbar_wait(&s_empty[s], ((j >> 1) & 1) ^ 1)) return false;
            tc_fence_after();
            const uint32_t kb = sK + s * kTile;
#pragma unroll
            for (int kk = 0; kk < kHd / 16; ++kk) {
                const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                tc_mma_16(tmem + s * kTk, smem_desc_k_sw128(sQ + off), smem_desc_k_sw128(kb + off), idesc_s,
                          kk > 0 ? 1u : 0u);
            }
            tc_commit(&s_full[s]);
            return true;
        };
        if (ok) ok = issue_s(0);
        if (ok && nkt > 1) ok = issue_s(1);
        for (int j = 0; ok && j < nkt; ++j) {
            const int s = j & 1;
            if (!mbar_wait(p_full, j & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t vb = sV + s * kTile;
#pragma unroll
            for (int kk = 0; kk < kTk / 16; ++kk) {
                const uint32_t a_off = (kk >> 2) * kBox + (kk & 3) * 32;   // P: 16 keys of each query row
                const uint32_t b_off = kk * 16 * 128;                      // V: rows (keys) 16 kk .. 16 kk + 15
                tc_mma_16(tmem + 2 * kTk, smem_desc_k_sw128(sP + a_off), smem_desc_mn_sw128(vb + b_off, kBox),
                          idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(p_empty);       // P buffer free, O holds tiles 0 .. j
            tc_commit(&kv_empty[s]);  // K/V stage free
            if (j + 2 < nkt) ok = issue_s(j + 2);
        }
        if (!ok) atomicExch(&flag[0], 1);
        // every MMA issued here has finished before TMEM is freed
        tc_commit(mdone);
        if (!mbar_wait(mdone, 0)) atomicExch(&flag[0], 1);
    } else if (warp >= 2) {
        // ---------------- softmax and epilogue: thread = query row r (TMEM lane r)
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const int qpos = p0 + r;
        const float scale_log2 = 0.08838834764831845f * 1.4426950408889634f;   // log2(e) / sqrt(128)
        float m_run = -INFINITY, l = 0.f;
        uint8_t* prow = smem + kOffP + r * 128;
        const int sw = r & 7;
        bool ok = true;
        for (int j = 0; j < nkt; ++j) {
            const int s = j & 1;
            ok = mbar_wait(&s_full[s], (j >> 1) & 1);
            tc_fence_after();
            if (named_any(1, 128, !ok || *reinterpret_cast<volatile int*>(&flag[0]) != 0)) { ok = false; break; }
            float v[kTk];
#pragma unroll
            for (int c = 0; c < kTk / 32; ++c) tmem_ld_32x32b_x16(tmem + lane_base + s * kTk + c * 32, v + 32 * c),
                                               tmem_ld_32x32b_x16(tmem + lane_base + s * kTk + c * 32 + 16, v + 32 * c + 16);
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(&s_empty[s]);
            const int key0 = j * kTk;
            float mx = -INFINITY;
            if (key0 + kTk - 1 <= p0 && key0 + kTk <= kend) {
                // every key of the tile is visible to every row
#pragma unroll
                for (int c = 0; c < kTk; ++c) { v[c] *= scale_log2; mx = fmaxf(mx, v[c]); }
            } else {
#pragma unroll
                for (int c = 0; c < kTk; ++c) {
                    const int key = key0 + c;
                    v[c] = (key <= qpos && key < kend) ? v[c] * scale_log2 : -INFINITY;
                    mx = fmaxf(mx, v[c]);
                }
            }
            // the maximum P is taken against: moved on the first tile, and
            // afterwards only when this tile raises it by more than 8
            bool rescale = false;
            float corr = 1.f;
            if (j == 0) {
                m_run = mx;
            } else if (mx > m_run + 8.f) {
                rescale = true;
                corr = exp2f(m_run - mx);
                m_run = mx;
            }
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < kTk; ++c) { v[c] = exp2f(v[c] - m_run); sum += v[c]; }
            l = l * corr + sum;
            // P buffer and O are free once the previous P V product has finished
            if (j > 0) {
                const bool okp = mbar_wait(p_empty, (j - 1) & 1);
                tc_fence_after();
                if (named_any(1, 128, !okp)) { ok = false; break; }
            }
            if (named_any(1, 128, rescale)) {
                // some row's maximum moved: every warp rescales its O rows in
                // TMEM together (tcgen05.ld/st are warp-wide), factor 1 where
                // the maximum stayed
#pragma unroll 1
                for (int c = 0; c < kHd / 32; ++c) {
                    float o[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + 2 * kTk + c * 32, o);
                    tc_wait_ld();
#pragma unroll
                    for (int t = 0; t < 32; ++t) o[t] *= corr;
                    tmem_st_32x32b_x32(tmem + lane_base + 2 * kTk + c * 32, o);
                }
                tc_wait_st();
            }
            // P row r into the K-major, 128-byte-swizzled operand tile: keys
            // 64 * box + 8 * chunk .. +7 sit in 16-byte chunk (chunk ^ (r & 7))
#pragma unroll
            for (int box = 0; box < 2; ++box) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const float* pv = v + box * 64 + ch * 8;
                    uint4 u;
                    u.x = pack2<E>(pv[0], pv[1]);
                    u.y = pack2<E>(pv[2], pv[3]);
                    u.z = pack2<E>(pv[4], pv[5]);
                    u.w = pack2<E>(pv[6], pv[7]);
                    *reinterpret_cast<uint4*>(prow + box * kBox + ((ch ^ sw) << 4)) = u;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok) {
            const bool okl = mbar_wait(p_empty, (nkt - 1) & 1);
            tc_fence_after();
            ok = !named_any(1, 128, !okl);
        }
        if (ok) {
            const float inv = 1.f / l;
            E* dst = out + static_cast<long long>(tok0 + r) * nq + h * kHd;
#pragma unroll 1
            for (int c = 0; c < kHd / 32; ++c) {
                float o[32];
                tmem_ld_32x32b_x32(tmem + lane_base + 2 * kTk + c * 32, o);
                tc_wait_ld();
                if (r < nqt) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                    for (int qv = 0; qv < 4; ++qv) {
                        uint4 u;
                        u.x = pack2<E>(o[8 * qv + 0] * inv, o[8 * qv + 1] * inv);
                        u.y = pack2<E>(o[8 * qv + 2] * inv, o[8 * qv + 3] * inv);
                        u.z = pack2<E>(o[8 * qv + 4] * inv, o[8 * qv + 5] * inv);
                        u.w = pack2<E>(o[8 * qv + 6] * inv, o[8 * qv + 7] * inv);
                        d4[qv] = u;
                    }
                }
            }
        } else if (threadIdx.x == 64) {
            atomicExch(&flag[0], 1);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
    if (warp == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&flag[0]) != 0) {
        report_status(status, LLAMA_ERR_DEVICE_TIMEOUT);
        // the copies still in flight land before the CTA exits
        if (issued > 0) mbar_wait(&kv_full[(issued - 1) & 1], ((issued - 1) >> 1) & 1);
        if (issued > 1) mbar_wait(&kv_full[(issued - 2) & 1], ((issued - 2) >> 1) & 1);
        mbar_wait(q_full, 0);
    }
}

// ---------------------------------------------------------------- host side

template <typename E>
static int go(const Model* m, int layer, const RowTable& rt, cudaStream_t st) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(attn_prefill_tmem_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_prefill_tmem_kernel)");
        attr = true;
    }
    int maxlen = 0;
    for (int b = 0; b < rt.B; ++b) maxlen = max(maxlen, rt.cu[b + 1] - rt.cu[b]);
    const dim3 grid((maxlen + kTq - 1) / kTq, m->nh, rt.B);
    const long long base = static_cast<long long>(layer) * m->Bmax * m->nkv * m->S;
    attn_prefill_tmem_kernel<E><<<grid, kThreads, kSmem, st>>>(m->m_qtile, m->m_kcache, m->m_vcache, rt,
                                                               static_cast<int>(base), m->nkv, m->S, m->nq, m->n_rep,
                                                               static_cast<E*>(m->attn), m->status);
    LLB_CHECK_LAUNCH("attn_prefill_tmem_kernel");
    return LLAMA_OK;
}

bool attention_prefill_tmem_ok(const Model* m) {
    return m->dtype != LLAMA_F32 && m->hd == kHd && m->has_attn_maps;
}

int launch_attention_prefill_tmem(const Model* m, int layer, const RowTable& rt, cudaStream_t st) {
    if (!attention_prefill_tmem_ok(m)) { set_error("tensor-memory prefill attention needs a 16-bit model with head_dim 128"); return LLAMA_ERR_INVALID_ARG; }
    return m->dtype == LLAMA_F16 ? go<f16>(m, layer, rt, st) : go<bf16>(m, layer, rt, st);
}

}  // namespace llb
