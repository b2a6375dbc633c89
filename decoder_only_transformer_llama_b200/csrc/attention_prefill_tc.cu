// Causal GQA prefill attention for 16-bit (bf16 or fp16) models on the tensor cores
// (Admin Guide §8.4, Attention steps 5-7 and the mask NOTE; repeat_kv from
// the source tour): o_h = softmax(q_h K_g^T / sqrt(hd)) V_g over keys
// 0 .. position of the query, g = h / n_rep.
//
// One CTA = 64 queries of one (row, head); 4 warps x 16 queries.  Key/value
// tiles of 64 positions stream through a double-buffered, XOR-swizzled
// shared-memory ring (cp.async, 16-byte chunks).  S = Q K^T and O += P V are
// m16n8k16 16-bit MMAs with fp32 accumulation; the online softmax runs on the
// S accumulator registers, which are re-packed as the A operand of P V
// without leaving registers.  The causal mask is a key-range bound plus a
// per-element test on the diagonal tile.
#include <type_traits>

#include "common.cuh"
#include "model.h"

namespace llb {

namespace {
constexpr int FQ = 64;    // queries per CTA
constexpr int FK = 64;    // keys per tile

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int n = valid ? 16 : 0;   // zero-fill when invalid
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D (+)= A B, m16n8k16, 16-bit E operands (bf16 or fp16), fp32 accumulate.
template <typename E>
__device__ __forceinline__ void mma16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                      uint32_t b0, uint32_t b1) {
    if constexpr (std::is_same<E, bf16>::value) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

// byte offset of 16-byte chunk `c` of row `r` in a tile whose rows hold HD
// 16-bit values (HD/8 chunks); chunks are XOR-swizzled by the row to spread banks.
template <int HD>
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>(r * (HD * 2) + ((c ^ (r & 7)) << 4));
}
}  // namespace

template <int HD, typename E>
__global__ void __launch_bounds__(128)
attn_prefill_tc_kernel(RowTable rt, const E* __restrict__ q, const E* __restrict__ kc,
                       const E* __restrict__ vc, int nq, int n_rep, int S, long long row_stride,
                       E* __restrict__ out) {
    constexpr int CH = HD / 8;                 // 16-byte chunks per row
    constexpr int TILE_BYTES = FK * HD * 2;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* sQ = smem;                        // [FQ][HD]
    uint8_t* sK = smem + FQ * HD * 2;          // 2 x [FK][HD]
    uint8_t* sV = sK + 2 * TILE_BYTES;         // 2 x [FK][HD]

    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int len = rt.cu[b + 1] - rt.cu[b];
    const int t0 = qt * FQ;
    if (t0 >= len) return;
    const int nqt = min(FQ, len - t0);
    const int g = h / n_rep;
    const long long tok0 = rt.cu[b] + t0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kend = rt.start_pos + t0 + nqt;            // keys [0, kend) are needed
    const int ntiles = (kend + FK - 1) / FK;
    const E* kb = kc + static_cast<long long>(b) * row_stride + static_cast<long long>(g) * S * HD;
    const E* vb = vc + static_cast<long long>(b) * row_stride + static_cast<long long>(g) * S * HD;

    const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
    // Q tile (rows beyond the row's length are zero)
    for (int i = tid; i < FQ * CH; i += 128) {
        const int r = i / CH, c = i % CH;
        const bool ok = r < nqt;
        cp_async16(sQa + swz<HD>(r, c), q + (tok0 + (ok ? r : 0)) * nq + h * HD + c * 8, ok);
    }
    auto load_kv = [&](int tile, int buf) {
        const int k0 = tile * FK;
        for (int i = tid; i < FK * CH; i += 128) {
            const int r = i / CH, c = i % CH;
            const bool ok = k0 + r < kend;
            const long long off = static_cast<long long>(ok ? k0 + r : 0) * HD + c * 8;
            cp_async16(sKa + buf * TILE_BYTES + swz<HD>(r, c), kb + off, ok);
            cp_async16(sVa + buf * TILE_BYTES + swz<HD>(r, c), vb + off, ok);
        }
    };
    load_kv(0, 0);
    cp_async_commit();

    const int gq = lane >> 2, tq = lane & 3;              // mma fragment coordinates
    const float scale_log2 = rsqrtf(static_cast<float>(HD)) * 1.4426950408889634f;
    // absolute positions of this thread's two query rows
    const int qrow0 = warp * 16 + gq, qrow1 = qrow0 + 8;
    const int pos0 = rt.start_pos + t0 + qrow0, pos1 = rt.start_pos + t0 + qrow1;

    float o[HD / 8][4];
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    uint32_t qa[HD / 16][4];

    for (int tile = 0; tile < ntiles; ++tile) {
        const int buf = tile & 1;
        if (tile + 1 < ntiles) load_kv(tile + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (tile == 0) {
            // Q fragments: matrices (rows 0-7|8-15) x (cols 0-7|8-15) of each 16-wide k step
            const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < HD / 16; ++ks) {
                const int c = ks * 2 + (lane >> 4);
                ldsm_x4(sQa + swz<HD>(r, c), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
            }
        }
        const int k0 = tile * FK;
        // ---- S = Q K^T  (16 queries x 64 keys per warp)
        float s[FK / 8][4];
#pragma unroll
        for (int j = 0; j < FK / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
        const uint32_t kbase = sKa + buf * TILE_BYTES;
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
#pragma unroll
            for (int jp = 0; jp < FK / 16; ++jp) {
                // matrices: (keys 16jp+0..7, hd lo), (keys 16jp+0..7, hd hi), (keys +8..15, lo), (+8..15, hi)
                const int r = jp * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int c = ks * 2 + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + swz<HD>(r, c), b0, b1, b2, b3);
                mma16<E>(s[2 * jp], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
                mma16<E>(s[2 * jp + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
            }
        }
        // ---- mask + online softmax (rows gq and gq+8 of this warp's 16)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < FK / 8; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int key = k0 + j * 8 + 2 * tq + e;
                s[j][e] = (key <= pos0 && key < kend) ? s[j][e] * scale_log2 : -INFINITY;
                s[j][2 + e] = (key <= pos1 && key < kend) ? s[j][2 + e] * scale_log2 : -INFINITY;
                mx0 = fmaxf(mx0, s[j][e]);
                mx1 = fmaxf(mx1, s[j][2 + e]);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
        const float c0 = exp2f(m0 - base0), c1 = exp2f(m1 - base1);   // m == -inf gives 0
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int j = 0; j < FK / 8; ++j) {
            s[j][0] = exp2f(s[j][0] - base0);
            s[j][1] = exp2f(s[j][1] - base0);
            s[j][2] = exp2f(s[j][2] - base1);
            s[j][3] = exp2f(s[j][3] - base1);
            ps0 += s[j][0] + s[j][1];
            ps1 += s[j][2] + s[j][3];
        }
        ps0 += __shfl_xor_sync(0xffffffffu, ps0, 1);
        ps0 += __shfl_xor_sync(0xffffffffu, ps0, 2);
        ps1 += __shfl_xor_sync(0xffffffffu, ps1, 1);
        ps1 += __shfl_xor_sync(0xffffffffu, ps1, 2);
        l0 = l0 * c0 + ps0;
        l1 = l1 * c1 + ps1;
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) {
            o[j][0] *= c0; o[j][1] *= c0;
            o[j][2] *= c1; o[j][3] *= c1;
        }
        // ---- O += P V
        const uint32_t vbase = sVa + buf * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < FK / 16; ++kk) {
            const uint32_t a0 = pack2<E>(s[2 * kk][0], s[2 * kk][1]);
            const uint32_t a1 = pack2<E>(s[2 * kk][2], s[2 * kk][3]);
            const uint32_t a2 = pack2<E>(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            const uint32_t a3 = pack2<E>(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int jd = 0; jd < HD / 16; ++jd) {
                // matrices (transposed): (keys lo, d 16jd+0..7), (keys hi, d lo), (keys lo, d +8..15), (keys hi, d hi)
                const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int c = jd * 2 + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vbase + swz<HD>(r, c), b0, b1, b2, b3);
                mma16<E>(o[2 * jd], a0, a1, a2, a3, b0, b1);
                mma16<E>(o[2 * jd + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncthreads();   // buffer `buf` is refilled two tiles later
    }

    // ---- normalise and store
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
        const int d = j * 8 + 2 * tq;
        if (qrow0 < nqt)
            *reinterpret_cast<uint32_t*>(out + (tok0 + qrow0) * nq + h * HD + d) = pack2<E>(o[j][0] * inv0, o[j][1] * inv0);
        if (qrow1 < nqt)
            *reinterpret_cast<uint32_t*>(out + (tok0 + qrow1) * nq + h * HD + d) = pack2<E>(o[j][2] * inv1, o[j][3] * inv1);
    }
}

template <int HD, typename E>
static int prefill_tc_go(const Model* m, int layer, const RowTable& rt, cudaStream_t st) {
    const int smem = (FQ * HD + 4 * FK * HD) * 2;
    auto kern = attn_prefill_tc_kernel<HD, E>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_prefill_tc_kernel)");
        attr = true;
    }
    int maxlen = 0;
    for (int b = 0; b < rt.B; ++b) maxlen = max(maxlen, rt.cu[b + 1] - rt.cu[b]);
    dim3 grid((maxlen + FQ - 1) / FQ, m->nh, rt.B);
    const E* kc = static_cast<const E*>(m->kc) + layer * m->kv_layer_elems;
    const E* vc = static_cast<const E*>(m->vc) + layer * m->kv_layer_elems;
    kern<<<grid, 128, smem, st>>>(rt, static_cast<const E*>(m->q), kc, vc, m->nq, m->n_rep, m->S,
                                  m->kv_row_elems, static_cast<E*>(m->attn));
    LLB_CHECK_LAUNCH("attn_prefill_tc_kernel");
    return LLAMA_OK;
}

int launch_attention_prefill_tc(const Model* m, int layer, const RowTable& rt, cudaStream_t st) {
    const bool f16m = m->dtype == LLAMA_F16;
    switch (m->hd) {
        case 32: return f16m ? prefill_tc_go<32, f16>(m, layer, rt, st) : prefill_tc_go<32, bf16>(m, layer, rt, st);
        case 64: return f16m ? prefill_tc_go<64, f16>(m, layer, rt, st) : prefill_tc_go<64, bf16>(m, layer, rt, st);
        case 128: return f16m ? prefill_tc_go<128, f16>(m, layer, rt, st) : prefill_tc_go<128, bf16>(m, layer, rt, st);
    }
    set_error("head_dim %d unsupported", m->hd);
    return LLAMA_ERR_INVALID_ARG;
}

}  // namespace llb
