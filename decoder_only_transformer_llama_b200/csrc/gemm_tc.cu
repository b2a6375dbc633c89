// bf16 projections on the 5th-generation tensor cores (tcgen05), fed by TMA,
// accumulating in TMEM, with the fused epilogues of the forward pass
// (Admin Guide §8.4: wq/wk/wv + RoPE + KV-cache append, wo + residual,
// w1/w3 + silu*mul, w2 + residual, output projection).
//
// This file holds the prefill-shaped kernel (many token rows); decode-shaped
// projections (<= 64 rows) run in gemm_decode.cu.
//
// D[i, j] = sum_k A[i, k] * B[j, k]; A = activations [tokens, K], B = weights
// [N, K], both K-major bf16 read through 128-byte-swizzled TMA boxes of 64
// K-elements.  One CTA computes one 128 x 256 tile of D:
//   warp 0 lane 0  TMA producer (STAGES-deep ring of A/B tiles)
//   warp 1 lane 0  MMA issuer (tcgen05.mma kind::f16, M=128, N=256, K=16)
//   warp 1         TMEM allocation / release
//   warps 0-3      epilogue: TMEM lane i (token row i of the tile) -> thread i,
//                  TMEM columns = output features
// No TMA multicast is used.
#include "common.cuh"
#include "epilogue.cuh"
#include "model.h"

#include <cudaTypedefs.h>

namespace llb {

namespace {

constexpr int kA_BYTES = 128 * 128;          // 128 rows x 64 bf16

template <int BN>
struct TcCfg {
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = kA_BYTES + B_BYTES;
    static constexpr uint32_t TMEM_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&p);
}

// Store 32 consecutive values as bf16 (64 bytes, 16-byte aligned destination).
__device__ __forceinline__ void store32_bf16(bf16* dst, const float* v) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 u;
        u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        d[q] = u;
    }
}

}  // namespace

template <int BN, int STAGES, int B_BOX>
__global__ void __launch_bounds__(128, 1)
linear_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 int rowsA, int rowsB, int K, int kt_per_split, Epi ep) {
    using C = TcCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* accum = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tileA = blockIdx.x, tileB = blockIdx.y;
    const int KT = (K + 63) / 64;
    const int kt0 = blockIdx.z * kt_per_split;
    const int kt1 = min(KT, kt0 + kt_per_split);
    const int nk = kt1 - kt0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapA);
        tma_prefetch_desc(&mapB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            const uint32_t ph = (i / STAGES) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1)) { atomicExch(abort_flag, 1); break; }
            mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
            const int kx = (kt0 + i) * 64;
            uint8_t* st = smem + s * C::STAGE_BYTES;
            tma_load_2d(st, &mapA, kx, tileA * 128, &full[s]);
#pragma unroll
            for (int j = 0; j < BN / B_BOX; ++j)
                tma_load_2d(st + kA_BYTES + j * B_BOX * 128, &mapB, kx, tileB * BN + j * B_BOX, &full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        const uint32_t idesc = idesc_bf16_f32(128, BN);
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            const uint32_t ph = (i / STAGES) & 1;
            if (!mbar_wait(&full[s], ph)) { atomicExch(abort_flag, 1); break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + s * C::STAGE_BYTES);
            const uint32_t b0 = a0 + kA_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                tc_mma_bf16(tmem, smem_desc_k_sw128(a0 + kk * 32), smem_desc_k_sw128(b0 + kk * 32), idesc,
                            (i > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&empty[s]);
        }
        tc_commit(accum);
    }
    __syncthreads();

    // ---------------- epilogue
    const bool acc_ok = mbar_wait(accum, 0);
    tc_fence_after();
    __syncwarp();
    const bool ok = acc_ok && (*reinterpret_cast<volatile int*>(abort_flag) == 0) && nk > 0;
    if (!ok && threadIdx.x == 0) report_status(ep.status, LLAMA_ERR_DEVICE_TIMEOUT);
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);

    {
        // thread = token row m; TMEM columns = features n
        const int m = tileA * 128 + warp * 32 + lane;
        const bool row_ok = ok && m < rowsA;
        const int nbase = tileB * BN;
        if (ep.mode == EPI_SWIGLU) {
            // each 32-column chunk holds 16 w1 outputs then the same 16 w3 outputs
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                float v[32];
                tmem_ld_32x32b_x32(trow + c * 32, v);
                tc_wait_ld();
                const int n0 = nbase + c * 32;
                if (row_ok && n0 < rowsB) {
                    float g16[16];
#pragma unroll
                    for (int t = 0; t < 16; ++t) g16[t] = silu_f(v[t]) * v[16 + t];
                    bf16* dst = static_cast<bf16*>(ep.g) + static_cast<long long>(m) * ep.H + (n0 / 32) * 16;
                    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint4 u;
                        u.x = pack_bf16x2(g16[8 * q + 0], g16[8 * q + 1]);
                        u.y = pack_bf16x2(g16[8 * q + 2], g16[8 * q + 3]);
                        u.z = pack_bf16x2(g16[8 * q + 4], g16[8 * q + 5]);
                        u.w = pack_bf16x2(g16[8 * q + 6], g16[8 * q + 7]);
                        d4[q] = u;
                    }
                }
            }
        } else {
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                float v[32];
                tmem_ld_32x32b_x32(trow + c * 32, v);
                tc_wait_ld();
                const int n0 = nbase + c * 32;
                if (!row_ok || n0 >= rowsB) continue;
                if (ep.mode == EPI_QKV) {
                    const int pos = ep.tok_pos[m];
                    if (pos < 0 || pos >= ep.max_seq) continue;
                    bf16* dst;
                    bool rot;
                    int d0;
                    if (n0 < ep.nq) {
                        d0 = n0 % ep.hd;
                        rot = true;
                        dst = static_cast<bf16*>(ep.q) + static_cast<long long>(m) * ep.nq + n0;
                    } else {
                        int cc = n0 - ep.nq;
                        bf16* cache = static_cast<bf16*>(ep.kc);
                        rot = cc < ep.nkvc;
                        if (!rot) { cc -= ep.nkvc; cache = static_cast<bf16*>(ep.vc); }
                        const int head = cc / ep.hd;
                        d0 = cc % ep.hd;
                        const int row = ep.tok_row ? ep.tok_row[m] : m;
                        dst = cache + static_cast<long long>(row) * ep.kv_row_stride +
                              (static_cast<long long>(head) * ep.max_seq + pos) * ep.hd + d0;
                    }
                    if (rot) {
#pragma unroll
                        for (int t = 0; t < 32; t += 2) rope_pair(ep.rope, ep.hd, pos, (d0 + t) >> 1, v[t], v[t + 1]);
                    }
                    store32_bf16(dst, v);
                } else {
                    float* o = ep.out + static_cast<long long>(m) * ep.ldo + n0;
                    const int lim = min(32, rowsB - n0);
                    if (lim == 32 && (ep.ldo % 4) == 0) {
                        float4* o4 = reinterpret_cast<float4*>(o);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 r = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                            if (ep.mode == EPI_RESID_F32) {
                                const float4 p = o4[q];
                                r.x += p.x; r.y += p.y; r.z += p.z; r.w += p.w;
                            }
                            o4[q] = r;
                        }
                    } else {
                        for (int t = 0; t < lim; ++t) o[t] = (ep.mode == EPI_RESID_F32) ? o[t] + v[t] : v[t];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int encode_kmajor_bf16(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
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
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) rows=%d cols=%d box=%d", static_cast<int>(r), rows,
                  cols, box_rows);
        return LLAMA_ERR_CUDA;
    }
    return LLAMA_OK;
}

template <int BN, int STAGES, int B_BOX>
static int launch_tc(const CUtensorMap& a, const CUtensorMap& b, int rowsA, int rowsB, int K, int splits,
                     const Epi& ep, cudaStream_t st) {
    using C = TcCfg<BN>;
    constexpr int smem = STAGES * C::STAGE_BYTES + 1024 + (2 * STAGES + 1) * 8 + 16;
    auto kern = linear_tc_kernel<BN, STAGES, B_BOX>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(linear_tc_kernel)");
        attr_set = true;
    }
    const int KT = (K + 63) / 64;
    const int per = (KT + splits - 1) / splits;
    const int z = (KT + per - 1) / per;   // every split gets >= 1 k-tile
    dim3 grid((rowsA + 127) / 128, (rowsB + BN - 1) / BN, z);
    kern<<<grid, 128, smem, st>>>(a, b, rowsA, rowsB, K, per, ep);
    LLB_CHECK_LAUNCH("linear_tc_kernel");
    return LLAMA_OK;
}

int linear_bf16_tc(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, const Epi& ep,
                   cudaStream_t st) {
    if (M <= 0 || N <= 0) return LLAMA_OK;
    return launch_tc<256, 4, 256>(mapA->a128, mapW->b, M, N, K, 1, ep, st);
}

int linear_bf16(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, const Epi& ep, float* part,
                int* counters, cudaStream_t st, bool pdl, const NormIO* nio, const NextProj* next) {
    if (M <= 64) return linear_bf16_decode(mapA, mapW, M, N, K, ep, part, counters, st, pdl, nio, next);
    if (nio && (nio->ssq_in || nio->ssq_out)) { set_error("fused RMSNorm is a decode-shape feature"); return LLAMA_ERR_INVALID_ARG; }
    return linear_bf16_tc(mapA, mapW, M, N, K, ep, st);
}

}  // namespace llb
