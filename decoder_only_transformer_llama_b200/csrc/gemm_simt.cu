// fp32 projection kernel (CUDA-core FFMA, no TF32) for fp32 models, with the
// fused epilogues.  acc[m, n] = sum_k A[m, k] * W[n, k]  (nn.Linear, y = x W^T).
//
// Tile 32 x 128, k-step 16, 256 threads.  Thread (ty, tx) owns rows
// 4ty..4ty+3 and columns {c0, c0+1, c0+16, c0+17}, c0 = 32*(tx/8) + 2*(tx%8):
// the first two form a RoPE pair, and column c with c+16 form a w1/w3 pair of
// the SwiGLU weight (interleaved in blocks of 16 rows), so every epilogue
// sees its operands in one thread.
#include "common.cuh"
#include "epilogue.cuh"
#include "model.h"

namespace llb {

namespace {
constexpr int BM = 32, BN = 128, BK = 16;
}

__global__ void __launch_bounds__(256) linear_f32_kernel(const float* __restrict__ A,
                                                         const float* __restrict__ W, int M, int N,
                                                         int K, Epi ep) {
    __shared__ float As[BK][BM];
    __shared__ float Ws[BK][BN + 4];
    const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    float acc[4][4] = {};
    const int c0 = 32 * (tx >> 3) + 2 * (tx & 7);
    const int cols[4] = {c0, c0 + 1, c0 + 16, c0 + 17};

    for (int k0 = 0; k0 < K; k0 += BK) {
        for (int i = tid; i < BM * BK; i += 256) {
            const int r = i / BK, c = i % BK;
            const int gm = m0 + r, gk = k0 + c;
            As[c][r] = (gm < M && gk < K) ? A[static_cast<long long>(gm) * K + gk] : 0.f;
        }
        for (int i = tid; i < BN * BK; i += 256) {
            const int r = i / BK, c = i % BK;
            const int gn = n0 + r, gk = k0 + c;
            Ws[c][r] = (gn < N && gk < K) ? W[static_cast<long long>(gn) * K + gk] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = Ws[kk][cols[j]];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
        if (ep.mode == EPI_SWIGLU) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int n = n0 + cols[e];
                if (n >= N) continue;
                const int h = ((n0 + cols[e]) / 32) * 16 + (cols[e] & 15);
                static_cast<float*>(ep.g)[static_cast<long long>(m) * ep.H + h] =
                    silu_f(acc[i][e]) * acc[i][e + 2];
            }
            continue;
        }
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int n = n0 + cols[2 * p];
            if (n >= N) continue;
            const float v0 = acc[i][2 * p], v1 = acc[i][2 * p + 1];
            if (ep.mode == EPI_QKV) {
                epi_qkv_pair<float>(ep, m, n, v0, v1);
            } else {
                float* o = ep.out + static_cast<long long>(m) * ep.ldo + n;
                if (ep.mode == EPI_RESID_F32) {
                    o[0] += v0;
                    if (n + 1 < N) o[1] += v1;
                } else {
                    o[0] = v0;
                    if (n + 1 < N) o[1] = v1;
                }
            }
        }
    }
}

int linear_f32(const float* A, const float* W, int M, int N, int K, const Epi& ep, cudaStream_t st) {
    if (M <= 0 || N <= 0) return LLAMA_OK;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
    linear_f32_kernel<<<grid, 256, 0, st>>>(A, W, M, N, K, ep);
    LLB_CHECK_LAUNCH("linear_f32_kernel");
    return LLAMA_OK;
}

}  // namespace llb
