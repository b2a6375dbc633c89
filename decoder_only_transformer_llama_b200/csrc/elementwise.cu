// Memory-bound helper kernels of the forward pass: RoPE table, token map,
// embedding lookup, RMSNorm, and the w1/w3 interleaving copy used at weight
// upload.  All HBM access is 16-byte vectorised where the row allows it.
#include "common.cuh"
#include "model.h"

namespace llb {

// ---------------------------------------------------------------- RoPE table
// rope[t][j] = (cos, sin)(t * theta^(-2j/hd)), evaluated in fp64 and rounded
// once to fp32 (Admin Guide §8.4, precompute_freqs_cis; standard schedule).
__global__ void rope_table_kernel(float2* rope, int S, int hd, double theta) {
    const int half = hd / 2;
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= S * half) return;
    const int t = idx / half, j = idx % half;
    const double freq = pow(theta, -2.0 * j / hd);
    const double ang = static_cast<double>(t) * freq;
    rope[idx] = make_float2(static_cast<float>(cos(ang)), static_cast<float>(sin(ang)));
}

int launch_rope_table(float2* rope, int S, int hd, float theta, cudaStream_t st) {
    const int n = S * (hd / 2);
    rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(rope, S, hd, static_cast<double>(theta));
    LLB_CHECK_LAUNCH("rope_table_kernel");
    return LLAMA_OK;
}

// ---------------------------------------------------------------- token map
// Packs the right-padded [B, T] token rectangle into Σlens rows and records
// each packed token's batch row and absolute position.
__global__ void token_map_kernel(RowTable rt, const int32_t* tokens, int* tok_ids, int* tok_row,
                                 int* tok_pos, int* last_idx) {
    const int b = blockIdx.x;
    const int beg = rt.cu[b], len = rt.cu[b + 1] - rt.cu[b];
    for (int t = threadIdx.x; t < len; t += blockDim.x) {
        tok_ids[beg + t] = tokens[static_cast<long long>(b) * rt.T + t];
        tok_row[beg + t] = b;
        tok_pos[beg + t] = rt.start_pos + t;
    }
    if (threadIdx.x == 0) last_idx[b] = beg + len - 1;
}

int launch_token_map(const RowTable& rt, const int32_t* tokens, int* tok_ids, int* tok_row,
                     int* tok_pos, int* last_idx, cudaStream_t st) {
    token_map_kernel<<<rt.B, 256, 0, st>>>(rt, tokens, tok_ids, tok_row, tok_pos, last_idx);
    LLB_CHECK_LAUNCH("token_map_kernel");
    return LLAMA_OK;
}

// ---------------------------------------------------------------- embedding
// x[m, :] = E[tok[m], :] as fp32 (Admin Guide §8.4, tok_embeddings).  An id
// outside [0, V) yields a zero row and sets LLAMA_ERR_TOKEN_RANGE.
// With `ssq`, also writes the sum of x^2 over each 128-feature block of the
// row (ssq[m * dim/128 + block]) and y[m, :] = x * w_next rounded to the
// 16-bit type: the next projection's fused RMSNorm inputs.
template <typename T>
__global__ void embed_kernel(const int* tok, const T* emb, int dim, int V, float* x, int* status, float* ssq,
                             T* y, const float* w_next, unsigned long long* tl) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x;
    const int id = tok[m];
    float* dst = x + static_cast<long long>(m) * dim;
    if (id < 0 || id >= V) {
        if (threadIdx.x == 0) report_status(status, LLAMA_ERR_TOKEN_RANGE);
        for (int i = threadIdx.x; i < dim; i += blockDim.x) dst[i] = 0.f;
        if (ssq)
            for (int i = threadIdx.x; i < dim / 128; i += blockDim.x) ssq[static_cast<long long>(m) * (dim / 128) + i] = 0.f;
        if (threadIdx.x == 0) tl_stamp(tl);
        return;
    }
    const T* src = emb + static_cast<long long>(id) * dim;
    if constexpr (sizeof(T) == 2) {
        // 8 16-bit values per 16-byte load
        // blockDim.x is a multiple of 16, so the 16 vectors of one 128-feature
        // block always sit in 16 adjacent lanes of one pass
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        for (int base = 0; base < dim / 8; base += blockDim.x) {
            const int i = base + threadIdx.x;
            float sq = 0.f;
            if (i < dim / 8) {
                uint4 u = s4[i];
                const T* h = reinterpret_cast<const T*>(&u);
                float4 lo = make_float4(to_f32(h[0]), to_f32(h[1]), to_f32(h[2]), to_f32(h[3]));
                float4 hi = make_float4(to_f32(h[4]), to_f32(h[5]), to_f32(h[6]), to_f32(h[7]));
                reinterpret_cast<float4*>(dst)[2 * i] = lo;
                reinterpret_cast<float4*>(dst)[2 * i + 1] = hi;
                sq = lo.x * lo.x + lo.y * lo.y + lo.z * lo.z + lo.w * lo.w + hi.x * hi.x + hi.y * hi.y +
                     hi.z * hi.z + hi.w * hi.w;
                if (y) {
                    const float4 w0 = reinterpret_cast<const float4*>(w_next)[2 * i];
                    const float4 w1 = reinterpret_cast<const float4*>(w_next)[2 * i + 1];
                    uint4 pk;
                    pk.x = pack2<T>(lo.x * w0.x, lo.y * w0.y);
                    pk.y = pack2<T>(lo.z * w0.z, lo.w * w0.w);
                    pk.z = pack2<T>(hi.x * w1.x, hi.y * w1.y);
                    pk.w = pack2<T>(hi.z * w1.z, hi.w * w1.w);
                    reinterpret_cast<uint4*>(y + static_cast<long long>(m) * dim)[i] = pk;
                }
            }
            if (ssq) {
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                if ((threadIdx.x & 15) == 0 && i < dim / 8)
                    ssq[static_cast<long long>(m) * (dim / 128) + i / 16] = sq;
            }
        }
    } else {
        const float4* s4 = reinterpret_cast<const float4*>(src);
        for (int i = threadIdx.x; i < dim / 4; i += blockDim.x)
            reinterpret_cast<float4*>(dst)[i] = s4[i];
    }
    if (threadIdx.x == 0) tl_stamp(tl);
}

int launch_embed(const int* tok_ids, const void* emb, int dtype, int M, int dim, int V, float* x,
                 int* status, cudaStream_t st, bool pdl, float* ssq, void* y, const float* w_next,
                 unsigned long long* tl) {
    if (M <= 0) return LLAMA_OK;
    static bool attr = false;
    if (!attr) {
        cudaError_t ce = carveout_max(embed_kernel<bf16>);
        if (ce == cudaSuccess) ce = carveout_max(embed_kernel<f16>);
        if (ce == cudaSuccess) ce = carveout_max(embed_kernel<float>);
        if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(embed_kernel)");
        attr = true;
    }
    cudaError_t e;
    if (dtype == LLAMA_BF16)
        e = launch_k(embed_kernel<bf16>, dim3(M), dim3(128), 0, st, pdl, tok_ids, static_cast<const bf16*>(emb),
                     dim, V, x, status, ssq, static_cast<bf16*>(y), w_next, tl);
    else if (dtype == LLAMA_F16)
        e = launch_k(embed_kernel<f16>, dim3(M), dim3(128), 0, st, pdl, tok_ids, static_cast<const f16*>(emb),
                     dim, V, x, status, ssq, static_cast<f16*>(y), w_next, tl);
    else
        e = launch_k(embed_kernel<float>, dim3(M), dim3(128), 0, st, pdl, tok_ids, static_cast<const float*>(emb),
                     dim, V, x, status, static_cast<float*>(nullptr), static_cast<float*>(nullptr),
                     static_cast<const float*>(nullptr), tl);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "embed_kernel");
    return LLAMA_OK;
}

// ---------------------------------------------------------------- RMSNorm
// out[m, :] = x[r, :] * rsqrt(mean(x[r, :]^2) + eps) * w, r = row_idx[m] (or m),
// all in fp32, one rounding to the output type (Admin Guide §8.4, RMSNorm).
// One CTA per row; each thread keeps its float4 slices in registers.
template <typename TO, int kVecPerThread>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* x, const int* row_idx,
                                                      const float* w, int dim, float eps, TO* out,
                                                      unsigned long long* tl) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x;
    const int r = row_idx ? row_idx[m] : m;
    const float4* xr = reinterpret_cast<const float4*>(x + static_cast<long long>(r) * dim);
    const int nv = dim / 4;
    float4 v[kVecPerThread];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
        const int c = threadIdx.x + i * blockDim.x;
        v[i] = c < nv ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    }
    __shared__ float red[32];
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        t = warp_sum(t);
        if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    const float inv = rsqrtf(red[0] / static_cast<float>(dim) + eps);
    const float4* w4 = reinterpret_cast<const float4*>(w);
    TO* orow = out + static_cast<long long>(m) * dim;
#pragma unroll
    for (int i = 0; i < kVecPerThread; ++i) {
        const int c = threadIdx.x + i * blockDim.x;
        if (c < nv) {
            const float4 ww = w4[c];
            if constexpr (sizeof(TO) == 2) {
                uint2 u;
                u.x = pack2<TO>(v[i].x * inv * ww.x, v[i].y * inv * ww.y);
                u.y = pack2<TO>(v[i].z * inv * ww.z, v[i].w * inv * ww.w);
                reinterpret_cast<uint2*>(orow)[c] = u;
            } else {
                reinterpret_cast<float4*>(orow)[c] =
                    make_float4(v[i].x * inv * ww.x, v[i].y * inv * ww.y, v[i].z * inv * ww.z,
                                v[i].w * inv * ww.w);
            }
        }
    }
    if (threadIdx.x == 0) tl_stamp(tl);
}

template <typename TO>
static int rmsnorm_dispatch(const float* x, const int* row_idx, const float* w, int M, int dim,
                            float eps, TO* out, cudaStream_t st, bool pdl, unsigned long long* tl) {
    const int nv = dim / 4;
    const int threads = nv >= 256 ? 256 : ((nv + 31) / 32) * 32;
    const int per = (nv + threads - 1) / threads;
    cudaError_t e;
    if (per <= 1)       e = launch_k(rmsnorm_kernel<TO, 1>, dim3(M), dim3(threads), 0, st, pdl, x, row_idx, w, dim, eps, out, tl);
    else if (per <= 2)  e = launch_k(rmsnorm_kernel<TO, 2>, dim3(M), dim3(threads), 0, st, pdl, x, row_idx, w, dim, eps, out, tl);
    else if (per <= 4)  e = launch_k(rmsnorm_kernel<TO, 4>, dim3(M), dim3(threads), 0, st, pdl, x, row_idx, w, dim, eps, out, tl);
    else if (per <= 8)  e = launch_k(rmsnorm_kernel<TO, 8>, dim3(M), dim3(threads), 0, st, pdl, x, row_idx, w, dim, eps, out, tl);
    else if (per <= 16) e = launch_k(rmsnorm_kernel<TO, 16>, dim3(M), dim3(threads), 0, st, pdl, x, row_idx, w, dim, eps, out, tl);
    else { set_error("rmsnorm: dim %d too large", dim); return LLAMA_ERR_INVALID_ARG; }
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "rmsnorm_kernel");
    return LLAMA_OK;
}

int launch_rmsnorm(const float* x, const int* row_idx, const float* w, int M, int dim, float eps,
                   void* out, int out_dtype, cudaStream_t st, bool pdl, unsigned long long* tl) {
    if (M <= 0) return LLAMA_OK;
    if (out_dtype == LLAMA_BF16)
        return rmsnorm_dispatch<bf16>(x, row_idx, w, M, dim, eps, static_cast<bf16*>(out), st, pdl, tl);
    if (out_dtype == LLAMA_F16)
        return rmsnorm_dispatch<f16>(x, row_idx, w, M, dim, eps, static_cast<f16*>(out), st, pdl, tl);
    return rmsnorm_dispatch<float>(x, row_idx, w, M, dim, eps, static_cast<float*>(out), st, pdl, tl);
}

// ---------------------------------------------------------------- w1/w3 interleave
// Copies w1 (which=0) or w3 (which=1) [H, dim] into the fused w13 matrix,
// whose rows are blocks of 16: block 2i holds w1 rows 16i..16i+15 and block
// 2i+1 the same w3 rows, so that a w1 row and its w3 row are 16 rows apart
// inside every 32-row group.  One CTA per source row, 16-byte copies.
__global__ void interleave_w13_kernel(const uint4* src, uint4* dst, int row_vecs, int which) {
    const int r = blockIdx.x;
    const int drow = (r / 16) * 32 + which * 16 + (r % 16);
    const uint4* s = src + static_cast<long long>(r) * row_vecs;
    uint4* d = dst + static_cast<long long>(drow) * row_vecs;
    for (int i = threadIdx.x; i < row_vecs; i += blockDim.x) d[i] = s[i];
}

int launch_copy_interleave_w13(const void* src, void* w13, int H, int dim, int which, int esz,
                               cudaStream_t st) {
    const int row_vecs = dim * esz / 16;
    interleave_w13_kernel<<<H, 128, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(w13),
                                             row_vecs, which);
    LLB_CHECK_LAUNCH("interleave_w13_kernel");
    return LLAMA_OK;
}

}  // namespace llb
