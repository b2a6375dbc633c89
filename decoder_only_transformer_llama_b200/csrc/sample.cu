// Next-token selection (Admin Guide §6.3 and §8.5; source tour, sample_top_p).
//
// Greedy: argmax over the vocabulary, lowest id on ties.
//
// Top-p: p = softmax(l / T); tokens ordered by p descending, ties by id
// ascending; token k is kept iff the mass before it is <= top_p; the draw is
// the first kept token whose cumulative mass exceeds u * (kept mass).
// The reference sorts the whole vocabulary; here one CTA per row finds the
// two tokens that matter (the last kept one and the drawn one) without a
// sort, by a most-significant-digit radix select over a 64-bit order key
//     key = ordered_bits(logit) << 32 | ~id      (descending key = sampling order)
// using histograms of probability mass.  Masses are e_i = exp((l_i - l_max)/T)
// evaluated in fp64 and held as 64-bit fixed point (2^-46 resolution), so
// every prefix sum is an exact integer and the result does not depend on the
// summation order.
#include "common.cuh"
#include "model.h"

namespace llb {

namespace {
constexpr int kSampleThreads = 1024;
constexpr int kWarps = kSampleThreads / 32;
constexpr double kFixScale = 70368744177664.0;    // 2^46: V * 2^46 < 2^64 for V <= 262144
}

__device__ __forceinline__ uint32_t ordered_bits(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t sort_key(float l, int id) {
    return (static_cast<uint64_t>(ordered_bits(l)) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(id));
}

// ---------------------------------------------------------------- argmax
__global__ void __launch_bounds__(kSampleThreads)
argmax_kernel(const float* __restrict__ logits, int V, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
              unsigned long long* tl) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const float* row = logits + static_cast<long long>(b) * V;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
        const float v = row[i];
        if (v > best || (v == best && i < bi)) { best = v; bi = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
    }
    __shared__ float sv[kWarps];
    __shared__ int si[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { sv[warp] = best; si[warp] = bi; }
    __syncthreads();
    if (warp == 0) {
        best = lane < (blockDim.x >> 5) ? sv[lane] : -INFINITY;
        bi = lane < (blockDim.x >> 5) ? si[lane] : 0x7fffffff;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
        }
        if (lane == 0) {
            if (bi == 0x7fffffff) bi = 0;   // all NaN: token 0
            out[b] = bi;
            if (tokens_adv) tokens_adv[b] = bi;
            if (pos_adv) pos_adv[b] += 1;
            tl_stamp(tl);
        }
    }
}

// ---------------------------------------------------------------- top-p
struct TopPShared {
    unsigned long long hist_mass[kWarps][256];
    unsigned int hist_cnt[kWarps][256];
    unsigned long long tot_mass[256];
    unsigned int tot_cnt[256];
    unsigned long long red_u64[kWarps];
    float red_f[kWarps];
    unsigned long long sel_prefix, sel_before;
    unsigned long long result_key[2], result_before[2];
    float lmax;
};

__device__ __forceinline__ unsigned long long fixed_mass(float l, double lmax, double inv_t) {
    const double e = exp((static_cast<double>(l) - lmax) * inv_t);
    return static_cast<unsigned long long>(e * kFixScale + 0.5);
}

// First key in descending order whose inclusive prefix mass exceeds `target`
// (or the smallest key if none does).  Returns the key; *before_out = mass of
// all keys strictly before it.
__device__ uint64_t radix_select(TopPShared& sh, const float* row, int V, double lmax, double inv_t,
                                 unsigned long long target, unsigned long long* before_out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t prefix = 0, mask = 0;
    unsigned long long before = 0;
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int i = lane; i < 256; i += 32) {
            sh.hist_mass[warp][i] = 0ull;
            sh.hist_cnt[warp][i] = 0u;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < V; i += blockDim.x) {
            const float l = row[i];
            const uint64_t key = sort_key(l, i);
            if ((key & mask) == prefix) {
                const int bin = static_cast<int>((key >> shift) & 255u);
                atomicAdd(&sh.hist_mass[warp][bin], fixed_mass(l, lmax, inv_t));
                atomicAdd(&sh.hist_cnt[warp][bin], 1u);
            }
        }
        __syncthreads();
        if (threadIdx.x < 256) {
            unsigned long long m = 0;
            unsigned int c = 0;
            for (int w = 0; w < kWarps; ++w) {
                m += sh.hist_mass[w][threadIdx.x];
                c += sh.hist_cnt[w][threadIdx.x];
            }
            sh.tot_mass[threadIdx.x] = m;
            sh.tot_cnt[threadIdx.x] = c;
        }
        __syncthreads();
        if (warp == 0) {
            // lane L scans bins 255-8L .. 248-8L (descending)
            unsigned long long part = 0;
            for (int k = 0; k < 8; ++k) part += sh.tot_mass[255 - 8 * lane - k];
            // exclusive scan from lane 0 (highest bins) upwards
            unsigned long long incl = part;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const unsigned long long excl = incl - part;
            const bool cross = before + incl > target;
            const unsigned int ballot = __ballot_sync(0xffffffffu, cross);
            int chosen = -1;
            unsigned long long chosen_before = 0;
            if (ballot) {
                const int L = __ffs(ballot) - 1;
                if (lane == L) {
                    unsigned long long cum = before + excl;
                    for (int k = 0; k < 8; ++k) {
                        const int bin = 255 - 8 * lane - k;
                        if (sh.tot_cnt[bin] == 0) continue;
                        if (cum + sh.tot_mass[bin] > target) { chosen = bin; chosen_before = cum; break; }
                        cum += sh.tot_mass[bin];
                    }
                }
                chosen = __shfl_sync(0xffffffffu, chosen, L);
                chosen_before = __shfl_sync(0xffffffffu, chosen_before, L);
            }
            if (chosen < 0) {
                // no bin crosses: take the lowest non-empty bin (the last key in order)
                if (lane == 0) {
                    unsigned long long cum = before;
                    for (int bin = 255; bin >= 0; --bin) {
                        if (sh.tot_cnt[bin] == 0) continue;
                        chosen = bin;
                        chosen_before = cum;
                        cum += sh.tot_mass[bin];
                    }
                }
                chosen = __shfl_sync(0xffffffffu, chosen, 0);
                chosen_before = __shfl_sync(0xffffffffu, chosen_before, 0);
            }
            if (lane == 0) {
                sh.sel_prefix = prefix | (static_cast<uint64_t>(chosen) << shift);
                sh.sel_before = chosen_before;
            }
        }
        __syncthreads();
        prefix = sh.sel_prefix;
        before = sh.sel_before;
        mask |= static_cast<uint64_t>(255) << shift;
        __syncthreads();
    }
    *before_out = before;
    return prefix;
}

__global__ void __launch_bounds__(kSampleThreads)
top_p_kernel(const float* __restrict__ logits, int V, float temperature, float top_p,
             const float* __restrict__ uniforms, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
             unsigned long long* tl) {
    extern __shared__ uint8_t smem_raw[];
    TopPShared& sh = *reinterpret_cast<TopPShared*>(smem_raw);
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* row = logits + static_cast<long long>(b) * V;

    // max logit
    float mx = -INFINITY;
    for (int i = threadIdx.x; i < V; i += blockDim.x) mx = fmaxf(mx, row[i]);
    mx = warp_max(mx);
    if (lane == 0) sh.red_f[warp] = mx;
    __syncthreads();
    if (warp == 0) {
        float t = lane < kWarps ? sh.red_f[lane] : -INFINITY;
        t = warp_max(t);
        if (lane == 0) sh.lmax = t;
    }
    __syncthreads();
    const double lmax = static_cast<double>(sh.lmax);
    const double inv_t = 1.0 / static_cast<double>(temperature);

    // total mass
    unsigned long long tot = 0;
    for (int i = threadIdx.x; i < V; i += blockDim.x) tot += fixed_mass(row[i], lmax, inv_t);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if (lane == 0) sh.red_u64[warp] = tot;
    __syncthreads();
    unsigned long long S = 0;
    for (int w = 0; w < kWarps; ++w) S += sh.red_u64[w];

    // nucleus edge: first key whose inclusive mass exceeds top_p * S
    const double tp = static_cast<double>(top_p) * static_cast<double>(S);
    const unsigned long long t1 = tp >= 18446744073709549568.0 ? ~0ull : static_cast<unsigned long long>(tp);
    unsigned long long before_edge;
    const uint64_t edge = radix_select(sh, row, V, lmax, inv_t, t1, &before_edge);
    const int edge_id = static_cast<int>(~static_cast<uint32_t>(edge & 0xffffffffu));
    const unsigned long long Z = before_edge + fixed_mass(row[edge_id], lmax, inv_t);

    // draw: first kept key whose inclusive mass exceeds u * Z
    double u = static_cast<double>(uniforms[b]);
    u = fmin(fmax(u, 0.0), 1.0);
    const unsigned long long t2 = static_cast<unsigned long long>(u * static_cast<double>(Z));
    unsigned long long before_draw;
    const uint64_t drawn = radix_select(sh, row, V, lmax, inv_t, t2, &before_draw);
    const uint64_t pick = drawn < edge ? edge : drawn;   // never past the nucleus edge
    if (threadIdx.x == 0) {
        const int id = static_cast<int>(~static_cast<uint32_t>(pick & 0xffffffffu));
        out[b] = id;
        if (tokens_adv) tokens_adv[b] = id;
        if (pos_adv) pos_adv[b] += 1;
        tl_stamp(tl);
    }
}

// ---------------------------------------------------------------- token log-probabilities
// out[i] = log softmax(logits[i, :])[tok[i]] = l[tok] - (m + log sum_j exp(l_j - m)),
// m = max_j l_j, the sum in fp64 (the log-probabilities that generate returns,
// Admin Guide §8.5).  An id outside [0, V) gives NaN.
__global__ void __launch_bounds__(kSampleThreads)
logprob_kernel(const float* __restrict__ logits, const int32_t* __restrict__ tok, int V, float* __restrict__ out) {
    __shared__ float s_max[kWarps];
    __shared__ double s_sum[kWarps];
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* row = logits + static_cast<long long>(i) * V;
    float mx = -INFINITY;
    for (int j = threadIdx.x; j < V; j += blockDim.x) mx = fmaxf(mx, row[j]);
    mx = warp_max(mx);
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
    mx = s_max[0];
    for (int w = 1; w < kWarps; ++w) mx = fmaxf(mx, s_max[w]);
    const double m = static_cast<double>(mx);
    double sum = 0.0;
    for (int j = threadIdx.x; j < V; j += blockDim.x) sum += exp(static_cast<double>(row[j]) - m);
    sum = warp_sum_d(sum);
    if (lane == 0) s_sum[warp] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        double total = 0.0;
        for (int w = 0; w < kWarps; ++w) total += s_sum[w];
        const int t = tok[i];
        out[i] = (t >= 0 && t < V) ? static_cast<float>(static_cast<double>(row[t]) - m - log(total)) : NAN;
    }
}

int launch_logprobs(const float* logits, const int32_t* tokens, int N, int V, float* out, cudaStream_t st) {
    logprob_kernel<<<N, kSampleThreads, 0, st>>>(logits, tokens, V, out);
    LLB_CHECK_LAUNCH("logprob_kernel");
    return LLAMA_OK;
}

int launch_argmax(const float* logits, int B, int V, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
                  cudaStream_t st, bool pdl, unsigned long long* tl) {
    static bool attr = false;
    if (!attr) {
        cudaError_t ce = carveout_max(argmax_kernel);
        if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(argmax_kernel)");
        attr = true;
    }
    cudaError_t e = launch_k(argmax_kernel, dim3(B), dim3(kSampleThreads), 0, st, pdl, logits, V, out, tokens_adv,
                             pos_adv, tl);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "argmax_kernel");
    return LLAMA_OK;
}

int launch_top_p(const float* logits, int B, int V, float temperature, float top_p, const float* uniforms,
                 int32_t* out, int32_t* tokens_adv, int32_t* pos_adv, cudaStream_t st, bool pdl,
                 unsigned long long* tl) {
    const int smem = static_cast<int>(sizeof(TopPShared));
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(top_p_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess) e = carveout_max(top_p_kernel);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(top_p_kernel)");
        attr = true;
    }
    cudaError_t e = launch_k(top_p_kernel, dim3(B), dim3(kSampleThreads), smem, st, pdl, logits, V, temperature,
                             top_p, uniforms, out, tokens_adv, pos_adv, tl);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "top_p_kernel");
    return LLAMA_OK;
}

}  // namespace llb
