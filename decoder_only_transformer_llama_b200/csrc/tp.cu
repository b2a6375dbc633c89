// Tensor parallelism (Admin Guide §1.3 NOTE, §4.2 and §6.1; source tour, "One
// model.py"): every rank holds whole attention heads and whole SwiGLU
// features (column-parallel wq/wk/wv, w1/w3 and the vocabulary projection,
// row-parallel wo and w2), so wo and w2 leave per-rank partial sums of the
// residual update.  The reduce kernel adds them, in rank order, to each
// rank's copy of the residual stream -- every rank computes the same sums in
// the same order, so the copies stay identical -- and writes the next
// RMSNorm's inputs (the fused norm of the projections).  The gather kernel
// assembles the vocabulary slices of the logits.
//
// Ranks read each other's buffers directly (peer loads over NVLink; no TMA
// multicast, no library kernel on peer memory).  In a group whose ranks run
// on separate GPUs, a launch first announces its phase to every peer (a
// flag word in the peer's memory) and waits, bounded, until every peer has
// announced the same phase: the peers' partial sums of that phase are then
// complete.  Partial buffers alternate between two phases, and a rank can
// only overwrite the buffer of phase k after every peer has announced phase
// k + 1, i.e. finished reading phase k.  When one GPU runs every rank, stream
// order alone guarantees this and the handshake is skipped.
#include "common.cuh"
#include "model.h"

namespace llb {

struct TpParts {
    const float* p[kMaxTp];
};

// Thread 0 of a CTA: announce this launch's phase and wait for every peer's.
// Returns false when a wait ran out (the status word records it).
__device__ __forceinline__ bool tp_handshake(const TpSync& s, unsigned long long phase) {
    if (blockIdx.x == 0 && blockIdx.y == 0) {
        __threadfence_system();   // this rank's partial sums (written by the previous launch) before the flag
        for (int q = 0; q < s.size; ++q)
            *reinterpret_cast<volatile unsigned long long*>(s.peer_flags[q] + s.rank) = phase;
        __threadfence_system();
    }
    const uint64_t limit = s.wait_ns > 0 ? static_cast<uint64_t>(s.wait_ns) : kWaitLimitNs;
    for (int q = 0; q < s.size; ++q) {
        const volatile unsigned long long* f = s.my_flags + q;
        if (*f >= phase) continue;
        const uint64_t t0 = globaltimer_ns();
        while (*f < phase) {
            if (globaltimer_ns() - t0 > limit) {
                report_status(s.status, LLAMA_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
    __threadfence_system();
    return true;
}

// Thread 0 of a CTA, after its handshake: the launch's last CTA advances the
// rank's phase count.
__device__ __forceinline__ void tp_arrive(const TpSync& s, unsigned long long phase) {
    const int total = static_cast<int>(gridDim.x * gridDim.y);
    if (atomicAdd(s.arrivals, 1) == total - 1) {
        *s.epoch = phase;
        *s.arrivals = 0;
        __threadfence();
    }
}

template <typename T>
__global__ void __launch_bounds__(128)
tp_reduce_kernel(TpParts parts, int tp, float* __restrict__ x, int dim, const float* __restrict__ w_next,
                 T* __restrict__ y, float* __restrict__ ssq, TpSync sync) {
    __shared__ float red[4];
    __shared__ int ok_s;
    const int blk = blockIdx.x, m = blockIdx.y;
    if (sync.wait) {
        if (threadIdx.x == 0) {
            const unsigned long long phase = *reinterpret_cast<volatile unsigned long long*>(sync.epoch) + 1;
            ok_s = tp_handshake(sync, phase);
            tp_arrive(sync, phase);
        }
        __syncthreads();
        if (!ok_s) return;
    }
    const int f = blk * 128 + threadIdx.x;
    const long long i = static_cast<long long>(m) * dim + f;
    float v = x[i];
    for (int r = 0; r < tp; ++r) v += __ldcg(parts.p[r] + i);
    x[i] = v;
    y[i] = from_f32<T>(v * w_next[f]);
    float sq = warp_sum(v * v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sq;
    __syncthreads();
    if (threadIdx.x == 0) ssq[static_cast<long long>(m) * (dim / 128) + blk] = ((red[0] + red[1]) + red[2]) + red[3];
}

__global__ void __launch_bounds__(256)
tp_gather_kernel(TpParts slices, int tp, int rank, float* __restrict__ logits, int V, int Vl, TpSync sync) {
    __shared__ int ok_s;
    const int r = blockIdx.y;   // row
    if (sync.wait) {
        if (threadIdx.x == 0) {
            const unsigned long long phase = *reinterpret_cast<volatile unsigned long long*>(sync.epoch) + 1;
            ok_s = tp_handshake(sync, phase);
            tp_arrive(sync, phase);
        }
        __syncthreads();
        if (!ok_s) return;
    }
    for (int q = 0; q < tp; ++q) {
        if (q == rank) continue;
        const float* src = slices.p[q] + static_cast<long long>(r) * V + static_cast<long long>(q) * Vl;
        float* dst = logits + static_cast<long long>(r) * V + static_cast<long long>(q) * Vl;
        for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < Vl; j += gridDim.x * blockDim.x) dst[j] = __ldcg(src + j);
    }
}

int launch_tp_reduce(const Model* m, const float* const* parts, int M, const float* w_next, const TpSync& sync,
                     cudaStream_t st) {
    if (M <= 0) return LLAMA_OK;
    if (m->dim % 128 || m->tp_size < 1 || m->tp_size > kMaxTp) { set_error("tensor-parallel reduce: bad shape"); return LLAMA_ERR_INVALID_ARG; }
    TpParts p = {};
    for (int r = 0; r < m->tp_size; ++r) p.p[r] = parts[r];
    const dim3 grid(m->dim / 128, M);
    if (m->dtype == LLAMA_F16)
        tp_reduce_kernel<f16><<<grid, 128, 0, st>>>(p, m->tp_size, m->x, m->dim, w_next, static_cast<f16*>(m->y), m->ssq, sync);
    else
        tp_reduce_kernel<bf16><<<grid, 128, 0, st>>>(p, m->tp_size, m->x, m->dim, w_next, static_cast<bf16*>(m->y), m->ssq, sync);
    LLB_CHECK_LAUNCH("tp_reduce_kernel");
    return LLAMA_OK;
}

int launch_tp_gather_logits(const Model* m, float* logits, int rows, const TpSync& sync, cudaStream_t st) {
    if (rows <= 0) return LLAMA_OK;
    TpParts p = {};
    for (int r = 0; r < m->tp_size; ++r) p.p[r] = m->peers.logits[r];
    const dim3 grid((m->Vl + 255) / 256 < 8 ? (m->Vl + 255) / 256 : 8, rows);
    tp_gather_kernel<<<grid, 256, 0, st>>>(p, m->tp_size, m->tp_rank, logits, m->V, m->Vl, sync);
    LLB_CHECK_LAUNCH("tp_gather_kernel");
    return LLAMA_OK;
}

}  // namespace llb
