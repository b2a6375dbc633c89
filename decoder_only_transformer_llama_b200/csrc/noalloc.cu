// Allocation-free variant of the decode-shaped bf16 projection.
//
// Some callers cannot allocate device memory at all: code that runs where
// cudaMalloc is off limits (inside a memory-pool or arena owned by someone
// else, in a process whose allocator is locked down, or a plug-in that must
// not touch the device heap) still wants the weight-streaming projection.
// llama_op_linear needs a caller-provided scratch workspace for its split-tile
// partial sums and per-tile counters; this entry point takes that scratch from
// a fixed array in the library's own device image instead, so the caller
// passes only inputs and outputs and nothing is allocated on any call.
//
// The array lives for as long as the library is loaded on each device that
// uses it (every such GPU holds it until process exit), is shared by every
// call, and keeps the previous call's contents: the counters that must start
// at zero are cleared on the stream before each launch.  Calls that overlap on
// the GPU (on different streams, or on one device from several threads without
// ordering) race on the array and give wrong results.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "model.h"
#include "../../include/llama_b200_ops.h"

namespace llb {

namespace {
constexpr int kNoAllocMaxRows = 16;   // token rows (the 16-column MMA tile)
constexpr size_t kNoAllocPartBytes = static_cast<size_t>(kMaxDecodeCtas) * 2 * 128 * kNoAllocMaxRows * 4;
constexpr size_t kNoAllocCntBytes = static_cast<size_t>(kMaxTiles) * 4;
constexpr size_t kNoAllocBytes = kNoAllocPartBytes + kNoAllocCntBytes;   // 4 MiB + 16 KiB
constexpr int kMaxDevices = 64;
}  // namespace

// Scratch of the allocation-free projection: partials, then tile counters.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch on each device, looked up on the first
// call made with that device current (a host-side symbol lookup, no
// allocation).
static void* g_scratch_addr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

static int scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("device %d beyond the %d devices the allocation-free projection supports", dev, kMaxDevices);
        return LLAMA_ERR_INVALID_ARG;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return LLAMA_OK;
}

}  // namespace llb

using namespace llb;

extern "C" int llama_op_linear_noalloc(const void* A, const void* W, int M, int N, int K, float* out, void* stream) {
    if (!A || !W || !out) { set_error("A, W and out must be device pointers"); return LLAMA_ERR_INVALID_ARG; }
    if (M < 1 || M > kNoAllocMaxRows) {
        set_error("llama_op_linear_noalloc takes 1..%d token rows (M=%d); use llama_op_linear for more",
                  kNoAllocMaxRows, M);
        return LLAMA_ERR_CAPACITY;
    }
    if (N <= 0 || K <= 0 || K % 8) { set_error("N must be positive and K a positive multiple of 8"); return LLAMA_ERR_INVALID_ARG; }
    if ((N + 127) / 128 > kMaxTiles) {
        set_error("llama_op_linear_noalloc takes at most %d output rows (N=%d)", kMaxTiles * 128, N);
        return LLAMA_ERR_CAPACITY;
    }
    void* scratch = nullptr;
    const int rc = scratch_for_current_device(&scratch);
    if (rc != LLAMA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* part = static_cast<float*>(scratch);
    int* cnt = reinterpret_cast<int*>(static_cast<unsigned char*>(scratch) + kNoAllocPartBytes);
    // the tile counters start every call at zero, whatever the last call left
    cudaError_t e = cudaMemsetAsync(cnt, 0, kNoAllocCntBytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(noalloc counters)");
    TmaMaps ma, mw;
    int r2 = encode_kmajor_16(&ma.a128, A, M, K, 128);
    if (r2 == LLAMA_OK) r2 = encode_kmajor_16(&ma.b, A, M, K, 16);
    if (r2 == LLAMA_OK) r2 = encode_kmajor_16(&mw.a128, W, N, K, 128);
    if (r2 == LLAMA_OK) r2 = encode_kmajor_16(&mw.b, W, N, K, 256);
    if (r2 != LLAMA_OK) return r2;
    Epi ep;
    memset(&ep, 0, sizeof(ep));
    ep.mode = EPI_STORE_F32;
    ep.out = out;
    ep.ldo = N;
    return linear16_decode(&ma, &mw, M, N, K, LLAMA_BF16, ep, part, kNoAllocPartBytes, cnt, st, false);
}
