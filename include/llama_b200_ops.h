/*
 * llama_b200_ops.h — single-kernel entry points of libllama_b200.so.
 *
 * Each call runs one of the kernels the model path uses, on caller device
 * buffers, so that a kernel can be checked against the CPU oracle on its own
 * and timed in isolation.  Conventions (device pointers, void* stream,
 * LLAMA_OK / LLAMA_ERR_* return codes, llama_last_error) are those of
 * llama_b200.h.
 */
#ifndef LLAMA_B200_OPS_H
#define LLAMA_B200_OPS_H

#include <stddef.h>
#include <stdint.h>

#include "llama_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

/* RMSNorm of M rows: out[m,:] = x[m,:] / sqrt(mean(x[m,:]^2) + eps) * w
 * (Admin Guide §8.4, RMSNorm), fp32 arithmetic.
 *   x fp32 [M, dim]; w fp32 [dim]; out [M, dim] in out_dtype (LLAMA_F32,
 *   LLAMA_BF16 or LLAMA_F16, rounded once).  dim % 4 == 0. */
LLAMA_API int llama_op_rmsnorm(const float* x, const float* w, int M, int dim, float eps,
                     void* out, int out_dtype, void* stream);

/* Dense projection out[m,n] = sum_k A[m,k] * W[n,k]  (nn.Linear, y = x W^T).
 *   A [M, K] and W [N, K] in `dtype` (LLAMA_F32: SIMT fp32 FMA, no TF32;
 *   LLAMA_BF16 or LLAMA_F16: tcgen05 tensor cores, both operands of that
 *   type, fp32 accumulation in TMEM); out fp32 [M, N] (row-major,
 *   overwritten).  K % 8 == 0 for the 16-bit types; any other dtype code is
 *   LLAMA_ERR_INVALID_ARG.
 * The 16-bit kernels are the ones the model path uses: for M <= 64 the
 * persistent weight-streaming kernel (the weight is the 128-row MMA operand,
 * K split across CTAs), else the persistent 128 x 256-tile kernel.
 *   workspace  device scratch of llama_op_linear_workspace_bytes(), 256-byte
 *              aligned, zero-filled before its first use (the kernels leave
 *              their counters at zero again).  Required for the 16-bit
 *              types with M <= 64.  Optional for M > 64: with it the last
 *              wave of tiles is split along K over all SMs (stream-K), with
 *              NULL every tile runs whole.  A non-NULL workspace that is too small or
 *              misaligned is rejected (LLAMA_ERR_INVALID_ARG).  Calls sharing
 *              a workspace must not overlap on the device. */
LLAMA_API size_t llama_op_linear_workspace_bytes(void);
LLAMA_API int llama_op_linear(const void* A, const void* W, int M, int N, int K, int dtype,
                    float* out, void* workspace, size_t workspace_bytes, void* stream);

/* Allocation-free decode-shaped projection.  The source pages have no
 * counterpart: it exists for callers that cannot allocate device memory --
 * code running where cudaMalloc is not allowed (inside an allocator or memory
 * pool owned by someone else, a locked-down process, a plug-in that must not
 * touch the device heap) and so cannot provide the scratch workspace that
 * llama_op_linear needs.
 * Computes exactly what llama_op_linear computes for dtype LLAMA_BF16:
 *   out[m,n] = sum_k A[m,k] * W[n,k], A bf16 [M, K], W bf16 [N, K], out fp32
 *   [M, N] (device pointers owned by the caller), with the same persistent
 *   weight-streaming kernel, but its split-tile scratch is a fixed array in
 *   the library's device image (4 MiB + 16 KiB, held on every GPU that loads
 *   the library until the process exits).  Nothing is allocated on any call.
 * Limits: 1 <= M <= 16 token rows, N <= 4096 * 128, K a multiple of 8;
 *   larger M or N returns LLAMA_ERR_CAPACITY with a message.
 * The first call on a device, made with that device current, looks up the
 *   array's device address (a host-side symbol lookup); make that first call
 *   before any stream capture.  Every call clears the array's counters on
 *   `stream` before its kernel.
 * All calls share the one array: calls that overlap on the GPU (different
 *   streams, or threads without ordering) race and give wrong results. */
LLAMA_API int llama_op_linear_noalloc(const void* A, const void* W, int M, int N, int K, float* out,
                                      void* stream);

/* Per-launch timing of a model's projection kernels (for benchmarks).
 * llama_profile_start: from now on every projection launch the model enqueues
 *   (wq/wk/wv, wo, w1/w3, w2, output) is bracketed by two CUDA events recorded
 *   on the launch's own stream, for the first `capacity` launches.  Timed
 *   launches do not overlap their neighbours (no early launch).
 * llama_profile_stop: synchronises the events, writes up to `max` records
 *   (host arrays, any may be NULL): ms[i] = duration of launch i, bytes[i] =
 *   its algorithmic bytes (every weight once, the bf16 input rows once, the
 *   epilogue's outputs), flops[i] = 2*M*N*K summed over its projections,
 *   rows[i] = M; sets *n to the number of timed launches and stops timing.
 *   Events are created by start and destroyed by stop or llama_model_destroy. */
LLAMA_API int llama_profile_start(llama_model* m, int capacity);
LLAMA_API int llama_profile_stop(llama_model* m, float* ms, int64_t* bytes, int64_t* flops, int32_t* rows, int max,
                                 int* n);

/* Timeline of a model's decode steps (for benchmarks): where the time of a
 * step goes when its kernels overlap (programmatic dependent launch, CUDA
 * graph replay), which events between launches cannot show.
 * llama_timeline_start: zeroes the timeline on `stream` and, from now on,
 *   gives every kernel that llama_decode_step enqueues the next of up to 8192
 *   slots (embedding, RMSNorm, projection, attention, sampling launches).  A
 *   launch's CTAs leave in its slot the %globaltimer value (ns) at which the
 *   last of them finished (an atomic maximum), so launch i ran, exclusive of
 *   its predecessor, for end_ns[i] - end_ns[i-1].  A CUDA graph captured while
 *   the timeline records keeps its slots: each replay stamps them again
 *   (later replays leave later times).
 * llama_timeline_stop: stops giving out slots, synchronises the model's last
 *   stream and writes up to `max` records of the slots given out since the
 *   last start (host arrays, any may be NULL); it may be called again, e.g.
 *   after replaying a graph captured while recording, to read them anew:
 *   end_ns[i], kind[i] (LLAMA_TL_*), bytes[i] = the launch's algorithmic
 *   bytes where the host knows them (projections: every weight once, the
 *   16-bit input rows, the epilogue's outputs; embedding rows; sampling: the
 *   logits read), else 0; sets *n to the number of slots given out. */
#define LLAMA_TL_EMBED       0
#define LLAMA_TL_PROJECTION  1
#define LLAMA_TL_ATTENTION   2
#define LLAMA_TL_SAMPLE      3
#define LLAMA_TL_RMSNORM     4
LLAMA_API int llama_timeline_start(llama_model* m, void* stream);
LLAMA_API int llama_timeline_stop(llama_model* m, uint64_t* end_ns, int32_t* kind, int64_t* bytes, int max, int* n);

/* A stalled producer, for tests of the device-side timeout (failure
 * detection without a GPU fault).  Every wait of a kernel on another agent is
 * bounded; when one gives up, the kernel lets its own copies and tensor-core
 * operations in flight finish, releases its tensor memory, records
 * LLAMA_ERR_DEVICE_TIMEOUT in the model's device status word and returns.
 * llama_debug_stall arms that path once: in the next launch of the chosen
 * kernel by this model (16-bit models; LLAMA_STALL_PROJECTION: the next
 * projection, decode-shaped or prefill-shaped, on single SMs or CTA pairs;
 * LLAMA_STALL_ATTENTION: the next decode attention), CTA 0 never issues the
 * copies of pipeline stage `unit` of its run nor the barrier signal that
 * would announce them, and every wait of that launch gives up after wait_limit_ns
 * (1 us .. 2 s).  A unit past the end of CTA 0's run stalls nothing.  The
 * outputs of that step are unspecified; llama_model_status then returns the
 * timeout code and resets the model's internal counters, after which the next
 * call computes correctly.  LLAMA_STALL_NONE disarms a stall not yet taken. */
#define LLAMA_STALL_NONE        0
#define LLAMA_STALL_PROJECTION  1
#define LLAMA_STALL_ATTENTION   2
LLAMA_API int llama_debug_stall(llama_model* m, int which, int unit, int64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_B200_OPS_H */
