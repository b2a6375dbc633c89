/*
 * llama_b200.h — C ABI of the single-GPU Llama-2 decoder forward pass
 * (prefill and single-token decode over a preallocated KV cache, greedy and
 * top-p sampling) for NVIDIA B200 (sm_100a).
 *
 * What each call computes is defined by "Llama 2 Reference Implementation —
 * Administrator & Developer Guide" (meta-llama/llama @ 689c7f2):
 *   §3.3  ModelArgs (the structural configuration)
 *   §6.2  KV cache footprint (cache shape per layer)
 *   §8.4  The model architecture in detail (RMSNorm, RoPE, Attention with
 *         repeat_kv and the causal mask, SwiGLU FeedForward, pre-norm
 *         TransformerBlock, Transformer.forward)
 *   §8.5  The generation loop in detail (temperature softmax, top-p, argmax)
 * and the pyshine.com source tour of the same repository ("One model.py,
 * Four Ideas"; "Sampling, Stopping, and the Chat Template").
 *
 * Conventions shared by every entry point
 *   - Memory: every data pointer is a DEVICE pointer allocated by the caller,
 *     unless its comment says "host".  The library allocates no device memory:
 *     the model lives in one caller-owned arena (see llama_model_bytes).
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  Calls enqueue work and return; the library never
 *     synchronises the device except inside llama_model_status.
 *   - Errors: every call returns LLAMA_OK (0) or a LLAMA_ERR_* code and, on
 *     error, sets a thread-local message readable with llama_last_error().
 *     Argument errors are detected on the host before any work is enqueued.
 *     Errors that depend on device-resident values (a position past
 *     max_seq_len, a token id out of range, a wait that timed out) set the
 *     model's device status word instead; read it with llama_model_status.
 *   - Layouts: matrices are row-major [out_features, in_features] like
 *     nn.Linear (y = x W^T); RMSNorm weights are fp32; other weights are in
 *     the model dtype (fp32, bf16 or fp16).
 *   - Thread safety: calls on one model must be serialised by the caller
 *     (they share the model's workspace).
 *   - Devices: one CUDA device per process (one process per GPU).  The
 *     first launch of each kernel sets its shared-memory attributes and
 *     reads the SM count on the device current at that time, and later
 *     launches reuse them; a second device in the same process is not
 *     supported (its large-shared-memory launches may fail with
 *     LLAMA_ERR_CUDA).
 */
#ifndef LLAMA_B200_H
#define LLAMA_B200_H

#include <stddef.h>
#include <stdint.h>

/* Exported symbols keep default visibility in a library built with hidden visibility. */
#if defined(__GNUC__)
#define LLAMA_API __attribute__((visibility("default")))
#else
#define LLAMA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define LLAMA_OK                  0
#define LLAMA_ERR_INVALID_ARG     1  /* null pointer, bad size, unsupported shape   */
#define LLAMA_ERR_CAPACITY        2  /* batch / sequence / token budget exceeded    */
#define LLAMA_ERR_CUDA            3  /* a CUDA runtime call failed                  */
#define LLAMA_ERR_DEVICE_TIMEOUT  4  /* a bounded device-side wait gave up          */
#define LLAMA_ERR_TOKEN_RANGE     5  /* device status only: a token id outside [0,V) */

/* ---- dtypes --------------------------------------------------------------- */
#define LLAMA_F32   0   /* fp32 storage and fp32 arithmetic (no TF32)          */
#define LLAMA_BF16  1   /* bf16 storage, fp32 accumulation                     */
#define LLAMA_F16   2   /* fp16 storage (the reference's own dtype, Admin Guide
                           §1.4 and §6.4), fp32 accumulation; the bf16
                           kernels instantiated for fp16                    */

/*
 * Structural configuration: the fields of ModelArgs (Admin Guide §3.3) plus
 * the storage dtype and a per-call token budget.
 *   n_kv_heads          0 means n_heads (multi-head attention).
 *   ffn_dim_multiplier  <= 0 means "None".
 *   rope_theta          RoPE base (10000 for Llama 2, Admin Guide §8.4).
 *   max_tokens          most tokens one llama_prefill call may process summed
 *                       over its rows; 0 means max_batch_size * max_seq_len.
 * Limits of this implementation: head_dim = dim / n_heads must be 32, 64 or
 * 128; n_heads % n_kv_heads == 0; dim % 64 == 0; max_batch_size <= 256.
 */
typedef struct llama_model_args {
    int32_t dim;
    int32_t n_layers;
    int32_t n_heads;
    int32_t n_kv_heads;
    int32_t vocab_size;
    int32_t multiple_of;
    float   ffn_dim_multiplier;
    float   norm_eps;
    float   rope_theta;
    int32_t max_seq_len;
    int32_t max_batch_size;
    int32_t max_tokens;
    int32_t dtype;
} llama_model_args;

typedef struct llama_model llama_model;   /* opaque; host-side bookkeeping only */

/* Weight identifiers for llama_set_weight (names follow the reference modules). */
enum llama_weight_id {
    LLAMA_W_TOK_EMBEDDINGS = 0,  /* [vocab, dim]                     layer = -1 */
    LLAMA_W_NORM           = 1,  /* [dim] fp32, final RMSNorm        layer = -1 */
    LLAMA_W_OUTPUT         = 2,  /* [vocab, dim]                     layer = -1 */
    LLAMA_W_ATTENTION_NORM = 3,  /* [dim] fp32                                  */
    LLAMA_W_WQ             = 4,  /* [n_heads*head_dim, dim]                     */
    LLAMA_W_WK             = 5,  /* [n_kv_heads*head_dim, dim]                  */
    LLAMA_W_WV             = 6,  /* [n_kv_heads*head_dim, dim]                  */
    LLAMA_W_WO             = 7,  /* [dim, n_heads*head_dim]                     */
    LLAMA_W_FFN_NORM       = 8,  /* [dim] fp32                                  */
    LLAMA_W_W1             = 9,  /* [hidden, dim]                               */
    LLAMA_W_W2             = 10, /* [dim, hidden]                               */
    LLAMA_W_W3             = 11  /* [hidden, dim]                               */
};

/* Sampling parameters (Admin Guide §3.4 / §8.5): temperature == 0 selects the
 * greedy argmax; otherwise softmax(logits / temperature) and top-p. */
typedef struct llama_sampling {
    float temperature;
    float top_p;
} llama_sampling;

/* Derived sizes of a configuration (no GPU work).  `hidden` is the SwiGLU
 * width (Admin Guide §8.4: int(2*4*dim/3), times ffn_dim_multiplier, rounded
 * up to multiple_of).  Any output pointer may be NULL.
 * Returns LLAMA_ERR_INVALID_ARG for an unsupported configuration. */
LLAMA_API int llama_model_bytes(const llama_model_args* args, size_t* weight_bytes, size_t* kv_bytes,
                      size_t* workspace_bytes, size_t* total_bytes, int32_t* hidden);

/* Lays the model out in a caller-owned device arena of at least total_bytes
 * (256-byte aligned) and initialises it on `stream`: the KV cache is zeroed
 * (Admin Guide §8.4, Attention: caches start at zero) and the RoPE cos/sin
 * table is computed.  The arena stays owned by the caller; destroying the
 * model frees only the host-side handle.  Weights must then be uploaded with
 * llama_set_weight before the first forward call. */
LLAMA_API int llama_model_create(const llama_model_args* args, void* dev_arena, size_t arena_bytes,
                       void* stream, llama_model** out);

/* Copies one weight tensor from caller device memory `src` (row-major, shape
 * as listed in llama_weight_id, model dtype; fp32 for the three norms) into
 * the model's internal layout, on `stream`.  The source may be freed once
 * the stream has passed this call.  layer = -1 for the global weights. */
LLAMA_API int llama_set_weight(llama_model* m, int layer, int which, const void* src, void* stream);

/* Device address of layer `layer`'s K and V caches and their element strides
 * for the logical index [batch_row][position][kv_head][d] (Admin Guide §6.2
 * order); strides[0..3] receive those four strides in elements.  Used to fill
 * a cache before a decode-only benchmark and by tests. */
LLAMA_API int llama_get_kv(llama_model* m, int layer, void** k, void** v, int64_t strides[4]);

/* Prefill: Transformer.forward(tokens, start_pos) for B rows at once
 * (Admin Guide §8.4, "The forward pass").
 *   tokens      device int32 [B, T], row-major, right-padded
 *   lens        HOST int32 [B]: real tokens of each row (1..T); NULL = all T
 *   start_pos   first position of every row (cache rows 0..start_pos-1 must
 *               already hold earlier tokens of the same rows)
 *   logits      device fp32 output.  logits_mode 0: [B, vocab], the logits of
 *               each row's last real token.  logits_mode 1: [sum(lens), vocab],
 *               every real token's logits, rows packed in order.  May be NULL
 *               (mode 0 only) to only fill the cache.
 * Writes K/V of positions start_pos .. start_pos+lens[b]-1 of row b.
 * LLAMA_ERR_CAPACITY if B > max_batch_size, sum(lens) > max_tokens or
 * start_pos + T > max_seq_len. */
LLAMA_API int llama_prefill(llama_model* m, const int32_t* tokens, const int32_t* lens, int B, int T,
                  int start_pos, float* logits, int logits_mode, void* stream);

/* One decode step: a forward pass of one new token per row at per-row
 * positions, then sampling.  Everything per-step lives in device memory, so
 * a step can be captured in a CUDA graph and replayed.
 *   tokens      device int32 [B], the token at position pos[b] of row b
 *   pos         device int32 [B], its position (< max_seq_len; keys 0..pos[b]
 *               are attended).  pos[b] equal for all rows reproduces the
 *               reference's scalar start_pos exactly.
 *   sampling    host struct; NULL = compute logits only
 *   uniforms    device fp32 [B] in [0,1), one per row (top-p only)
 *   next_tokens device int32 [B] (may alias `tokens`); required if sampling
 *   logits      device fp32 [B, vocab] output, or NULL
 *   flags       LLAMA_DECODE_ADVANCE: after sampling, write next_tokens and
 *               increment pos[b] on the device (for graph replay loops)
 * A row with pos[b] outside [0, max_seq_len) is skipped (its outputs are
 * unspecified) and the device status word records LLAMA_ERR_CAPACITY.
 * 16-bit models run steps of up to 64 rows as a fused chain (RMSNorm folded
 * into the weight-streaming projections); wider steps (up to max_batch_size)
 * run one RMSNorm kernel per norm and the prefill projections; both compute
 * the same forward pass. */
#define LLAMA_DECODE_ADVANCE 1
LLAMA_API int llama_decode_step(llama_model* m, const int32_t* tokens, int32_t* pos, int B,
                      const llama_sampling* sampling, const float* uniforms,
                      int32_t* next_tokens, float* logits, int flags, void* stream);

/* Sampling alone, on caller logits (Admin Guide §8.5; source tour, sample_top_p):
 *   logits   device fp32 [B, V];  uniforms device fp32 [B] (ignored when
 *   temperature == 0);  out device int32 [B].
 * temperature == 0: argmax, lowest id on ties.  Otherwise, in fp64: p =
 * softmax(logits / temperature); tokens ordered by p descending (ties by id
 * ascending); token k kept iff the mass before it <= top_p; returns the first
 * kept token whose cumulative mass exceeds uniforms[b] * (kept mass), or the
 * last kept token.  Needs no model and no workspace. */
LLAMA_API int llama_sample(const float* logits, int B, int V, float temperature, float top_p,
                 const float* uniforms, int32_t* out, void* stream);

/* Log-probabilities of given tokens under their logits rows: the per-token
 * logprobs that the generation loop returns (Admin Guide §8.5, generate with
 * logprobs=True):
 *   logits  device fp32 [N, V], row i the model's logits predicting token i;
 *   tokens  device int32 [N];  out  device fp32 [N], written
 *   out[i] = logits[i, t] - (m + log sum_j exp(logits[i, j] - m)),
 *   t = tokens[i], m = max_j logits[i, j], the sum in fp64.
 * A token outside [0, V) gives NaN.  N == 0 is a no-op.  Needs no model.
 * LLAMA_ERR_INVALID_ARG for NULL pointers, N < 0 or V <= 0. */
LLAMA_API int llama_token_logprobs(const float* logits, const int32_t* tokens, int N, int V, float* out,
                                   void* stream);

/* Copies the device status word to *device_status (synchronous on the model's
 * last stream) and clears it.  0 = no device-side error since the last read.
 * After a non-zero status it also resets the model's internal arrival
 * counters (a kernel that gave up on a wait leaves them part-counted), so the
 * next call computes correctly; read the status after any call whose result
 * is in doubt. */
LLAMA_API int llama_model_status(llama_model* m, int* device_status);

/* ---- tensor parallelism --------------------------------------------------
 * The reference's model-parallel layout (Admin Guide §1.3 NOTE on fairscale,
 * §4.2 "Single-host, multi-GPU", §6.1 "Hot path"; source tour, "One model.py"):
 * rank r of tp_size ranks holds query heads [r*nh/tp, (r+1)*nh/tp) with their
 * KV heads [r*nkv/tp, (r+1)*nkv/tp) (rows of wq, wk, wv; columns of wo), FFN
 * features [r*H/tp, (r+1)*H/tp) (rows of w1, w3; columns of w2), vocabulary
 * rows [r*V/tp, (r+1)*V/tp) of the output projection, and whole copies of the
 * token embedding and the three RMSNorm weights.  wo and w2 leave partial
 * residual updates; each rank adds every rank's update, in rank order, to its
 * own copy of the residual stream (two reductions per layer), so the copies
 * stay identical; the logits slices are gathered.  16-bit models only;
 * n_heads, n_kv_heads, vocab_size and the FFN width (in multiples of 64) must
 * split evenly.  Weights are uploaded with llama_set_weight in their shard
 * shapes ([nh/tp*hd, dim] for wq, [dim, nh/tp*hd] for wo, [V/tp, dim] for
 * output, ...).
 *
 * llama_model_bytes_tp / llama_model_create_tp: as llama_model_bytes /
 *   llama_model_create for shard tp_rank of tp_size (1 <= tp_size <= 8).
 * llama_tp_prefill_all / llama_tp_decode_step_all: one GPU runs every rank
 *   (shards[r] = rank r, all on this device): the calls of llama_prefill /
 *   llama_decode_step for the whole group, phase by phase on `stream`, each
 *   rank reading the others' partial sums directly; `logits` ([rows, V], or
 *   NULL) receives every rank's slice.  Used to check the sharded forward
 *   pass against the unsharded one.
 * llama_tp_buffers / llama_tp_bind: ranks on separate GPUs (one process per
 *   GPU).  Each rank publishes its two partial-sum buffers, its flag words and
 *   its logits buffer (device addresses; share them through CUDA IPC), and
 *   binds the table of every rank's buffers, mapped into its own address
 *   space (indexed by rank, its own included).  After that, llama_prefill
 *   (logits_mode 0) and llama_decode_step on each rank's shard run the
 *   group's forward pass: every reduction first announces its phase in every
 *   peer's flag words and waits (bounded, LLAMA_ERR_DEVICE_TIMEOUT) until all
 *   ranks announced it, then reads the peers' partial sums over NVLink (plain
 *   peer loads).  Every rank must make the same sequence of calls. */
LLAMA_API int llama_model_bytes_tp(const llama_model_args* args, int tp_rank, int tp_size, size_t* weight_bytes,
                                   size_t* kv_bytes, size_t* workspace_bytes, size_t* total_bytes, int32_t* hidden);
LLAMA_API int llama_model_create_tp(const llama_model_args* args, int tp_rank, int tp_size, void* dev_arena,
                                    size_t arena_bytes, void* stream, llama_model** out);
LLAMA_API int llama_tp_prefill_all(llama_model* const* shards, int tp, const int32_t* tokens, const int32_t* lens,
                                   int B, int T, int start_pos, float* logits, int logits_mode, void* stream);
LLAMA_API int llama_tp_decode_step_all(llama_model* const* shards, int tp, const int32_t* tokens, int32_t* pos, int B,
                                       const llama_sampling* sampling, const float* uniforms, int32_t* next_tokens,
                                       float* logits, int flags, void* stream);
LLAMA_API int llama_tp_buffers(llama_model* m, float** part0, float** part1, unsigned long long** flags,
                               float** logits);
LLAMA_API int llama_tp_bind(llama_model* m, float* const* part0, float* const* part1,
                            unsigned long long* const* flags, float* const* logits);

/* Frees the host handle; the arena and everything in it stay with the caller. */
LLAMA_API int llama_model_destroy(llama_model* m);

/* Message for the last non-zero status returned on this thread ("" if none). */
LLAMA_API const char* llama_last_error(void);

/* Number of kernel launches this library has enqueued since load (all
 * models, all threads); used to report how many of this library's kernels ran
 * in a timed region.  A launch captured into a CUDA graph counts once, when
 * captured. */
LLAMA_API uint64_t llama_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_B200_H */
