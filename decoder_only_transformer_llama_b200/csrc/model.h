// Host-side model description and the internal launchers shared by the
// C-ABI implementation (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <vector>

#include "../../include/llama_b200.h"

namespace llb {

constexpr int kMaxRows = 256;         // max_batch_size limit (by-value row tables)
constexpr int kChunk = 64;            // keys per chunk in decode attention
constexpr int kMaxDecodeCtas = 512;   // persistent CTAs of the decode projection kernel (two per SM)
constexpr int kMaxPrefillCtas = 256;  // persistent CTAs of the prefill projection kernel (one per SM)
// fp32 partials of split tiles, two per persistent CTA: 128 x 64 blocks in the
// decode projection, 128 x 256 tiles in the prefill projection
constexpr size_t kDecodePartBytes = static_cast<size_t>(kMaxDecodeCtas) * 2 * 128 * 64 * 4;
constexpr size_t kPrefillPartBytes = static_cast<size_t>(kMaxPrefillCtas) * 2 * 128 * 256 * 4;
constexpr size_t kGemmPartBytes = kPrefillPartBytes > kDecodePartBytes ? kPrefillPartBytes : kDecodePartBytes;
constexpr int kMaxTiles = 4096;       // tile counters: N / 128 of the widest projection
constexpr int kMaxAttnCtas = 1024;    // persistent CTAs of the decode attention kernel
constexpr int kTimelineCap = 8192;    // launches one timeline can stamp
constexpr int kStepCounters = 4;      // per-step finish counters
constexpr int kMaxTp = 8;             // tensor-parallel ranks of one model

// Tensor parallelism: the buffers of every rank of a group, as device
// addresses this GPU can read (its own, or peers' through NVLink / P2P).
struct TpPeers {
    float* part[kMaxTp][2];               // fp32 partial residual updates (wo / w2), by phase parity
    unsigned long long* flag[kMaxTp];     // flag words: flag[q][r] = last phase rank r announced to rank q
    float* logits[kMaxTp];                // each rank's logits buffer [Bmax][V]
};

// Cross-rank handshake of one reduce or gather launch (multi-GPU groups only).
struct TpSync {
    int wait;                             // 0: every rank's data is ready by stream order (one GPU)
    int rank, size;
    unsigned long long* my_flags;         // [kMaxTp] this rank's flag words
    unsigned long long* peer_flags[kMaxTp];
    unsigned long long* epoch;            // this rank's count of completed handshakes
    int* arrivals;                        // CTAs of the launch that passed the handshake
    int* status;
    long long wait_ns;
};

// Token -> (batch row, position) map of one prefill call, passed by value.
struct RowTable {
    int B, T, start_pos;
    int cu[kMaxRows + 1];    // packed token offsets of each row
};

// Epilogue of a projection: what happens to acc[m, n] = sum_k A[m,k] W[n,k].
enum EpiMode { EPI_STORE_F32 = 0, EPI_RESID_F32 = 1, EPI_QKV = 2, EPI_SWIGLU = 3, EPI_LOGITS_ARGMAX = 4 };

struct Epi {
    int mode;
    // STORE_F32: out[m*ldo + n] = acc.  RESID_F32: out[m*ldo + n] += acc.
    float* out;
    int ldo;
    // QKV: columns [0, nq) -> q[m*nq + n] (RoPE), [nq, nq+nkvc) -> K cache (RoPE),
    // [nq+nkvc, nq+2*nkvc) -> V cache; token m sits in batch row tok_row[m]
    // (identity when NULL) at position tok_pos[m].
    void* q;
    void* kc;
    void* vc;
    const int* tok_row;
    const int* tok_pos;
    int nq, nkvc, hd, max_seq;
    long long kv_row_stride;   // elements between batch rows of one layer's cache
    const float2* rope;        // [max_seq][hd/2] (cos, sin)
    // SWIGLU: interleaved columns (16 w1 rows, then the same 16 w3 rows, ...)
    // -> g[m*H + h] = silu(w1) * w3.
    void* g;
    int H;
    int* status;
    // Timeline slot of this launch (see Model::tl_end), or null.
    unsigned long long* tl;
    // LOGITS_ARGMAX (decode projection only): out[m*ldo + n] = acc if out is
    // not null, and the greedy pick of every token row m: best[m] collects the
    // largest key (ordered logit bits << 32 | ~n, so equal logits keep the
    // lowest id); the CTA that finishes last (done counter) writes
    // next[m] = its id, tok_adv[m] = id and ++pos_adv[m] where those are not
    // null, and leaves best[] and the counter at zero again.
    unsigned long long* best;
    int* done;
    int32_t* next;
    int32_t* tok_adv;
    int32_t* pos_adv;
    // Decode projection only: every wait gives up after wait_ns (0 = the
    // default limit); stall = u + 1 (tests of the timeout path) makes CTA 0
    // issue neither the copies nor the barrier signal of ring stage u
    // (0 = no stall, the value of a zero-initialised Epi).
    long long wait_ns;
    int stall;
};

// RMSNorm folded into the decode projections (bf16 decode chain), using
// norm(x) W^T = r_b * ((x * w) W^T) with r_b = 1/sqrt(mean(x_b^2) + eps):
//   producer side (residual epilogue of wo / w2, and the embedding): besides
//     x it writes y_out[b, n] = bf16(x[b, n] * w_next[n]) -- the operand of the
//     next projection, w_next the weight of the norm in front of it -- and
//     ssq_out[b * n_tiles + t] = sum of x^2 over the 128 features of tile t;
//   consumer side (wq/wk/wv, w1/w3, output): multiplies accumulator column b
//     by r_b = 1/sqrt(sum_t ssq_in[b * n_in + t] / K + eps) before its epilogue.
// Null pointers switch either side off.
struct NormIO {
    const float* ssq_in;
    int n_in;
    float eps;
    float* ssq_out;
    void* y_out;
    const float* w_next;
};

struct TmaMaps {               // tensor maps of one K-major bf16 matrix
    CUtensorMap a128;          // box 64 x 128 rows (the MMA's A operand)
    CUtensorMap b;             // box 64 x 256 rows (weights as B) or 64 x 16 (activations as B)
};

struct LayerPtrs {
    float* attn_norm;
    void* wqkv;
    void* wo;
    float* ffn_norm;
    void* w13;   // interleaved in blocks of 16 rows: w1[0:16], w3[0:16], w1[16:32], ...
    void* w2;
    TmaMaps m_wqkv, m_wo, m_w13, m_w2;
};

struct Profile {
    int capacity = 0;
    int n = 0;
    std::vector<cudaEvent_t> ev;     // 2 per launch
    std::vector<int64_t> bytes;      // algorithmic bytes per launch
    std::vector<int64_t> flops;      // flops per launch
    std::vector<int32_t> rows;       // token rows (M) per launch
};

// Kinds of launches a timeline records (the LLAMA_TL_* codes of llama_b200_ops.h).
enum TlKind { TL_EMBED = 0, TL_PROJECTION = 1, TL_ATTENTION = 2, TL_SAMPLE = 3, TL_RMSNORM = 4 };

struct Model {
    llama_model_args a;
    int dim, L, nh, nkv, hd, n_rep, H, V, S, Bmax, Mmax, dtype, esz;
    int nq, nkvc, nqkv;
    int n_splits;
    // weights
    void* tok_emb;
    float* norm;
    void* output;
    TmaMaps m_output;
    std::vector<LayerPtrs> layers;
    // KV cache: [L][Bmax][nkv][S][hd]
    void* kc;
    void* vc;
    long long kv_layer_elems, kv_row_elems, kv_head_elems;
    float2* rope;
    // workspace
    float* x;        // [Mmax, dim] fp32 residual stream
    void* y;         // [Mmax, dim] normed activations (model dtype)
    void* q;         // [Mmax, nq]
    void* attn;      // [Mmax, nq]
    void* g;         // [Mmax, H]
    void* ylast;     // [Bmax, dim] final-norm rows that get logits
    int* tok_ids;    // [Mmax]
    int* tok_row;    // [Mmax]
    int* tok_pos;    // [Mmax]
    int* last_idx;   // [Bmax]
    float* logits_ws;   // [Bmax, V]
    float* part_o;      // [2 * kMaxAttnCtas * n_rep, hd] split partials of decode attention
    float* part_ml;     // [2 * kMaxAttnCtas * n_rep, 2]
    int* attn_cnt;      // [Bmax*nkv] split arrival counters (zero between launches)
    float* gemm_part;   // split-tile partials of the decode projection kernel
    int* gemm_cnt;      // per-tile arrival counters (zero between launches)
    float* ssq;         // [Bmax, dim/128] per-tile sums of x^2 for the fused RMSNorm
    unsigned long long* best;   // [Bmax] greedy-pick keys of the fused output projection (zero between steps)
    int* step_cnt;      // [kStepCounters] finish counters of the fused greedy pick (zero between steps)
    int* status;
    TmaMaps m_y, m_attn, m_g, m_ylast;   // activation maps (A box 128 rows, B box 16 rows)
    // Tensor-memory prefill attention (16-bit, head_dim 128): q as [rows][nq]
    // and every layer's K and V caches as [L * Bmax * nkv * S][hd], boxes of
    // 64 columns x 128 rows.
    CUtensorMap m_qtile, m_kcache, m_vcache;
    bool has_attn_maps = false;
    // the same caches in 64-key x 64-dim boxes (decode attention on the tensor cores)
    CUtensorMap m_kdec, m_vdec;
    bool has_dec_maps = false;
    cudaStream_t last_stream;
    Profile prof;
    // Timeline of decode launches: while tl_on, launch i of llama_decode_step
    // is given slot tl_end + i, where its CTAs leave the %globaltimer value
    // (ns) at which the last of them finished (atomicMax).
    unsigned long long* tl_end;
    // One-shot stall for tests of the device timeout (llama_debug_stall): the
    // next launch of the chosen kernel gets it, then it is cleared.
    // tensor parallelism: this shard's rank and group size, its vocabulary
    // slice, its double-buffered partial sums, flag words and handshake
    // counters, and every rank's buffers once bound
    int tp_rank = 0, tp_size = 1, Vl = 0;
    float* tp_part[2] = {nullptr, nullptr};
    unsigned long long* tp_flag = nullptr;     // [kMaxTp]
    unsigned long long* tp_epoch = nullptr;
    int* tp_arrivals = nullptr;
    TpPeers peers = {};
    bool tp_bound = false, tp_wait = false;
    int dbg_kind = 0;          // 0 none, LLAMA_STALL_PROJECTION or LLAMA_STALL_ATTENTION
    int dbg_unit = -1;
    long long dbg_wait_ns = 0;
    bool tl_on = false;
    int tl_n = 0;
    std::vector<int> tl_kind;
    std::vector<int64_t> tl_bytes;
};

// Next timeline slot of `m` for a launch of `kind` moving `bytes` algorithmic
// bytes, or null when no timeline is recording (or it is full).
unsigned long long* tl_next(Model* m, int kind, int64_t bytes);

// ---------------------------------------------------------------- launchers (return LLAMA_* codes)
int launch_rope_table(float2* rope, int S, int hd, float theta, cudaStream_t st);
int launch_token_map(const RowTable& rt, const int32_t* tokens, int* tok_ids, int* tok_row,
                     int* tok_pos, int* last_idx, cudaStream_t st);
// `pdl`: launch as part of the decode chain (may start before its predecessor ends).
// With `ssq`, also writes the sum of x^2 of every 128-feature block and
// y = bf16(x * w_next) (the fused RMSNorm's producer side, see NormIO).
int launch_embed(const int* tok_ids, const void* emb, int dtype, int M, int dim, int V, float* x,
                 int* status, cudaStream_t st, bool pdl = false, float* ssq = nullptr, void* y = nullptr,
                 const float* w_next = nullptr, unsigned long long* tl = nullptr);
int launch_rmsnorm(const float* x, const int* row_idx, const float* w, int M, int dim, float eps,
                   void* out, int out_dtype, cudaStream_t st, bool pdl = false, unsigned long long* tl = nullptr);
int launch_copy_interleave_w13(const void* src, void* w13, int H, int dim, int which, int esz,
                               cudaStream_t st);

// out = A W^T with epilogue `ep`.  A rows: M (tokens), W rows: N, K.
// 16-bit dtypes use tcgen05 with the given maps (A-side/W-side), fp32 the SIMT kernel.
// With `stamp`, the launch takes the next timeline slot (see Model::tl_end).
int run_linear(const Model* m, int dtype, const void* A, const TmaMaps* mapA, const void* W,
               const TmaMaps* mapW, int M, int N, int K, const Epi& ep, cudaStream_t st, bool pdl = false,
               const NormIO* nio = nullptr, bool stamp = false);
int linear_f32(const float* A, const float* W, int M, int N, int K, const Epi& ep, cudaStream_t st);
// Prefill-shaped projection; with part/counters (kGemmPartBytes, kMaxTiles
// zeroed ints) the tail wave is split stream-K, without them whole tiles only.
int linear16_tc(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, int dtype, const Epi& ep, float* part,
                int* counters, cudaStream_t st, const NormIO* nio = nullptr);
int linear16_decode(const TmaMaps* mapX, const TmaMaps* mapW, int M, int N, int K, int dtype, const Epi& ep, float* part,
                    size_t part_bytes, int* counters, cudaStream_t st, bool pdl, const NormIO* nio = nullptr);
// 16-bit projection: M <= 64 token rows -> linear16_decode, else linear16_tc.
int linear16(const TmaMaps* mapA, const TmaMaps* mapW, int M, int N, int K, int dtype, const Epi& ep, float* part,
             size_t part_bytes, int* counters, cudaStream_t st, bool pdl = false, const NormIO* nio = nullptr);

int launch_attention_prefill(const Model* m, int layer, const RowTable& rt, cudaStream_t st);
int launch_attention_prefill_tc(const Model* m, int layer, const RowTable& rt, cudaStream_t st);
bool attention_prefill_tmem_ok(const Model* m);
int launch_attention_prefill_tmem(const Model* m, int layer, const RowTable& rt, cudaStream_t st);
// wait_ns > 0 replaces the default wait limit; stall_unit >= 0: CTA 0 never
// issues that unit's copies or their barrier signal (tests of the timeout).
int launch_attention_decode(const Model* m, int layer, const int32_t* pos, int B, cudaStream_t st,
                            bool pdl = false, unsigned long long* tl = nullptr, long long wait_ns = 0,
                            int stall_unit = -1);

int launch_argmax(const float* logits, int B, int V, int32_t* out, int32_t* tokens_adv,
                  int32_t* pos_adv, cudaStream_t st, bool pdl = false, unsigned long long* tl = nullptr);
int launch_logprobs(const float* logits, const int32_t* tokens, int N, int V, float* out, cudaStream_t st);
int launch_top_p(const float* logits, int B, int V, float temperature, float top_p,
                 const float* uniforms, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
                 cudaStream_t st, bool pdl = false, unsigned long long* tl = nullptr);

// Tensor parallelism: x[m, :] += sum over ranks r (in rank order) of
// part_r[m, :] for M rows, then the next RMSNorm's producer side (y =
// x * w_next in the model's 16-bit type, per-128-feature sums of x^2).
int launch_tp_reduce(const Model* m, const float* const* parts, int M, const float* w_next, const TpSync& sync,
                     cudaStream_t st);
// Copies every other rank's [rows, Vl] logits slice into this rank's [rows, V] buffer.
int launch_tp_gather_logits(const Model* m, float* logits, int rows, const TpSync& sync, cudaStream_t st);

// TMA descriptor of a K-major 16-bit matrix (dtype LLAMA_BF16 or LLAMA_F16),
// boxes of 64 columns x box_rows rows, 128-byte swizzle (driver entry point
// resolved at run time).
int encode_kmajor_16(CUtensorMap* map, const void* base, int rows, int cols, int box_rows, int dtype = LLAMA_BF16);

}  // namespace llb
