// C ABI of libllama_b200.so: argument validation, the arena layout, and the
// order of kernels in prefill and decode (Admin Guide §8.4, "The forward
// pass"; §8.5 for the sampling step).  All arithmetic happens in the kernels.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>

#include "common.cuh"
#include "model.h"
#include "../../include/llama_b200_ops.h"

namespace llb {

static thread_local char g_err[512] = "";
static std::atomic<uint64_t> g_launches{0};

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
int cuda_fail(cudaError_t e, const char* what) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return LLAMA_ERR_CUDA;
}

#define LLB_TRY(x)                       \
    do {                                 \
        const int _rc = (x);             \
        if (_rc != LLAMA_OK) return _rc; \
    } while (0)

static int hidden_dim(int dim, int multiple_of, float mult) {
    long long h = 4LL * dim;
    h = static_cast<long long>(2 * h / 3);
    if (mult > 0.f) h = static_cast<long long>(static_cast<double>(mult) * static_cast<double>(h));
    return static_cast<int>(multiple_of * ((h + multiple_of - 1) / multiple_of));
}

static size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Sizes and offsets of everything in the arena.
struct Layout {
    int dim, L, nh, nkv, hd, n_rep, H, V, Vl, S, Bmax, Mmax, Mrows, Brows, dtype, esz, nq, nkvc, nqkv, n_splits;
    int tp_rank, tp_size;
    size_t off_tok_emb, off_norm, off_output, layer_bytes;
    size_t l_attn_norm, l_wqkv, l_wo, l_ffn_norm, l_w13, l_w2;
    size_t off_layers, weight_bytes;
    size_t off_kc, off_vc, kv_bytes;
    size_t off_x, off_y, off_q, off_attn, off_g, off_ylast, off_tok_ids, off_tok_row, off_tok_pos, off_last,
        off_logits, off_part_o, off_part_ml, off_attn_cnt, off_status, off_rope, off_gemm_part, off_gemm_cnt,
        off_ssq, off_tl, off_best, off_step_cnt, off_tp_part, off_tp_flag, ws_end;
};

// Sizes and offsets of one model, or of shard tp_rank of a tensor-parallel
// group of tp_size: local query/KV heads, FFN hidden features and vocabulary
// rows are 1/tp_size of the model's (the sharding of Admin Guide §1.3 / §4.2).
static int make_layout(const llama_model_args* a, Layout* o, int tp_rank = 0, int tp_size = 1) {
    if (!a) { set_error("args is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (tp_size < 1 || tp_size > kMaxTp || tp_rank < 0 || tp_rank >= tp_size) {
        set_error("tensor-parallel rank %d of %d invalid (at most %d ranks)", tp_rank, tp_size, kMaxTp);
        return LLAMA_ERR_INVALID_ARG;
    }
    if (a->dim <= 0 || a->n_layers <= 0 || a->n_heads <= 0 || a->vocab_size <= 0 || a->multiple_of <= 0 ||
        a->max_seq_len <= 0 || a->max_batch_size <= 0 || a->n_kv_heads < 0 || a->max_tokens < 0) {
        set_error("non-positive size in llama_model_args");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (a->dtype != LLAMA_F32 && a->dtype != LLAMA_BF16 && a->dtype != LLAMA_F16) {
        set_error("dtype must be LLAMA_F32, LLAMA_BF16 or LLAMA_F16");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (!(a->norm_eps >= 0.f) || !(a->rope_theta > 0.f)) { set_error("norm_eps must be >= 0 and rope_theta > 0"); return LLAMA_ERR_INVALID_ARG; }
    const int nkv = a->n_kv_heads ? a->n_kv_heads : a->n_heads;
    if (a->n_heads % nkv) { set_error("n_heads %% n_kv_heads != 0"); return LLAMA_ERR_INVALID_ARG; }
    const int n_rep = a->n_heads / nkv;
    if (n_rep != 1 && n_rep != 2 && n_rep != 4 && n_rep != 8) { set_error("n_heads / n_kv_heads must be 1, 2, 4 or 8"); return LLAMA_ERR_INVALID_ARG; }
    if (a->dim % a->n_heads) { set_error("dim %% n_heads != 0"); return LLAMA_ERR_INVALID_ARG; }
    const int hd = a->dim / a->n_heads;
    if (hd != 32 && hd != 64 && hd != 128) { set_error("head_dim %d unsupported (32, 64, 128)", hd); return LLAMA_ERR_INVALID_ARG; }
    if (a->dim % 64) { set_error("dim must be a multiple of 64"); return LLAMA_ERR_INVALID_ARG; }
    if (a->max_batch_size > kMaxRows) { set_error("max_batch_size > %d", kMaxRows); return LLAMA_ERR_INVALID_ARG; }
    const int H_full = hidden_dim(a->dim, a->multiple_of, a->ffn_dim_multiplier);
    if (H_full % 64) { set_error("FFN hidden %d must be a multiple of 64", H_full); return LLAMA_ERR_INVALID_ARG; }
    if (tp_size > 1) {
        if (a->dtype == LLAMA_F32) { set_error("tensor parallelism runs 16-bit models"); return LLAMA_ERR_INVALID_ARG; }
        if (a->n_heads % tp_size || nkv % tp_size || H_full % tp_size || a->vocab_size % tp_size ||
            (H_full / tp_size) % 64) {
            set_error("n_heads, n_kv_heads, vocab_size and the FFN hidden width (in multiples of 64) must split "
                      "evenly over %d ranks", tp_size);
            return LLAMA_ERR_INVALID_ARG;
        }
    }
    const int H = H_full / tp_size;
    {
        const long long nq_l = static_cast<long long>(a->n_heads / tp_size) * (a->dim / a->n_heads);
        const long long widest = std::max(std::max(static_cast<long long>(a->vocab_size / tp_size), 2LL * H),
                                          nq_l + 2LL * (nkv / tp_size) * (a->dim / a->n_heads));
        if ((widest + 127) / 128 > kMaxTiles) { set_error("a projection is wider than %d x 128 rows", kMaxTiles); return LLAMA_ERR_INVALID_ARG; }
    }
    if (a->dtype != LLAMA_F32 && (a->dim < 256 || a->vocab_size < 256 || a->dim % 128)) {
        set_error("16-bit models need dim >= 256 (a multiple of 128) and vocab_size >= 256");
        return LLAMA_ERR_INVALID_ARG;
    }
    Layout& l = *o;
    l.dim = a->dim; l.L = a->n_layers; l.nh = a->n_heads / tp_size; l.nkv = nkv / tp_size; l.hd = hd; l.n_rep = n_rep;
    l.H = H; l.V = a->vocab_size; l.Vl = a->vocab_size / tp_size; l.tp_rank = tp_rank; l.tp_size = tp_size;
    l.S = a->max_seq_len; l.Bmax = a->max_batch_size; l.dtype = a->dtype;
    l.esz = a->dtype == LLAMA_F32 ? 4 : 2;
    const long long mt = a->max_tokens ? a->max_tokens : 1LL * a->max_batch_size * a->max_seq_len;
    if (mt > (1LL << 30)) { set_error("max_tokens too large"); return LLAMA_ERR_INVALID_ARG; }
    l.Mmax = static_cast<int>(mt > l.Bmax ? mt : l.Bmax);
    l.Mrows = l.Mmax < 128 ? 128 : l.Mmax;    // activation buffers hold whole 128-row tiles
    l.Brows = l.Bmax < 128 ? 128 : l.Bmax;
    l.nq = l.nh * hd; l.nkvc = l.nkv * hd; l.nqkv = l.nq + 2 * l.nkvc;
    l.n_splits = (l.S + kChunk - 1) / kChunk;
    const size_t e = l.esz, D = l.dim;
    size_t off = 0;
    l.off_tok_emb = off; off = align256(off + static_cast<size_t>(l.V) * D * e);
    l.off_norm = off; off = align256(off + D * 4);
    l.off_output = off; off = align256(off + static_cast<size_t>(l.Vl) * D * e);
    l.off_layers = off;
    size_t lo = 0;
    l.l_attn_norm = lo; lo = align256(lo + D * 4);
    l.l_wqkv = lo; lo = align256(lo + static_cast<size_t>(l.nqkv) * D * e);
    l.l_wo = lo; lo = align256(lo + D * l.nq * e);
    l.l_ffn_norm = lo; lo = align256(lo + D * 4);
    l.l_w13 = lo; lo = align256(lo + 2ull * H * D * e);
    l.l_w2 = lo; lo = align256(lo + D * H * e);
    l.layer_bytes = lo;
    off += lo * l.L;
    l.weight_bytes = off;
    const size_t kv_one = static_cast<size_t>(l.L) * l.Bmax * l.nkv * l.S * hd * e;
    l.off_kc = off; off = align256(off + kv_one);
    l.off_vc = off; off = align256(off + kv_one);
    l.kv_bytes = off - l.weight_bytes;
    const size_t M = l.Mrows, Bn = l.Brows;
    l.off_x = off; off = align256(off + M * D * 4);
    l.off_y = off; off = align256(off + M * D * e);
    l.off_q = off; off = align256(off + M * l.nq * e);
    l.off_attn = off; off = align256(off + M * l.nq * e);
    l.off_g = off; off = align256(off + M * H * e);
    l.off_ylast = off; off = align256(off + Bn * D * e);
    l.off_tok_ids = off; off = align256(off + M * 4);
    l.off_tok_row = off; off = align256(off + M * 4);
    l.off_tok_pos = off; off = align256(off + M * 4);
    l.off_last = off; off = align256(off + Bn * 4);
    l.off_logits = off; off = align256(off + static_cast<size_t>(l.Bmax) * l.V * 4);
    const size_t slots = static_cast<size_t>(2) * kMaxAttnCtas * n_rep;   // decode attention partials
    l.off_part_o = off; off = align256(off + slots * hd * 4);
    l.off_part_ml = off; off = align256(off + slots * 2 * 4);
    l.off_attn_cnt = off; off = align256(off + static_cast<size_t>(l.Bmax) * l.nkv * 4);
    l.off_status = off; off = align256(off + 16);
    l.off_rope = off; off = align256(off + static_cast<size_t>(l.S) * (hd / 2) * 8);
    l.off_gemm_part = off; off = align256(off + (a->dtype != LLAMA_F32 ? kGemmPartBytes : 0));
    l.off_gemm_cnt = off; off = align256(off + kMaxTiles * sizeof(int));
    l.off_ssq = off; off = align256(off + static_cast<size_t>(M > Bn ? M : Bn) * (l.dim / 128 + 1) * 4);
    l.off_tl = off; off = align256(off + static_cast<size_t>(kTimelineCap) * 8);
    l.off_best = off; off = align256(off + static_cast<size_t>(l.Bmax) * 8);
    l.off_step_cnt = off; off = align256(off + kStepCounters * sizeof(int));
    l.off_tp_part = off; off = align256(off + (tp_size > 1 ? 2 * M * D * 4 : 0));
    l.off_tp_flag = off; off = align256(off + (kMaxTp + 2) * 8 + 16);
    l.ws_end = off;
    return LLAMA_OK;
}

static int make_maps(TmaMaps* t, const void* base, int rows, int cols, int b_box, int dtype) {
    LLB_TRY(encode_kmajor_16(&t->a128, base, rows, cols, 128, dtype));
    LLB_TRY(encode_kmajor_16(&t->b, base, rows, cols, b_box, dtype));
    return LLAMA_OK;
}

// Algorithmic bytes of one projection: the weight once, the 16-bit input rows
// once, and what its epilogue must move (fp32 store; fp32 residual read and
// write; 16-bit q/k/v; the 16-bit SwiGLU product, half as wide as N; the
// logits only when they are stored).
static int64_t proj_bytes(int M, int N, int K, const Epi& ep) {
    const int64_t mn = static_cast<int64_t>(M) * N;
    int64_t out = 0;
    switch (ep.mode) {
        case EPI_STORE_F32: out = 4 * mn; break;
        case EPI_RESID_F32: out = 8 * mn; break;
        case EPI_QKV: out = 2 * mn; break;
        case EPI_SWIGLU: out = mn; break;
        case EPI_LOGITS_ARGMAX: out = ep.out ? 4 * mn : 0; break;
    }
    return 2LL * N * K + 2LL * M * K + out;
}

// The one-shot stall of llama_debug_stall, taken by the first launch of the
// chosen kind: returns true and the stall's unit and wait limit, and clears it.
static bool take_stall(Model* m, int kind, int* unit, long long* wait_ns) {
    if (m->dbg_kind != kind) return false;
    *unit = m->dbg_unit;
    *wait_ns = m->dbg_wait_ns;
    m->dbg_kind = 0;
    return true;
}

unsigned long long* tl_next(Model* m, int kind, int64_t bytes) {
    if (!m->tl_on || m->tl_n >= kTimelineCap) return nullptr;
    m->tl_kind.push_back(kind);
    m->tl_bytes.push_back(bytes);
    return m->tl_end + m->tl_n++;
}

int run_linear(const Model* m, int dtype, const void* A, const TmaMaps* mapA, const void* W,
               const TmaMaps* mapW, int M, int N, int K, const Epi& ep_in, cudaStream_t st, bool pdl,
               const NormIO* nio, bool stamp) {
    Epi ep = ep_in;
    if (stamp) ep.tl = tl_next(const_cast<Model*>(m), TL_PROJECTION, proj_bytes(M, N, K, ep));
    if (dtype != LLAMA_F32) {
        int unit = 0;
        long long wait_ns = 0;
        if (take_stall(const_cast<Model*>(m), LLAMA_STALL_PROJECTION, &unit, &wait_ns)) {
            ep.stall = unit + 1;
            ep.wait_ns = wait_ns;
        }
    }
    Profile* pr = const_cast<Profile*>(&m->prof);
    const bool timed = pr->n < pr->capacity;
    if (timed) {
        cudaError_t e = cudaEventRecord(pr->ev[2 * pr->n], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord(profile)");
    }
    int rc;
    if (dtype == LLAMA_F32)
        rc = linear_f32(static_cast<const float*>(A), static_cast<const float*>(W), M, N, K, ep, st);
    else
        rc = linear16(mapA, mapW, M, N, K, dtype, ep, m->gemm_part, kGemmPartBytes, m->gemm_cnt, st, pdl && !timed, nio);
    if (timed && rc == LLAMA_OK) {
        cudaError_t e = cudaEventRecord(pr->ev[2 * pr->n + 1], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord(profile)");
        pr->bytes[pr->n] = proj_bytes(M, N, K, ep);
        pr->flops[pr->n] = 2LL * M * N * K;
        pr->rows[pr->n] = M;
        pr->n++;
    }
    return rc;
}

static void profile_release(Profile& p) {
    for (cudaEvent_t e : p.ev) cudaEventDestroy(e);
    p.ev.clear();
    p.bytes.clear();
    p.flops.clear();
    p.rows.clear();
    p.capacity = 0;
    p.n = 0;
}

static Epi base_epi(const Model* m) {
    Epi ep;
    memset(&ep, 0, sizeof(ep));
    ep.status = m->status;
    ep.nq = m->nq;
    ep.nkvc = m->nkvc;
    ep.hd = m->hd;
    ep.max_seq = m->S;
    ep.kv_row_stride = m->kv_row_elems;
    ep.rope = m->rope;
    ep.H = m->H;
    return ep;
}

static char* at(void* base, size_t off) { return static_cast<char*>(base) + off; }

// Widest decode step (token rows) that runs the fused chain of
// llama_decode_step: the weight-streaming projection's MMA N limit.
constexpr int kFusedDecodeRows = 64;

// One transformer block of a 16-bit model on M token rows (Admin Guide §8.4,
// TransformerBlock: h = x + attn(norm(x)); out = h + ffn(norm(h))), with both
// RMSNorms folded into the projections: on entry m->y holds bf16(x * w_attn)
// and m->ssq the per-128-feature sums of x^2 (left by the embedding or the
// previous block); wq/wk/wv and w1/w3 scale their accumulator rows by 1/rms,
// and the residual epilogues of wo and w2 leave the next norm's inputs
// (w_ffn, then the next block's w_attn or the final norm's weight).  M <= 64
// rows run the weight-streaming projections (pdl: launched early in the
// decode chain), more rows the 128 x 256-tile ones.
template <typename AttnFn>
static int block_forward_fused(Model* m, int l, int M, const int* tok_row, const int* tok_pos, AttnFn attn,
                               cudaStream_t st, bool pdl, bool stamp) {
    LayerPtrs& Lp = m->layers[l];
    const size_t esz = m->esz;
    const float* next_norm = l + 1 < m->L ? m->layers[l + 1].attn_norm : m->norm;
    const NormIO n_in = {m->ssq, m->dim / 128, m->a.norm_eps, nullptr, nullptr, nullptr};
    const NormIO n_to_ffn = {nullptr, 0, 0.f, m->ssq, m->y, Lp.ffn_norm};
    const NormIO n_to_next = {nullptr, 0, 0.f, m->ssq, m->y, next_norm};
    Epi ep = base_epi(m);
    ep.mode = EPI_QKV;
    ep.q = m->q;
    ep.kc = static_cast<char*>(m->kc) + l * m->kv_layer_elems * esz;
    ep.vc = static_cast<char*>(m->vc) + l * m->kv_layer_elems * esz;
    ep.tok_row = tok_row;
    ep.tok_pos = tok_pos;
    LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, Lp.wqkv, &Lp.m_wqkv, M, m->nqkv, m->dim, ep, st, pdl, &n_in,
                       stamp));
    LLB_TRY(attn());
    Epi er = base_epi(m);
    er.mode = EPI_RESID_F32;
    er.out = m->x;
    er.ldo = m->dim;
    LLB_TRY(run_linear(m, m->dtype, m->attn, &m->m_attn, Lp.wo, &Lp.m_wo, M, m->dim, m->nq, er, st, pdl, &n_to_ffn,
                       stamp));
    Epi es = base_epi(m);
    es.mode = EPI_SWIGLU;
    es.g = m->g;
    LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, Lp.w13, &Lp.m_w13, M, 2 * m->H, m->dim, es, st, pdl, &n_in,
                       stamp));
    return run_linear(m, m->dtype, m->g, &m->m_g, Lp.w2, &Lp.m_w2, M, m->dim, m->H, er, st, pdl, &n_to_next, stamp);
}

// One transformer block of an fp32 model: RMSNorm kernels, then the SIMT projections.
template <typename AttnFn>
static int block_forward(Model* m, int l, int M, const int* tok_row, const int* tok_pos, AttnFn attn,
                         cudaStream_t st, bool pdl, bool stamp = false) {
    LayerPtrs& Lp = m->layers[l];
    const size_t esz = m->esz;
    auto norm_tl = [&]() { return stamp ? tl_next(m, TL_RMSNORM, 0) : nullptr; };
    LLB_TRY(launch_rmsnorm(m->x, nullptr, Lp.attn_norm, M, m->dim, m->a.norm_eps, m->y, m->dtype, st, pdl,
                           norm_tl()));
    Epi ep = base_epi(m);
    ep.mode = EPI_QKV;
    ep.q = m->q;
    ep.kc = static_cast<char*>(m->kc) + l * m->kv_layer_elems * esz;
    ep.vc = static_cast<char*>(m->vc) + l * m->kv_layer_elems * esz;
    ep.tok_row = tok_row;
    ep.tok_pos = tok_pos;
    LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, Lp.wqkv, &Lp.m_wqkv, M, m->nqkv, m->dim, ep, st, pdl, nullptr,
                       stamp));
    LLB_TRY(attn());
    Epi er = base_epi(m);
    er.mode = EPI_RESID_F32;
    er.out = m->x;
    er.ldo = m->dim;
    LLB_TRY(run_linear(m, m->dtype, m->attn, &m->m_attn, Lp.wo, &Lp.m_wo, M, m->dim, m->nq, er, st, pdl, nullptr,
                       stamp));
    LLB_TRY(launch_rmsnorm(m->x, nullptr, Lp.ffn_norm, M, m->dim, m->a.norm_eps, m->y, m->dtype, st, pdl,
                           norm_tl()));
    Epi es = base_epi(m);
    es.mode = EPI_SWIGLU;
    es.g = m->g;
    LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, Lp.w13, &Lp.m_w13, M, 2 * m->H, m->dim, es, st, pdl, nullptr,
                       stamp));
    LLB_TRY(run_linear(m, m->dtype, m->g, &m->m_g, Lp.w2, &Lp.m_w2, M, m->dim, m->H, er, st, pdl, nullptr, stamp));
    return LLAMA_OK;
}

// ---------------------------------------------------------------- tensor parallelism
// The shards one call runs: every rank of a group on this GPU, or this rank
// alone (its peers on other GPUs, reached through the bound buffers).
struct Shards {
    Model* m[kMaxTp];
    int n;
};

static TpSync tp_sync_of(const Model* m) {
    TpSync s = {};
    s.wait = m->tp_wait ? 1 : 0;
    s.rank = m->tp_rank;
    s.size = m->tp_size;
    s.my_flags = m->tp_flag;
    for (int q = 0; q < m->tp_size; ++q) s.peer_flags[q] = m->peers.flag[q];
    s.epoch = m->tp_epoch;
    s.arrivals = m->tp_arrivals;
    s.status = m->status;
    return s;
}

// x += the partial sums of phase `parity` of every rank, then the next
// RMSNorm's inputs, on every shard of `sh`.
static int tp_reduce_all(const Shards& sh, int parity, int M, const float* const* w_next, cudaStream_t st) {
    for (int i = 0; i < sh.n; ++i) {
        const Model* m = sh.m[i];
        const float* parts[kMaxTp];
        for (int r = 0; r < m->tp_size; ++r) parts[r] = m->peers.part[r][parity];
        LLB_TRY(launch_tp_reduce(m, parts, M, w_next[i], tp_sync_of(m), st));
    }
    return LLAMA_OK;
}

// One transformer block of a tensor-parallel group (Admin Guide §8.4
// TransformerBlock, sharded as §1.3 / §4.2): each shard computes its query
// and KV heads (wq/wk/wv, RoPE, cache append, attention) and its slice of
// wo's input columns, leaving a partial residual update; the reduce adds the
// ranks' updates to x and writes the FFN norm's inputs; each shard computes
// its SwiGLU features (w1/w3) and its slice of w2's input columns; a second
// reduce finishes the block.  M token rows; per-shard token maps.
template <typename AttnFn>
static int tp_block(const Shards& sh, int l, int M, bool prefill, const int32_t* pos, AttnFn attn, cudaStream_t st) {
    for (int i = 0; i < sh.n; ++i) {
        Model* m = sh.m[i];
        LayerPtrs& Lp = m->layers[l];
        const NormIO n_in = {m->ssq, m->dim / 128, m->a.norm_eps, nullptr, nullptr, nullptr};
        Epi ep = base_epi(m);
        ep.mode = EPI_QKV;
        ep.q = m->q;
        ep.kc = static_cast<char*>(m->kc) + l * m->kv_layer_elems * m->esz;
        ep.vc = static_cast<char*>(m->vc) + l * m->kv_layer_elems * m->esz;
        ep.tok_row = prefill ? m->tok_row : nullptr;
        ep.tok_pos = prefill ? m->tok_pos : pos;
        LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, Lp.wqkv, &Lp.m_wqkv, M, m->nqkv, m->dim, ep, st, false, &n_in));
        LLB_TRY(attn(m));
        Epi ew = base_epi(m);
        ew.mode = EPI_STORE_F32;
        ew.out = m->tp_part[0];
        ew.ldo = m->dim;
        LLB_TRY(run_linear(m, m->dtype, m->attn, &m->m_attn, Lp.wo, &Lp.m_wo, M, m->dim, m->nq, ew, st));
    }
    const float* ffn_norm[kMaxTp];
    for (int i = 0; i < sh.n; ++i) ffn_norm[i] = sh.m[i]->layers[l].ffn_norm;
    LLB_TRY(tp_reduce_all(sh, 0, M, ffn_norm, st));
    for (int i = 0; i < sh.n; ++i) {
        Model* m = sh.m[i];
        LayerPtrs& Lp = m->layers[l];
        const NormIO n_in = {m->ssq, m->dim / 128, m->a.norm_eps, nullptr, nullptr, nullptr};
        Epi es = base_epi(m);
        es.mode = EPI_SWIGLU;
        es.g = m->g;
        LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, Lp.w13, &Lp.m_w13, M, 2 * m->H, m->dim, es, st, false, &n_in));
        Epi ew = base_epi(m);
        ew.mode = EPI_STORE_F32;
        ew.out = m->tp_part[1];
        ew.ldo = m->dim;
        LLB_TRY(run_linear(m, m->dtype, m->g, &m->m_g, Lp.w2, &Lp.m_w2, M, m->dim, m->H, ew, st));
    }
    const float* next_norm[kMaxTp];
    for (int i = 0; i < sh.n; ++i)
        next_norm[i] = l + 1 < sh.m[i]->L ? sh.m[i]->layers[l + 1].attn_norm : sh.m[i]->norm;
    return tp_reduce_all(sh, 1, M, next_norm, st);
}

// The vocabulary projection of a group: shard r writes logits columns
// [r * Vl, (r + 1) * Vl) of `out` ([rows, V]); with the shards on separate
// GPUs each writes its own logits buffer, gathers the others' slices and
// copies the rows to `out`.
static int tp_logits(const Shards& sh, int rows, bool last_rows, float* out, cudaStream_t st) {
    for (int i = 0; i < sh.n; ++i) {
        Model* m = sh.m[i];
        const bool remote = m->tp_wait;
        float* dst = remote ? m->logits_ws : out;
        Epi eo = base_epi(m);
        eo.mode = EPI_STORE_F32;
        eo.out = dst + static_cast<size_t>(m->tp_rank) * m->Vl;
        eo.ldo = m->V;
        if (last_rows) {
            LLB_TRY(launch_rmsnorm(m->x, m->last_idx, m->norm, rows, m->dim, m->a.norm_eps, m->ylast, m->dtype, st));
            LLB_TRY(run_linear(m, m->dtype, m->ylast, &m->m_ylast, m->output, &m->m_output, rows, m->Vl, m->dim, eo, st));
        } else {
            const NormIO n_in = {m->ssq, m->dim / 128, m->a.norm_eps, nullptr, nullptr, nullptr};
            LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, m->output, &m->m_output, rows, m->Vl, m->dim, eo, st, false,
                               &n_in));
        }
        if (remote) {
            LLB_TRY(launch_tp_gather_logits(m, m->logits_ws, rows, tp_sync_of(m), st));
            if (out && out != m->logits_ws) {
                cudaError_t e = cudaMemcpyAsync(out, m->logits_ws, static_cast<size_t>(rows) * m->V * 4,
                                                cudaMemcpyDeviceToDevice, st);
                if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(tp logits)");
            }
        }
    }
    return LLAMA_OK;
}

static int tp_prefill(const Shards& sh, const RowTable& rt, const int32_t* tokens, float* logits, int logits_mode,
                      cudaStream_t st) {
    const int M = rt.cu[rt.B];
    for (int i = 0; i < sh.n; ++i) {
        Model* m = sh.m[i];
        LLB_TRY(launch_token_map(rt, tokens, m->tok_ids, m->tok_row, m->tok_pos, m->last_idx, st));
        LLB_TRY(launch_embed(m->tok_ids, m->tok_emb, m->dtype, M, m->dim, m->V, m->x, m->status, st, false, m->ssq,
                             m->y, m->layers[0].attn_norm));
    }
    for (int l = 0; l < sh.m[0]->L; ++l) {
        auto attn = [&](Model* m) { return launch_attention_prefill(m, l, rt, st); };
        LLB_TRY(tp_block(sh, l, M, true, nullptr, attn, st));
    }
    if (!logits) return LLAMA_OK;
    return tp_logits(sh, logits_mode == 0 ? rt.B : M, logits_mode == 0, logits, st);
}

static int tp_decode(const Shards& sh, const int32_t* tokens, int32_t* pos, int B, const llama_sampling* sampling,
                     const float* uniforms, int32_t* next_tokens, float* logits, int flags, cudaStream_t st) {
    for (int i = 0; i < sh.n; ++i) {
        Model* m = sh.m[i];
        LLB_TRY(launch_embed(tokens, m->tok_emb, m->dtype, B, m->dim, m->V, m->x, m->status, st, false, m->ssq, m->y,
                             m->layers[0].attn_norm));
    }
    for (int l = 0; l < sh.m[0]->L; ++l) {
        auto attn = [&](Model* m) { return launch_attention_decode(m, l, pos, B, st); };
        LLB_TRY(tp_block(sh, l, B, false, pos, attn, st));
    }
    Model* m0 = sh.m[0];
    float* lg = logits ? logits : m0->logits_ws;
    LLB_TRY(tp_logits(sh, B, false, lg, st));
    if (!sampling) return LLAMA_OK;
    const bool adv = (flags & LLAMA_DECODE_ADVANCE) != 0;
    int32_t* tok_adv = adv ? const_cast<int32_t*>(tokens) : nullptr;
    int32_t* pos_adv = adv ? pos : nullptr;
    if (sampling->temperature == 0.f) return launch_argmax(lg, B, m0->V, next_tokens, tok_adv, pos_adv, st);
    return launch_top_p(lg, B, m0->V, sampling->temperature, sampling->top_p, uniforms, next_tokens, tok_adv,
                        pos_adv, st);
}

// The shards of a one-GPU group, checked: ranks 0 .. tp-1 in order, one
// configuration; their buffers are bound to each other (no handshake).
static int group_of(llama_model_args* ref, Model* const* shards, int tp, Shards* out) {
    if (!shards || tp < 1 || tp > kMaxTp) { set_error("shards must hold 1..%d models", kMaxTp); return LLAMA_ERR_INVALID_ARG; }
    out->n = tp;
    for (int r = 0; r < tp; ++r) {
        Model* m = shards[r];
        if (!m) { set_error("shard %d is NULL", r); return LLAMA_ERR_INVALID_ARG; }
        if (m->tp_size != tp || m->tp_rank != r) {
            set_error("shard %d is rank %d of %d, expected rank %d of %d", r, m->tp_rank, m->tp_size, r, tp);
            return LLAMA_ERR_INVALID_ARG;
        }
        if (memcmp(&m->a, &shards[0]->a, sizeof(llama_model_args)) != 0) {
            set_error("shard %d was created with other model arguments", r);
            return LLAMA_ERR_INVALID_ARG;
        }
        out->m[r] = m;
    }
    for (int r = 0; r < tp; ++r) {
        Model* m = shards[r];
        for (int q = 0; q < tp; ++q) {
            m->peers.part[q][0] = shards[q]->tp_part[0];
            m->peers.part[q][1] = shards[q]->tp_part[1];
            m->peers.flag[q] = shards[q]->tp_flag;
            m->peers.logits[q] = shards[q]->logits_ws;
        }
        m->tp_bound = true;
        m->tp_wait = false;
    }
    if (ref) *ref = shards[0]->a;
    return LLAMA_OK;
}

}  // namespace llb

using namespace llb;

struct llama_model : public llb::Model {};

extern "C" {

const char* llama_last_error(void) { return g_err; }
uint64_t llama_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int llama_model_bytes(const llama_model_args* args, size_t* weight_bytes, size_t* kv_bytes,
                      size_t* workspace_bytes, size_t* total_bytes, int32_t* hidden) {
    return llama_model_bytes_tp(args, 0, 1, weight_bytes, kv_bytes, workspace_bytes, total_bytes, hidden);
}

int llama_model_bytes_tp(const llama_model_args* args, int tp_rank, int tp_size, size_t* weight_bytes,
                         size_t* kv_bytes, size_t* workspace_bytes, size_t* total_bytes, int32_t* hidden) {
    Layout l;
    LLB_TRY(make_layout(args, &l, tp_rank, tp_size));
    if (weight_bytes) *weight_bytes = l.weight_bytes;
    if (kv_bytes) *kv_bytes = l.kv_bytes;
    if (workspace_bytes) *workspace_bytes = l.ws_end - l.weight_bytes - l.kv_bytes;
    if (total_bytes) *total_bytes = l.ws_end;
    if (hidden) *hidden = l.H;
    return LLAMA_OK;
}

int llama_model_create(const llama_model_args* args, void* dev_arena, size_t arena_bytes, void* stream,
                       llama_model** out) {
    return llama_model_create_tp(args, 0, 1, dev_arena, arena_bytes, stream, out);
}

int llama_model_create_tp(const llama_model_args* args, int tp_rank, int tp_size, void* dev_arena,
                          size_t arena_bytes, void* stream, llama_model** out) {
    if (!out) { set_error("out is NULL"); return LLAMA_ERR_INVALID_ARG; }
    *out = nullptr;
    Layout l;
    LLB_TRY(make_layout(args, &l, tp_rank, tp_size));
    if (!dev_arena) { set_error("arena is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (reinterpret_cast<uintptr_t>(dev_arena) & 255) { set_error("arena must be 256-byte aligned"); return LLAMA_ERR_INVALID_ARG; }
    if (arena_bytes < l.ws_end) {
        set_error("arena too small: %zu < %zu bytes", arena_bytes, l.ws_end);
        return LLAMA_ERR_CAPACITY;
    }
    llama_model* m = new (std::nothrow) llama_model();
    if (!m) { set_error("host allocation failed"); return LLAMA_ERR_CAPACITY; }
    m->a = *args;
    m->dim = l.dim; m->L = l.L; m->nh = l.nh; m->nkv = l.nkv; m->hd = l.hd; m->n_rep = l.n_rep; m->H = l.H;
    m->V = l.V; m->S = l.S; m->Bmax = l.Bmax; m->Mmax = l.Mmax; m->dtype = l.dtype; m->esz = l.esz;
    m->Vl = l.Vl; m->tp_rank = l.tp_rank; m->tp_size = l.tp_size;
    m->nq = l.nq; m->nkvc = l.nkvc; m->nqkv = l.nqkv; m->n_splits = l.n_splits;
    void* A = dev_arena;
    m->tok_emb = at(A, l.off_tok_emb);
    m->norm = reinterpret_cast<float*>(at(A, l.off_norm));
    m->output = at(A, l.off_output);
    m->layers.resize(l.L);
    for (int i = 0; i < l.L; ++i) {
        char* base = at(A, l.off_layers + i * l.layer_bytes);
        LayerPtrs& p = m->layers[i];
        p.attn_norm = reinterpret_cast<float*>(base + l.l_attn_norm);
        p.wqkv = base + l.l_wqkv;
        p.wo = base + l.l_wo;
        p.ffn_norm = reinterpret_cast<float*>(base + l.l_ffn_norm);
        p.w13 = base + l.l_w13;
        p.w2 = base + l.l_w2;
    }
    m->kc = at(A, l.off_kc);
    m->vc = at(A, l.off_vc);
    m->kv_head_elems = static_cast<long long>(l.S) * l.hd;
    m->kv_row_elems = m->kv_head_elems * l.nkv;
    m->kv_layer_elems = m->kv_row_elems * l.Bmax;
    m->x = reinterpret_cast<float*>(at(A, l.off_x));
    m->y = at(A, l.off_y);
    m->q = at(A, l.off_q);
    m->attn = at(A, l.off_attn);
    m->g = at(A, l.off_g);
    m->ylast = at(A, l.off_ylast);
    m->tok_ids = reinterpret_cast<int*>(at(A, l.off_tok_ids));
    m->tok_row = reinterpret_cast<int*>(at(A, l.off_tok_row));
    m->tok_pos = reinterpret_cast<int*>(at(A, l.off_tok_pos));
    m->last_idx = reinterpret_cast<int*>(at(A, l.off_last));
    m->logits_ws = reinterpret_cast<float*>(at(A, l.off_logits));
    m->part_o = reinterpret_cast<float*>(at(A, l.off_part_o));
    m->part_ml = reinterpret_cast<float*>(at(A, l.off_part_ml));
    m->attn_cnt = reinterpret_cast<int*>(at(A, l.off_attn_cnt));
    m->status = reinterpret_cast<int*>(at(A, l.off_status));
    m->rope = reinterpret_cast<float2*>(at(A, l.off_rope));
    m->gemm_part = reinterpret_cast<float*>(at(A, l.off_gemm_part));
    m->gemm_cnt = reinterpret_cast<int*>(at(A, l.off_gemm_cnt));
    m->ssq = reinterpret_cast<float*>(at(A, l.off_ssq));
    m->tl_end = reinterpret_cast<unsigned long long*>(at(A, l.off_tl));
    m->best = reinterpret_cast<unsigned long long*>(at(A, l.off_best));
    m->step_cnt = reinterpret_cast<int*>(at(A, l.off_step_cnt));
    if (l.tp_size > 1) {
        m->tp_part[0] = reinterpret_cast<float*>(at(A, l.off_tp_part));
        m->tp_part[1] = m->tp_part[0] + static_cast<size_t>(l.Mrows) * l.dim;
    }
    m->tp_flag = reinterpret_cast<unsigned long long*>(at(A, l.off_tp_flag));
    m->tp_epoch = m->tp_flag + kMaxTp;
    m->tp_arrivals = reinterpret_cast<int*>(m->tp_epoch + 1);
    m->last_stream = static_cast<cudaStream_t>(stream);

    int rc = LLAMA_OK;
    if (l.dtype != LLAMA_F32) {
        for (int i = 0; i < l.L && rc == LLAMA_OK; ++i) {
            LayerPtrs& p = m->layers[i];
            if (rc == LLAMA_OK) rc = make_maps(&p.m_wqkv, p.wqkv, l.nqkv, l.dim, 256, l.dtype);
            if (rc == LLAMA_OK) rc = make_maps(&p.m_wo, p.wo, l.dim, l.nq, 256, l.dtype);
            if (rc == LLAMA_OK) rc = make_maps(&p.m_w13, p.w13, 2 * l.H, l.dim, 256, l.dtype);
            if (rc == LLAMA_OK) rc = make_maps(&p.m_w2, p.w2, l.dim, l.H, 256, l.dtype);
        }
        if (rc == LLAMA_OK) rc = make_maps(&m->m_output, m->output, l.Vl, l.dim, 256, l.dtype);
        if (rc == LLAMA_OK) rc = make_maps(&m->m_y, m->y, l.Mrows, l.dim, 16, l.dtype);
        if (rc == LLAMA_OK) rc = make_maps(&m->m_attn, m->attn, l.Mrows, l.nq, 16, l.dtype);
        if (rc == LLAMA_OK) rc = make_maps(&m->m_g, m->g, l.Mrows, l.H, 16, l.dtype);
        if (rc == LLAMA_OK) rc = make_maps(&m->m_ylast, m->ylast, l.Brows, l.dim, 16, l.dtype);
        const long long kv_rows = static_cast<long long>(l.L) * l.Bmax * l.nkv * l.S;
        if (rc == LLAMA_OK && l.hd == 128 && kv_rows + 128 < (1LL << 31)) {
            rc = encode_kmajor_16(&m->m_qtile, m->q, l.Mrows, l.nq, 128, l.dtype);
            if (rc == LLAMA_OK) rc = encode_kmajor_16(&m->m_kcache, m->kc, static_cast<int>(kv_rows), l.hd, 128, l.dtype);
            if (rc == LLAMA_OK) rc = encode_kmajor_16(&m->m_vcache, m->vc, static_cast<int>(kv_rows), l.hd, 128, l.dtype);
            m->has_attn_maps = rc == LLAMA_OK;
            if (rc == LLAMA_OK) rc = encode_kmajor_16(&m->m_kdec, m->kc, static_cast<int>(kv_rows), l.hd, 64, l.dtype);
            if (rc == LLAMA_OK) rc = encode_kmajor_16(&m->m_vdec, m->vc, static_cast<int>(kv_rows), l.hd, 64, l.dtype);
            m->has_dec_maps = rc == LLAMA_OK;
        }
    }
    cudaStream_t st = m->last_stream;
    if (rc == LLAMA_OK) {
        cudaError_t e = cudaMemsetAsync(m->kc, 0, l.kv_bytes, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(m->status, 0, 16, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(m->gemm_cnt, 0, kMaxTiles * sizeof(int), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(m->attn_cnt, 0, static_cast<size_t>(l.Bmax) * l.nkv * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(m->best, 0, static_cast<size_t>(l.Bmax) * 8, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(m->step_cnt, 0, kStepCounters * sizeof(int), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(m->tp_flag, 0, (kMaxTp + 2) * 8 + 16, st);
        if (e != cudaSuccess) rc = cuda_fail(e, "cudaMemsetAsync");
    }
    if (rc == LLAMA_OK) rc = launch_rope_table(m->rope, l.S, l.hd, args->rope_theta, st);
    if (rc != LLAMA_OK) {
        delete m;
        return rc;
    }
    *out = m;
    return LLAMA_OK;
}

int llama_set_weight(llama_model* m, int layer, int which, const void* src, void* stream) {
    if (!m || !src) { set_error("model or src is NULL"); return LLAMA_ERR_INVALID_ARG; }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    m->last_stream = st;
    const size_t e = m->esz, D = m->dim;
    const bool global = which == LLAMA_W_TOK_EMBEDDINGS || which == LLAMA_W_NORM || which == LLAMA_W_OUTPUT;
    if (which < 0 || which > LLAMA_W_W3) { set_error("unknown weight id %d", which); return LLAMA_ERR_INVALID_ARG; }
    if (global ? layer != -1 : (layer < 0 || layer >= m->L)) {
        set_error("layer %d invalid for weight %d", layer, which);
        return LLAMA_ERR_INVALID_ARG;
    }
    void* dst = nullptr;
    size_t bytes = 0;
    LayerPtrs* p = global ? nullptr : &m->layers[layer];
    switch (which) {
        case LLAMA_W_TOK_EMBEDDINGS: dst = m->tok_emb; bytes = static_cast<size_t>(m->V) * D * e; break;
        case LLAMA_W_NORM: dst = m->norm; bytes = D * 4; break;
        case LLAMA_W_OUTPUT: dst = m->output; bytes = static_cast<size_t>(m->Vl) * D * e; break;
        case LLAMA_W_ATTENTION_NORM: dst = p->attn_norm; bytes = D * 4; break;
        case LLAMA_W_WQ: dst = p->wqkv; bytes = static_cast<size_t>(m->nq) * D * e; break;
        case LLAMA_W_WK: dst = static_cast<char*>(p->wqkv) + static_cast<size_t>(m->nq) * D * e;
                         bytes = static_cast<size_t>(m->nkvc) * D * e; break;
        case LLAMA_W_WV: dst = static_cast<char*>(p->wqkv) + static_cast<size_t>(m->nq + m->nkvc) * D * e;
                         bytes = static_cast<size_t>(m->nkvc) * D * e; break;
        case LLAMA_W_WO: dst = p->wo; bytes = D * m->nq * e; break;
        case LLAMA_W_FFN_NORM: dst = p->ffn_norm; bytes = D * 4; break;
        case LLAMA_W_W2: dst = p->w2; bytes = D * m->H * e; break;
        case LLAMA_W_W1:
        case LLAMA_W_W3:
            if ((reinterpret_cast<uintptr_t>(src) & 15) != 0) { set_error("w1/w3 source must be 16-byte aligned"); return LLAMA_ERR_INVALID_ARG; }
            return launch_copy_interleave_w13(src, p->w13, m->H, m->dim, which == LLAMA_W_W3 ? 1 : 0,
                                              m->esz, st);
    }
    cudaError_t ce = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaMemcpyAsync(weight)");
    return LLAMA_OK;
}

int llama_get_kv(llama_model* m, int layer, void** k, void** v, int64_t strides[4]) {
    if (!m || layer < 0 || layer >= m->L) { set_error("bad model or layer"); return LLAMA_ERR_INVALID_ARG; }
    const size_t off = static_cast<size_t>(layer) * m->kv_layer_elems * m->esz;
    if (k) *k = static_cast<char*>(m->kc) + off;
    if (v) *v = static_cast<char*>(m->vc) + off;
    if (strides) {
        strides[0] = m->kv_row_elems;   // batch row
        strides[1] = m->hd;             // position
        strides[2] = m->kv_head_elems;  // kv head
        strides[3] = 1;                 // head dim
    }
    return LLAMA_OK;
}

}  // extern "C"

namespace llb {
// Argument checks of a prefill call and its row table (host lens).
static int prefill_rows(const Model* m, const int32_t* tokens, const int32_t* lens, int B, int T, int start_pos,
                        const float* logits, int logits_mode, RowTable* rt_out) {
    if (!m || !tokens) { set_error("model or tokens is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (B <= 0 || T <= 0 || start_pos < 0) { set_error("B and T must be positive, start_pos >= 0"); return LLAMA_ERR_INVALID_ARG; }
    if (logits_mode != 0 && logits_mode != 1) { set_error("logits_mode must be 0 or 1"); return LLAMA_ERR_INVALID_ARG; }
    if (logits_mode == 1 && !logits) { set_error("logits_mode 1 needs a logits buffer"); return LLAMA_ERR_INVALID_ARG; }
    if (logits_mode == 1 && m->tp_size > 1 && m->tp_wait) {
        set_error("a tensor-parallel rank on its own GPU returns last-token logits only (logits_mode 0)");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (B > m->Bmax) { set_error("B=%d > max_batch_size=%d", B, m->Bmax); return LLAMA_ERR_CAPACITY; }
    if (static_cast<long long>(start_pos) + T > m->S) {
        set_error("start_pos + T = %lld > max_seq_len=%d", static_cast<long long>(start_pos) + T, m->S);
        return LLAMA_ERR_CAPACITY;
    }
    RowTable& rt = *rt_out;
    rt.B = B; rt.T = T; rt.start_pos = start_pos;
    rt.cu[0] = 0;
    for (int b = 0; b < B; ++b) {
        const int len = lens ? lens[b] : T;
        if (len < 1 || len > T) { set_error("lens[%d]=%d outside [1, T=%d]", b, len, T); return LLAMA_ERR_INVALID_ARG; }
        rt.cu[b + 1] = rt.cu[b] + len;
    }
    if (rt.cu[B] > m->Mmax) { set_error("sum(lens)=%d > max_tokens=%d", rt.cu[B], m->Mmax); return LLAMA_ERR_CAPACITY; }
    return LLAMA_OK;
}

static int decode_args(const Model* m, const int32_t* tokens, const int32_t* pos, int B, const llama_sampling* sampling,
                       const float* uniforms, const int32_t* next_tokens, int flags) {
    if (!m || !tokens || !pos) { set_error("model, tokens or pos is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (B <= 0) { set_error("B must be positive"); return LLAMA_ERR_INVALID_ARG; }
    if (B > m->Bmax) { set_error("B=%d > max_batch_size=%d", B, m->Bmax); return LLAMA_ERR_CAPACITY; }
    if (sampling && !next_tokens) { set_error("sampling needs next_tokens"); return LLAMA_ERR_INVALID_ARG; }
    if (sampling && sampling->temperature < 0.f) { set_error("temperature must be >= 0"); return LLAMA_ERR_INVALID_ARG; }
    if (sampling && sampling->temperature > 0.f && !uniforms) { set_error("top-p sampling needs uniforms"); return LLAMA_ERR_INVALID_ARG; }
    if ((flags & LLAMA_DECODE_ADVANCE) && !sampling) { set_error("LLAMA_DECODE_ADVANCE needs sampling"); return LLAMA_ERR_INVALID_ARG; }
    return LLAMA_OK;
}
}  // namespace llb

extern "C" {

int llama_tp_prefill_all(llama_model* const* shards, int tp, const int32_t* tokens, const int32_t* lens, int B, int T,
                         int start_pos, float* logits, int logits_mode, void* stream) {
    Shards sh;
    LLB_TRY(group_of(nullptr, reinterpret_cast<Model* const*>(shards), tp, &sh));
    RowTable rt;
    LLB_TRY(prefill_rows(sh.m[0], tokens, lens, B, T, start_pos, logits, logits_mode, &rt));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int i = 0; i < sh.n; ++i) sh.m[i]->last_stream = st;
    return tp_prefill(sh, rt, tokens, logits, logits_mode, st);
}

int llama_tp_decode_step_all(llama_model* const* shards, int tp, const int32_t* tokens, int32_t* pos, int B,
                             const llama_sampling* sampling, const float* uniforms, int32_t* next_tokens,
                             float* logits, int flags, void* stream) {
    Shards sh;
    LLB_TRY(group_of(nullptr, reinterpret_cast<Model* const*>(shards), tp, &sh));
    LLB_TRY(decode_args(sh.m[0], tokens, pos, B, sampling, uniforms, next_tokens, flags));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int i = 0; i < sh.n; ++i) sh.m[i]->last_stream = st;
    return tp_decode(sh, tokens, pos, B, sampling, uniforms, next_tokens, logits, flags, st);
}

int llama_tp_buffers(llama_model* m, float** part0, float** part1, unsigned long long** flags, float** logits) {
    if (!m) { set_error("model is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (part0) *part0 = m->tp_part[0];
    if (part1) *part1 = m->tp_part[1];
    if (flags) *flags = m->tp_flag;
    if (logits) *logits = m->logits_ws;
    return LLAMA_OK;
}

int llama_tp_bind(llama_model* m, float* const* part0, float* const* part1, unsigned long long* const* flags,
                  float* const* logits) {
    if (!m || !part0 || !part1 || !flags || !logits) { set_error("model or buffer table is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (m->tp_size < 2) { set_error("llama_tp_bind needs a shard of a group of 2 or more ranks"); return LLAMA_ERR_INVALID_ARG; }
    for (int q = 0; q < m->tp_size; ++q) {
        if (!part0[q] || !part1[q] || !flags[q] || !logits[q]) { set_error("rank %d's buffers are NULL", q); return LLAMA_ERR_INVALID_ARG; }
        m->peers.part[q][0] = part0[q];
        m->peers.part[q][1] = part1[q];
        m->peers.flag[q] = flags[q];
        m->peers.logits[q] = logits[q];
    }
    m->tp_bound = true;
    m->tp_wait = true;
    return LLAMA_OK;
}

int llama_prefill(llama_model* m, const int32_t* tokens, const int32_t* lens, int B, int T, int start_pos,
                  float* logits, int logits_mode, void* stream) {
    if (m && m->tp_size > 1) {
        if (!m->tp_bound) { set_error("a tensor-parallel shard needs llama_tp_bind (or llama_tp_prefill_all)"); return LLAMA_ERR_INVALID_ARG; }
        RowTable rt;
        LLB_TRY(prefill_rows(m, tokens, lens, B, T, start_pos, logits, logits_mode, &rt));
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        m->last_stream = st;
        Shards sh = {{m}, 1};
        return tp_prefill(sh, rt, tokens, logits, logits_mode, st);
    }
    if (!m || !tokens) { set_error("model or tokens is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (B <= 0 || T <= 0 || start_pos < 0) { set_error("B and T must be positive, start_pos >= 0"); return LLAMA_ERR_INVALID_ARG; }
    if (logits_mode != 0 && logits_mode != 1) { set_error("logits_mode must be 0 or 1"); return LLAMA_ERR_INVALID_ARG; }
    if (logits_mode == 1 && !logits) { set_error("logits_mode 1 needs a logits buffer"); return LLAMA_ERR_INVALID_ARG; }
    if (B > m->Bmax) { set_error("B=%d > max_batch_size=%d", B, m->Bmax); return LLAMA_ERR_CAPACITY; }
    if (static_cast<long long>(start_pos) + T > m->S) {
        set_error("start_pos + T = %lld > max_seq_len=%d", static_cast<long long>(start_pos) + T, m->S);
        return LLAMA_ERR_CAPACITY;
    }
    RowTable rt;
    rt.B = B; rt.T = T; rt.start_pos = start_pos;
    rt.cu[0] = 0;
    for (int b = 0; b < B; ++b) {
        const int len = lens ? lens[b] : T;
        if (len < 1 || len > T) { set_error("lens[%d]=%d outside [1, T=%d]", b, len, T); return LLAMA_ERR_INVALID_ARG; }
        rt.cu[b + 1] = rt.cu[b] + len;
    }
    const int M = rt.cu[B];
    if (M > m->Mmax) { set_error("sum(lens)=%d > max_tokens=%d", M, m->Mmax); return LLAMA_ERR_CAPACITY; }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    m->last_stream = st;

    LLB_TRY(launch_token_map(rt, tokens, m->tok_ids, m->tok_row, m->tok_pos, m->last_idx, st));
    const bool fused = m->dtype != LLAMA_F32;
    if (fused) {
        LLB_TRY(launch_embed(m->tok_ids, m->tok_emb, m->dtype, M, m->dim, m->V, m->x, m->status, st, false, m->ssq,
                             m->y, m->layers[0].attn_norm));
    } else {
        LLB_TRY(launch_embed(m->tok_ids, m->tok_emb, m->dtype, M, m->dim, m->V, m->x, m->status, st));
    }
    for (int l = 0; l < m->L; ++l) {
        auto attn = [&]() { return launch_attention_prefill(m, l, rt, st); };
        if (fused)
            LLB_TRY(block_forward_fused(m, l, M, m->tok_row, m->tok_pos, attn, st, false, false));
        else
            LLB_TRY(block_forward(m, l, M, m->tok_row, m->tok_pos, attn, st, false));
    }
    if (!logits) return LLAMA_OK;
    Epi eo = base_epi(m);
    eo.mode = EPI_STORE_F32;
    eo.out = logits;
    eo.ldo = m->V;
    if (logits_mode == 0) {
        LLB_TRY(launch_rmsnorm(m->x, m->last_idx, m->norm, B, m->dim, m->a.norm_eps, m->ylast, m->dtype, st));
        return run_linear(m, m->dtype, m->ylast, &m->m_ylast, m->output, &m->m_output, B, m->V, m->dim, eo, st);
    }
    if (fused) {
        // every position: y and the sums of squares already hold the final norm's inputs
        const NormIO n_in = {m->ssq, m->dim / 128, m->a.norm_eps, nullptr, nullptr, nullptr};
        return run_linear(m, m->dtype, m->y, &m->m_y, m->output, &m->m_output, M, m->V, m->dim, eo, st, false, &n_in);
    }
    LLB_TRY(launch_rmsnorm(m->x, nullptr, m->norm, M, m->dim, m->a.norm_eps, m->y, m->dtype, st));
    return run_linear(m, m->dtype, m->y, &m->m_y, m->output, &m->m_output, M, m->V, m->dim, eo, st);
}

int llama_decode_step(llama_model* m, const int32_t* tokens, int32_t* pos, int B, const llama_sampling* sampling,
                      const float* uniforms, int32_t* next_tokens, float* logits, int flags, void* stream) {
    if (m && m->tp_size > 1) {
        if (!m->tp_bound) { set_error("a tensor-parallel shard needs llama_tp_bind (or llama_tp_decode_step_all)"); return LLAMA_ERR_INVALID_ARG; }
        LLB_TRY(decode_args(m, tokens, pos, B, sampling, uniforms, next_tokens, flags));
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        m->last_stream = st;
        Shards sh = {{m}, 1};
        return tp_decode(sh, tokens, pos, B, sampling, uniforms, next_tokens, logits, flags, st);
    }
    if (!m || !tokens || !pos) { set_error("model, tokens or pos is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (B <= 0) { set_error("B must be positive"); return LLAMA_ERR_INVALID_ARG; }
    if (B > m->Bmax) { set_error("B=%d > max_batch_size=%d", B, m->Bmax); return LLAMA_ERR_CAPACITY; }
    if (sampling && !next_tokens) { set_error("sampling needs next_tokens"); return LLAMA_ERR_INVALID_ARG; }
    if (sampling && sampling->temperature < 0.f) { set_error("temperature must be >= 0"); return LLAMA_ERR_INVALID_ARG; }
    if (sampling && sampling->temperature > 0.f && !uniforms) { set_error("top-p sampling needs uniforms"); return LLAMA_ERR_INVALID_ARG; }
    if ((flags & LLAMA_DECODE_ADVANCE) && !sampling) { set_error("LLAMA_DECODE_ADVANCE needs sampling"); return LLAMA_ERR_INVALID_ARG; }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    m->last_stream = st;

    float* lg = logits ? logits : m->logits_ws;
    Epi eo = base_epi(m);
    eo.mode = EPI_STORE_F32;
    eo.out = lg;
    eo.ldo = m->V;
    // 16-bit models fold RMSNorm into the projections (block_forward_fused).
    // Steps of up to 64 rows run the decode chain: the weight-streaming
    // projections, every kernel launched early (programmatic dependent
    // launch) and waiting for its predecessor before reading its outputs, and
    // the greedy pick inside the vocabulary projection.  Wider steps run the
    // 128 x 256-tile projections, launched one after another; fp32 models run
    // RMSNorm kernels and the SIMT projections.
    const bool chain = m->dtype != LLAMA_F32 && B <= kFusedDecodeRows;
    if (m->dtype != LLAMA_F32) {
        LLB_TRY(launch_embed(tokens, m->tok_emb, m->dtype, B, m->dim, m->V, m->x, m->status, st, chain, m->ssq, m->y,
                             m->layers[0].attn_norm, tl_next(m, TL_EMBED, 2LL * B * m->dim)));
        for (int l = 0; l < m->L; ++l) {
            auto attn = [&]() {
                int stall_unit = -1;
                long long stall_wait = 0;
                take_stall(m, LLAMA_STALL_ATTENTION, &stall_unit, &stall_wait);
                return launch_attention_decode(m, l, pos, B, st, chain, tl_next(m, TL_ATTENTION, 0), stall_wait,
                                               stall_unit);
            };
            LLB_TRY(block_forward_fused(m, l, B, nullptr, pos, attn, st, chain, true));
        }
        const NormIO n_in = {m->ssq, m->dim / 128, m->a.norm_eps, nullptr, nullptr, nullptr};
        const bool adv = (flags & LLAMA_DECODE_ADVANCE) != 0;
        if (chain && sampling && sampling->temperature == 0.f) {
            // greedy: the output projection picks the next tokens itself
            // (Admin Guide §8.5, argmax at temperature 0); logits are stored
            // only when the caller asked for them
            Epi eg = base_epi(m);
            eg.mode = EPI_LOGITS_ARGMAX;
            eg.out = logits;
            eg.ldo = m->V;
            eg.best = m->best;
            eg.done = m->step_cnt;
            eg.next = next_tokens;
            eg.tok_adv = adv ? const_cast<int32_t*>(tokens) : nullptr;
            eg.pos_adv = adv ? pos : nullptr;
            return run_linear(m, m->dtype, m->y, &m->m_y, m->output, &m->m_output, B, m->V, m->dim, eg, st, true,
                              &n_in, true);
        }
        LLB_TRY(run_linear(m, m->dtype, m->y, &m->m_y, m->output, &m->m_output, B, m->V, m->dim, eo, st, chain,
                           &n_in, true));
    } else {
        LLB_TRY(launch_embed(tokens, m->tok_emb, m->dtype, B, m->dim, m->V, m->x, m->status, st, false, nullptr,
                             nullptr, nullptr, tl_next(m, TL_EMBED, 2LL * B * m->dim)));
        for (int l = 0; l < m->L; ++l) {
            auto attn = [&]() { return launch_attention_decode(m, l, pos, B, st, false, tl_next(m, TL_ATTENTION, 0)); };
            LLB_TRY(block_forward(m, l, B, nullptr, pos, attn, st, false, true));
        }
        LLB_TRY(launch_rmsnorm(m->x, nullptr, m->norm, B, m->dim, m->a.norm_eps, m->ylast, m->dtype, st, false,
                               tl_next(m, TL_RMSNORM, 0)));
        LLB_TRY(run_linear(m, m->dtype, m->ylast, &m->m_ylast, m->output, &m->m_output, B, m->V, m->dim, eo, st,
                           false, nullptr, true));
    }
    if (!sampling) return LLAMA_OK;
    const bool pdl = chain;
    const bool adv = (flags & LLAMA_DECODE_ADVANCE) != 0;
    int32_t* tok_adv = adv ? const_cast<int32_t*>(tokens) : nullptr;
    int32_t* pos_adv = adv ? pos : nullptr;
    unsigned long long* tls = tl_next(m, TL_SAMPLE, 4LL * B * m->V);
    if (sampling->temperature == 0.f) return launch_argmax(lg, B, m->V, next_tokens, tok_adv, pos_adv, st, pdl, tls);
    return launch_top_p(lg, B, m->V, sampling->temperature, sampling->top_p, uniforms, next_tokens, tok_adv,
                        pos_adv, st, pdl, tls);
}

int llama_sample(const float* logits, int B, int V, float temperature, float top_p, const float* uniforms,
                 int32_t* out, void* stream) {
    if (!logits || !out) { set_error("logits or out is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (B <= 0 || V <= 0 || V > 262144) { set_error("B must be positive and 0 < V <= 262144"); return LLAMA_ERR_INVALID_ARG; }
    if (!(temperature >= 0.f)) { set_error("temperature must be >= 0"); return LLAMA_ERR_INVALID_ARG; }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (temperature == 0.f) return launch_argmax(logits, B, V, out, nullptr, nullptr, st);
    if (!uniforms) { set_error("top-p sampling needs uniforms"); return LLAMA_ERR_INVALID_ARG; }
    if (!(top_p >= 0.f)) { set_error("top_p must be >= 0"); return LLAMA_ERR_INVALID_ARG; }
    return launch_top_p(logits, B, V, temperature, top_p, uniforms, out, nullptr, nullptr, st);
}

int llama_token_logprobs(const float* logits, const int32_t* tokens, int N, int V, float* out, void* stream) {
    if (!logits || !tokens || !out) { set_error("logits, tokens or out is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (N < 0 || V <= 0) { set_error("N must be >= 0 and V positive"); return LLAMA_ERR_INVALID_ARG; }
    if (N == 0) return LLAMA_OK;
    return launch_logprobs(logits, tokens, N, V, out, static_cast<cudaStream_t>(stream));
}

int llama_model_status(llama_model* m, int* device_status) {
    if (!m || !device_status) { set_error("model or device_status is NULL"); return LLAMA_ERR_INVALID_ARG; }
    cudaError_t e = cudaStreamSynchronize(m->last_stream);
    if (e == cudaSuccess) e = cudaMemcpy(device_status, m->status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(m->status, 0, sizeof(int));
    // A kernel that gave up on a wait left without adding to, or clearing,
    // the arrival counters of its split tiles and split attention pairs; the
    // next launches would pick the wrong last arrival.  Nothing is in flight
    // here (the stream was synchronised), so start them all at zero again.
    if (e == cudaSuccess && *device_status != 0) {
        e = cudaMemset(m->gemm_cnt, 0, kMaxTiles * sizeof(int));
        if (e == cudaSuccess) e = cudaMemset(m->attn_cnt, 0, static_cast<size_t>(m->Bmax) * m->nkv * sizeof(int));
        if (e == cudaSuccess) e = cudaMemset(m->best, 0, static_cast<size_t>(m->Bmax) * 8);
        if (e == cudaSuccess) e = cudaMemset(m->step_cnt, 0, kStepCounters * sizeof(int));
    }
    if (e != cudaSuccess) return cuda_fail(e, "llama_model_status");
    return LLAMA_OK;
}

int llama_model_destroy(llama_model* m) {
    if (m) profile_release(m->prof);
    delete m;
    return LLAMA_OK;
}

int llama_debug_stall(llama_model* m, int which, int unit, int64_t wait_limit_ns) {
    if (!m) { set_error("model is NULL"); return LLAMA_ERR_INVALID_ARG; }
    if (which != LLAMA_STALL_NONE && which != LLAMA_STALL_PROJECTION && which != LLAMA_STALL_ATTENTION) {
        set_error("which must be LLAMA_STALL_NONE, _PROJECTION or _ATTENTION");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (which != LLAMA_STALL_NONE && (unit < 0 || wait_limit_ns < 1000 || wait_limit_ns > 2000000000LL)) {
        set_error("unit must be >= 0 and the wait limit between 1 us and 2 s");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (which != LLAMA_STALL_NONE && m->dtype == LLAMA_F32) {
        set_error("the stall is a feature of the 16-bit decode kernels");
        return LLAMA_ERR_INVALID_ARG;
    }
    m->dbg_kind = which;
    m->dbg_unit = unit;
    m->dbg_wait_ns = wait_limit_ns;
    return LLAMA_OK;
}

int llama_timeline_start(llama_model* m, void* stream) {
    if (!m) { set_error("model is NULL"); return LLAMA_ERR_INVALID_ARG; }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(m->tl_end, 0, static_cast<size_t>(kTimelineCap) * 8, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(timeline)");
    m->last_stream = st;
    m->tl_kind.clear();
    m->tl_bytes.clear();
    m->tl_n = 0;
    m->tl_on = true;
    return LLAMA_OK;
}

int llama_timeline_stop(llama_model* m, uint64_t* end_ns, int32_t* kind, int64_t* bytes, int max, int* n) {
    if (!m || max < 0) { set_error("bad timeline arguments"); return LLAMA_ERR_INVALID_ARG; }
    m->tl_on = false;
    const int cnt = m->tl_n < max ? m->tl_n : max;
    cudaError_t e = cudaStreamSynchronize(m->last_stream);
    if (e == cudaSuccess && end_ns && cnt > 0)
        e = cudaMemcpy(end_ns, m->tl_end, static_cast<size_t>(cnt) * 8, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "llama_timeline_stop");
    for (int i = 0; i < cnt; ++i) {
        if (kind) kind[i] = m->tl_kind[i];
        if (bytes) bytes[i] = m->tl_bytes[i];
    }
    if (n) *n = cnt;
    return LLAMA_OK;
}

int llama_profile_start(llama_model* m, int capacity) {
    if (!m || capacity <= 0) { set_error("bad profile arguments"); return LLAMA_ERR_INVALID_ARG; }
    profile_release(m->prof);
    m->prof.ev.resize(2 * static_cast<size_t>(capacity), nullptr);
    for (auto& e : m->prof.ev) {
        cudaError_t ce = cudaEventCreate(&e);
        if (ce != cudaSuccess) {
            profile_release(m->prof);
            return cuda_fail(ce, "cudaEventCreate(profile)");
        }
    }
    m->prof.bytes.assign(static_cast<size_t>(capacity), 0);
    m->prof.flops.assign(static_cast<size_t>(capacity), 0);
    m->prof.rows.assign(static_cast<size_t>(capacity), 0);
    m->prof.capacity = capacity;
    m->prof.n = 0;
    return LLAMA_OK;
}

int llama_profile_stop(llama_model* m, float* ms, int64_t* bytes, int64_t* flops, int32_t* rows, int max, int* n) {
    if (!m) { set_error("model is NULL"); return LLAMA_ERR_INVALID_ARG; }
    Profile& p = m->prof;
    const int cnt = p.n < max ? p.n : max;
    int rc = LLAMA_OK;
    for (int i = 0; i < cnt && rc == LLAMA_OK; ++i) {
        cudaError_t e = cudaEventSynchronize(p.ev[2 * i + 1]);
        float t = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, p.ev[2 * i], p.ev[2 * i + 1]);
        if (e != cudaSuccess) rc = cuda_fail(e, "profile events");
        if (ms) ms[i] = t;
        if (bytes) bytes[i] = p.bytes[i];
        if (flops) flops[i] = p.flops[i];
        if (rows) rows[i] = p.rows[i];
    }
    if (n) *n = cnt;
    profile_release(p);
    return rc;
}

// ---------------------------------------------------------------- single-kernel ops
int llama_op_rmsnorm(const float* x, const float* w, int M, int dim, float eps, void* out, int out_dtype,
                     void* stream) {
    if (!x || !w || !out || M < 0 || dim <= 0 || dim % 4) { set_error("bad rmsnorm arguments"); return LLAMA_ERR_INVALID_ARG; }
    if (out_dtype != LLAMA_F32 && out_dtype != LLAMA_BF16 && out_dtype != LLAMA_F16) { set_error("bad out_dtype"); return LLAMA_ERR_INVALID_ARG; }
    return launch_rmsnorm(x, nullptr, w, M, dim, eps, out, out_dtype, static_cast<cudaStream_t>(stream));
}

size_t llama_op_linear_workspace_bytes(void) { return kGemmPartBytes + kMaxTiles * sizeof(int); }

int llama_op_linear(const void* A, const void* W, int M, int N, int K, int dtype, float* out, void* workspace,
                    size_t workspace_bytes, void* stream) {
    if (!A || !W || !out || M < 0 || N <= 0 || K <= 0) { set_error("bad linear arguments"); return LLAMA_ERR_INVALID_ARG; }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Epi ep;
    memset(&ep, 0, sizeof(ep));
    ep.mode = EPI_STORE_F32;
    ep.out = out;
    ep.ldo = N;
    if (dtype == LLAMA_F32)
        return linear_f32(static_cast<const float*>(A), static_cast<const float*>(W), M, N, K, ep, st);
    if (dtype != LLAMA_BF16 && dtype != LLAMA_F16) { set_error("bad dtype"); return LLAMA_ERR_INVALID_ARG; }
    if (K % 8) { set_error("16-bit linear needs K %% 8 == 0"); return LLAMA_ERR_INVALID_ARG; }
    if ((N + 127) / 128 > kMaxTiles) { set_error("N too large"); return LLAMA_ERR_INVALID_ARG; }
    if ((M <= 64 || workspace) && (!workspace || workspace_bytes < llama_op_linear_workspace_bytes() ||
                                   (reinterpret_cast<uintptr_t>(workspace) & 255))) {
        set_error("16-bit linear needs a 256-byte aligned workspace of llama_op_linear_workspace_bytes() "
                  "(optional only for M > 64)");
        return LLAMA_ERR_INVALID_ARG;
    }
    if (M == 0) return LLAMA_OK;
    TmaMaps ma, mw;
    LLB_TRY(encode_kmajor_16(&ma.a128, A, M, K, 128, dtype));
    LLB_TRY(encode_kmajor_16(&ma.b, A, M, K, 16, dtype));
    LLB_TRY(encode_kmajor_16(&mw.a128, W, N, K, 128, dtype));
    LLB_TRY(encode_kmajor_16(&mw.b, W, N, K, 256, dtype));
    float* part = static_cast<float*>(workspace);
    int* cnt = workspace ? reinterpret_cast<int*>(static_cast<char*>(workspace) + kGemmPartBytes) : nullptr;
    return linear16(&ma, &mw, M, N, K, dtype, ep, part, part ? kGemmPartBytes : 0, cnt, st);
}

}  // extern "C"
