"""fp64 CPU oracle of the Llama-2 decoder forward pass with a KV cache, plus
greedy and top-p sampling.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never calls it and shares no code with
it.

It is the plain definition, written out: numpy float64 arithmetic, library
matmul/exp/sort as single steps, no blocking, fusion or reordering.  Every
function names the passage it follows.  Citations are to the two guides for
the meta-llama/llama repository ("Llama 2 Reference Implementation —
Administrator & Developer Guide", called *Admin Guide* below, and the
companion *User Guide*) and to the pyshine.com source tour ("meta-llama/llama
source tour").

Readings taken where the pages leave a step open (each one is listed again
in the design notes):
  * RoPE frequencies are the standard theta^(-2j/head_dim); pairs are the
    adjacent reals (2j, 2j+1) viewed as one complex number.  The pages fix
    only theta and the complex-pair view.  Parity of the frequency schedule
    is pinned by the textbook definition only ("parity unpinned" against the
    pages for the schedule itself).
  * repeat_kv maps query head h to KV head floor(h / n_rep).
  * Argmax ties go to the lowest token id.
  * top-p orders tokens by probability descending, equal probabilities by id
    ascending; a token is kept iff the mass strictly before it is <= top_p;
    the draw is the inverse CDF of the renormalised kept mass at the given
    uniform u (the multinomial draw made deterministic).
  * 16-bit storage (optional, `store=`): the reference holds its tensors in
    fp16 (Admin Guide §1.4, §6.4; RMSNorm normalises in fp32 and casts back,
    §8.4).  The oracle can round to bfloat16 or binary16 where a 16-bit run
    stores activations, leaving every sum exact; this measures the error that
    storage alone causes and is never the parity reference itself.

Weights are passed as a mapping:
  w["tok_embeddings"] [V, dim], w["norm"] [dim], w["output"] [V, dim],
  w["layers"][l][name] for name in attention_norm [dim], wq [nh*hd, dim],
  wk [nkv*hd, dim], wv [nkv*hd, dim], wo [dim, nh*hd], ffn_norm [dim],
  w1 [H, dim], w2 [dim, H], w3 [H, dim]   (nn.Linear layout: y = x W^T).
Any array-like works; each one is upcast to float64 at the point of use.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# 16-bit storage (an error model, used only when a caller asks for it)
# ---------------------------------------------------------------------------

def round_bf16(a) -> np.ndarray:
    """Round to the nearest bfloat16 value, ties to even, returned as fp64.

    bfloat16 is the upper half of an IEEE binary32 (sign, 8 exponent bits,
    7 fraction bits).  The value is first rounded to binary32 (as an fp32
    accumulator holds it), then the low 16 bits of that word are rounded off:
    add 0x7FFF plus the lowest kept bit, and clear them.  Finite inputs only.
    """
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32)
    u = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) & np.uint32(0xFFFF0000)
    return u.view(np.float32).astype(np.float64)


def round_f16(a) -> np.ndarray:
    """Round to the nearest IEEE binary16 value (the reference's own storage
    type, Admin Guide §1.4 and §6.4), ties to even, returned as fp64; the
    value passes through binary32 first, as above."""
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# Sizes
# ---------------------------------------------------------------------------

def ffn_hidden_dim(dim: int, multiple_of: int, ffn_dim_multiplier: Optional[float] = None) -> int:
    """SwiGLU hidden width.

    Admin Guide §8.4 (FeedForward): start from 4*dim, take int(2*hidden/3),
    optionally multiply by ffn_dim_multiplier (truncating), then round up to
    the next multiple of multiple_of.
    """
    hidden = 4 * dim
    hidden = int(2 * hidden / 3)
    if ffn_dim_multiplier is not None and ffn_dim_multiplier > 0:
        hidden = int(ffn_dim_multiplier * hidden)
    return multiple_of * ((hidden + multiple_of - 1) // multiple_of)


def kv_cache_bytes_per_tensor(max_batch_size: int, max_seq_len: int, n_kv_heads: int,
                              head_dim: int, bytes_per_elem: int) -> int:
    """Bytes of one cache tensor (cache_k or cache_v) of one layer.

    Admin Guide §6.2: shape (max_batch_size, max_seq_len, n_local_kv_heads, head_dim).
    """
    return max_batch_size * max_seq_len * n_kv_heads * head_dim * bytes_per_elem


def parameter_count(dim: int, n_layers: int, n_heads: int, n_kv_heads: int, vocab_size: int,
                    hidden: int) -> int:
    """Number of learned parameters (Admin Guide §8.4: Transformer, Attention,
    FeedForward, two RMSNorms per block, a final RMSNorm; embedding and output
    are separate modules; no biases anywhere — source tour, "One model.py")."""
    hd = dim // n_heads
    per_layer = (dim * n_heads * hd + 2 * dim * n_kv_heads * hd + n_heads * hd * dim  # wq wk wv wo
                 + 3 * dim * hidden                                               # w1 w2 w3
                 + 2 * dim)                                                       # two norms
    return vocab_size * dim * 2 + n_layers * per_layer + dim


# ---------------------------------------------------------------------------
# Building blocks
# ---------------------------------------------------------------------------

def rms_norm(x, weight, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x * 1/sqrt(mean(x^2) + eps), times weight.

    Admin Guide §8.4 (RMSNorm): no mean subtraction, no bias.  The reference
    computes the normalisation in fp32 and casts back before the weight; the
    oracle computes all of it in fp64.
    """
    x = _f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * _f64(weight)


def rope_frequencies(head_dim: int, theta: float) -> np.ndarray:
    """freq_j = theta^(-2j/head_dim), j = 0 .. head_dim/2 - 1.

    Admin Guide §8.4 (RoPE, precompute_freqs_cis): a table of e^{i t freq}
    of shape (end, head_dim/2) with theta = 10000; the schedule itself is the
    standard rotary one (a reading; the pages print no formula).
    """
    j = np.arange(head_dim // 2, dtype=np.float64)
    return np.float64(theta) ** (-2.0 * j / head_dim)


def apply_rope(v, positions, theta: float) -> np.ndarray:
    """Rotate each adjacent pair (v[2j], v[2j+1]) by the angle pos*freq_j.

    v: [T, n_heads, head_dim]; positions: [T].  The pair is read as the
    complex number v[2j] + i v[2j+1] and multiplied by e^{i pos freq_j}
    (Admin Guide §8.4, apply_rotary_emb; source tour, "One model.py").
    """
    v = _f64(v)
    T, nh, hd = v.shape
    ang = _f64(positions)[:, None] * rope_frequencies(hd, theta)[None, :]   # [T, hd/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    re = v[..., 0::2]
    im = v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = re * c - im * s
    out[..., 1::2] = re * s + im * c
    return out


def softmax(s, axis: int = -1) -> np.ndarray:
    """exp(s - max) / sum(exp(s - max)); -inf entries get probability 0."""
    s = _f64(s)
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def causal_mask(seqlen: int, start_pos: int) -> np.ndarray:
    """(seqlen, start_pos+seqlen) mask: 0 where key j <= start_pos + t, -inf above.

    Admin Guide §8.4 (the NOTE on mask construction in Transformer.forward):
    the cached prefix is fully visible; the new-token block is causal.
    """
    t = np.arange(seqlen)[:, None]
    j = np.arange(start_pos + seqlen)[None, :]
    m = np.zeros((seqlen, start_pos + seqlen), dtype=np.float64)
    m[j > start_pos + t] = -np.inf
    return m


def attention(q, keys, values, start_pos: int, n_rep: int, store=None) -> np.ndarray:
    """softmax(Q K^T / sqrt(head_dim) + mask) V for each query head.

    q: [T, n_heads, hd] (already rotated); keys/values: [start_pos+T, n_kv_heads, hd]
    (the whole cache prefix, already holding this call's keys).  Query head h
    reads KV head h // n_rep (repeat_kv; source tour, "One model.py").
    Admin Guide §8.4, Attention forward steps 5-7.  `store` (see
    layer_forward) rounds the probabilities before they multiply V.
    """
    q, keys, values = _f64(q), _f64(keys), _f64(values)
    T, nh, hd = q.shape
    mask = causal_mask(T, start_pos)
    out = np.empty((T, nh, hd), dtype=np.float64)
    for h in range(nh):
        g = h // n_rep
        scores = q[:, h, :] @ keys[:, g, :].T / math.sqrt(hd) + mask
        p = softmax(scores, axis=-1)
        if store is not None:
            p = store(p)
        out[:, h, :] = p @ values[:, g, :]
    return out


def silu(z) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + e^{-z})."""
    z = _f64(z)
    return z / (1.0 + np.exp(-z))


def feed_forward(x, w1, w2, w3, store=None) -> np.ndarray:
    """SwiGLU: w2(silu(w1 x) * w3 x)  (Admin Guide §8.4, FeedForward).
    `store` (see layer_forward) rounds the gated product before w2."""
    x = _f64(x)
    g = silu(x @ _f64(w1).T) * (x @ _f64(w3).T)
    if store is not None:
        g = store(g)
    return g @ _f64(w2).T


# ---------------------------------------------------------------------------
# Model with a KV cache (one batch row at a time: rows never interact)
# ---------------------------------------------------------------------------

class KVCache:
    """cache_k / cache_v of one batch row: per layer [max_seq_len, n_kv_heads, head_dim],
    zero-initialised (Admin Guide §6.2 and §8.4, Attention)."""

    def __init__(self, n_layers: int, max_seq_len: int, n_kv_heads: int, head_dim: int):
        self.k = [np.zeros((max_seq_len, n_kv_heads, head_dim)) for _ in range(n_layers)]
        self.v = [np.zeros((max_seq_len, n_kv_heads, head_dim)) for _ in range(n_layers)]


class Args:
    """The structural fields of ModelArgs (Admin Guide §3.3)."""

    def __init__(self, dim, n_layers, n_heads, n_kv_heads=None, vocab_size=-1, multiple_of=256,
                 ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0, max_seq_len=2048):
        self.dim = dim
        self.n_layers = n_layers
        self.n_heads = n_heads
        self.n_kv_heads = n_heads if not n_kv_heads else n_kv_heads
        assert n_heads % self.n_kv_heads == 0 and dim % n_heads == 0
        self.vocab_size = vocab_size
        self.multiple_of = multiple_of
        self.ffn_dim_multiplier = ffn_dim_multiplier
        self.norm_eps = norm_eps
        self.rope_theta = rope_theta
        self.max_seq_len = max_seq_len
        self.head_dim = dim // n_heads
        self.n_rep = n_heads // self.n_kv_heads
        self.hidden = ffn_hidden_dim(dim, multiple_of, ffn_dim_multiplier)


def new_cache(args: Args) -> KVCache:
    return KVCache(args.n_layers, args.max_seq_len, args.n_kv_heads, args.head_dim)


def layer_forward(args: Args, lw, x, cache: KVCache, layer: int, start_pos: int, store=None) -> np.ndarray:
    """One pre-norm TransformerBlock on the T new tokens of one row.

    h = x + attention(attention_norm(x)); out = h + feed_forward(ffn_norm(h))
    (Admin Guide §8.4, TransformerBlock).  The attention writes this call's
    keys and values into cache rows start_pos .. start_pos+T-1 and reads rows
    0 .. start_pos+T-1 (Admin Guide §8.4, Attention forward steps 1-8).

    store: None for the exact fp64 definition.  Otherwise a rounding function
    (round_bf16, round_f16) applied where a 16-bit run holds its activations
    in the 16-bit type: the normalised inputs of the projections, q, k and v
    after RoPE (so the cache holds 16-bit values), the attention
    probabilities and output, and the SwiGLU product; the residual stream and
    every sum stay exact.  It gives the error that 16-bit storage alone
    causes, which the parity bounds at full model depth are derived from.
    """
    x = _f64(x)
    T = x.shape[0]
    nh, nkv, hd = args.n_heads, args.n_kv_heads, args.head_dim
    keep = store if store is not None else (lambda a: a)
    pos = start_pos + np.arange(T)
    y = keep(rms_norm(x, lw["attention_norm"], args.norm_eps))
    q = (y @ _f64(lw["wq"]).T).reshape(T, nh, hd)
    k = (y @ _f64(lw["wk"]).T).reshape(T, nkv, hd)
    v = keep((y @ _f64(lw["wv"]).T).reshape(T, nkv, hd))
    q = keep(apply_rope(q, pos, args.rope_theta))
    k = keep(apply_rope(k, pos, args.rope_theta))
    cache.k[layer][start_pos:start_pos + T] = k
    cache.v[layer][start_pos:start_pos + T] = v
    keys = cache.k[layer][:start_pos + T]
    values = cache.v[layer][:start_pos + T]
    o = keep(attention(q, keys, values, start_pos, args.n_rep, store).reshape(T, nh * hd))
    h = x + o @ _f64(lw["wo"]).T
    f = keep(rms_norm(h, lw["ffn_norm"], args.norm_eps))
    return h + feed_forward(f, lw["w1"], lw["w2"], lw["w3"], store)


def forward(args: Args, w, tokens: Sequence[int], start_pos: int, cache: KVCache,
            n_layers: Optional[int] = None, logits_positions: Optional[Sequence[int]] = None,
            store=None) -> np.ndarray:
    """Transformer.forward(tokens, start_pos) for one batch row.

    Embedding lookup, the blocks, the final RMSNorm, the output projection;
    returns fp64 logits [T, V] for every new position (or only for the
    positions listed in `logits_positions`, indices into this call's tokens).
    Admin Guide §8.4 ("The forward pass", steps 1-6).  `store`: see
    layer_forward (it also rounds the final normalised rows).
    """
    toks = np.asarray(tokens, dtype=np.int64)
    x = _f64(w["tok_embeddings"][toks])
    layers = w["layers"]
    L = args.n_layers if n_layers is None else n_layers
    for l in range(L):
        x = layer_forward(args, layers[l], x, cache, l, start_pos, store)
    if logits_positions is not None:
        x = x[np.asarray(logits_positions, dtype=np.int64)]
    h = rms_norm(x, w["norm"], args.norm_eps)
    if store is not None:
        h = store(h)
    return h @ _f64(w["output"]).T


# ---------------------------------------------------------------------------
# Sampling
# ---------------------------------------------------------------------------

def greedy(logits) -> int:
    """argmax over the vocabulary, lowest id on ties (Admin Guide §8.5)."""
    return int(np.argmax(_f64(logits)))  # numpy returns the first maximum


def sampling_order(logits) -> np.ndarray:
    """Token ids by probability descending, equal probabilities by id ascending.

    softmax(l/T) is strictly increasing in the logit, so the exact order of
    the probabilities is the order of the logits.
    """
    l = _f64(logits)
    return np.lexsort((np.arange(l.shape[0]), -l))


def top_p_probs(logits, temperature: float) -> np.ndarray:
    """softmax(logits / temperature) in fp64 (Admin Guide §8.5)."""
    l = _f64(logits)
    return softmax((l - l.max()) / np.float64(temperature))


def sample_top_p(logits, temperature: float, top_p: float, u: float) -> int:
    """Nucleus sampling with the draw made deterministic by a given uniform u in [0,1).

    Follows sample_top_p as the source tour ("Sampling, Stopping, and the
    Chat Template") and the Admin Guide §6.3 / §8.5 describe it: sort the
    probabilities descending, zero every token whose preceding cumulative
    mass already exceeds top_p, renormalise, draw.  The draw is the inverse
    CDF: the first kept token whose inclusive cumulative mass exceeds u*Z,
    Z the kept mass (or the last kept token if rounding leaves none).
    temperature == 0 is the greedy argmax.
    """
    if temperature == 0:
        return greedy(logits)
    p = top_p_probs(logits, temperature)
    order = sampling_order(logits)
    ps = p[order]
    inclusive = np.cumsum(ps)
    exclusive = inclusive - ps
    kept = int(np.count_nonzero(exclusive <= np.float64(top_p)))
    kept = max(kept, 1)
    z = inclusive[kept - 1]
    target = np.float64(u) * z
    idx = int(np.searchsorted(inclusive[:kept], target, side="right"))
    if idx >= kept:
        idx = kept - 1
    return int(order[idx])


def top_p_kept(logits, temperature: float, top_p: float) -> List[int]:
    """The kept set of sample_top_p, in sampling order (for tests)."""
    p = top_p_probs(logits, temperature)
    order = sampling_order(logits)
    ps = p[order]
    exclusive = np.cumsum(ps) - ps
    kept = max(int(np.count_nonzero(exclusive <= np.float64(top_p))), 1)
    return [int(i) for i in order[:kept]]


def sample_margins(logits, temperature: float, top_p: float, u: float) -> float:
    """How far (relative to the kept mass) this draw sits from a decision
    boundary of sample_top_p.  A float-rounding difference can change the
    returned index only when this is tiny or negative.

    Two boundaries matter: the cumulative masses the draw target u*Z is
    compared with, and the nucleus edge.  A token whose preceding mass lies
    within 1e-9 of top_p may be kept or dropped by rounding; that moves Z, and
    so the draw target, by at most that token's own mass, which is subtracted
    from the draw margin.  For temperature 0 it is the top-2 logit gap.
    """
    if temperature == 0:
        l = np.sort(_f64(logits))[::-1]
        return float(l[0] - l[1]) if l.shape[0] > 1 else math.inf
    p = top_p_probs(logits, temperature)
    order = sampling_order(logits)
    ps = p[order]
    inclusive = np.cumsum(ps)
    exclusive = inclusive - ps
    kept = max(int(np.count_nonzero(exclusive <= np.float64(top_p))), 1)
    z = inclusive[kept - 1]
    target = np.float64(u) * z
    m = float(np.min(np.abs(inclusive[:kept] - target)) / z)
    near = np.abs(exclusive - np.float64(top_p)) < 1e-9
    near[0] = False   # the first token is always kept
    if near.any():
        m -= float(ps[near].sum() / z)
    return m


def token_logprobs(logits, tokens) -> np.ndarray:
    """log softmax(logits[i])[tokens[i]] for each row i, in fp64: the
    per-token log-probabilities generate returns (Admin Guide §8.5)."""
    lg = _f64(logits)
    m = lg.max(axis=-1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(lg - m).sum(axis=-1))
    return lg[np.arange(lg.shape[0]), np.asarray(tokens, dtype=np.int64)] - lse


def generate(args: Args, w, prompts: Sequence[Sequence[int]], max_gen_len: Optional[int] = None,
             temperature: float = 0.6, top_p: float = 0.9, uniforms=None, logprobs: bool = False,
             echo: bool = False, eos_id: Optional[int] = None):
    """The generation loop of the reference (Admin Guide §8.5; User Guide §1
    and the per-call parameters of §3.4; source tour, "The decode loop in
    generate"), one row at a time with its own KV cache.

    All rows advance through the same positions: prompts are right-padded into
    a (rows, total_len) table; the first forward runs the first min(prompt
    lengths) tokens of every row; then, for each later position, one forward
    over the slice not yet consumed, a greedy or nucleus choice for the next
    position, which keeps the prompt's own token where the row's prompt still
    covers that position; a row has finished once it produced EOS outside its
    prompt, and the loop ends early when every row has.

    Readings of what the pages leave open (the GPU driver takes the same):
    total_len = min(max_seq_len, max_gen_len + longest prompt), max_gen_len
    defaulting to max_seq_len - 1; the draw for position p of row b uses
    uniforms[p][b]; the log-probability of the token at position p is the
    log-softmax (of the raw logits, not temperature-scaled) at that token of
    the logits that predict p, and 0 for position 0, which nothing predicts; a
    row's result runs from position 0 (echo) or from the end of its prompt up
    to prompt length + max_gen_len, cut before the first EOS at or after the
    end of its prompt.  Returns (token lists, log-probability lists or None).
    """
    B = len(prompts)
    S = args.max_seq_len
    if max_gen_len is None:
        max_gen_len = S - 1
    lens = [len(p) for p in prompts]
    assert B >= 1 and min(lens) >= 1 and max(lens) <= S
    total = min(S, max_gen_len + max(lens))
    pad = -1
    tok = np.full((B, total), pad, dtype=np.int64)
    for b, p in enumerate(prompts):
        tok[b, :len(p)] = p
    in_prompt = tok != pad
    lp = np.zeros((B, total))
    caches = [new_cache(args) for _ in range(B)]
    done = np.zeros(B, dtype=bool)
    start = min(lens)
    if start == total:
        # nothing to generate: only the prompts' log-probabilities
        for b in range(B):
            lg = forward(args, w, tok[b, :total].tolist(), 0, caches[b])
            lp[b, 1:total] = token_logprobs(lg[:-1], tok[b, 1:total])
    prev = 0
    for cur in range(start, total):
        for b in range(B):
            lg = forward(args, w, tok[b, prev:cur].tolist(), prev, caches[b])   # rows predict prev+1 .. cur
            if in_prompt[b, cur]:
                nxt = int(tok[b, cur])
            elif temperature > 0:
                nxt = sample_top_p(lg[-1], temperature, top_p, float(uniforms[cur][b]))
            else:
                nxt = greedy(lg[-1])
            tok[b, cur] = nxt
            lp[b, prev + 1:cur + 1] = token_logprobs(lg, tok[b, prev + 1:cur + 1])
            if eos_id is not None and not in_prompt[b, cur] and nxt == eos_id:
                done[b] = True
        prev = cur
        if eos_id is not None and done.all():
            break
    out_tok, out_lp = [], []
    for b in range(B):
        first = 0 if echo else lens[b]
        last = min(total, lens[b] + max_gen_len)
        t = tok[b, first:last].tolist()
        l = lp[b, first:last].tolist()
        if eos_id is not None:
            for i in range(max(0, lens[b] - first), len(t)):
                if t[i] == eos_id:
                    t, l = t[:i], l[:i]
                    break
        out_tok.append(t)
        out_lp.append(l)
    return out_tok, (out_lp if logprobs else None)
