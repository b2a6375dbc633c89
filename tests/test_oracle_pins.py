"""Pins of the CPU oracle to facts the pages and mathematics fix (CPU only).

Each test names the plausible oracle mistake it would catch.  Sources: the
two meta-llama/llama guides (Admin Guide, User Guide) and the pyshine.com
source tour; see each test's docstring.
"""
import math
import os
import re

import numpy as np
import pytest

from oracle import llama_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny_args(n_layers=2, n_heads=4, n_kv_heads=2, dim=32, vocab=40, max_seq_len=32, mult=None,
               multiple_of=16):
    return O.Args(dim=dim, n_layers=n_layers, n_heads=n_heads, n_kv_heads=n_kv_heads,
                  vocab_size=vocab, multiple_of=multiple_of, ffn_dim_multiplier=mult,
                  norm_eps=1e-5, rope_theta=10000.0, max_seq_len=max_seq_len)


def _rand_weights(args, seed=0, scale=0.2):
    rng = np.random.default_rng(seed)
    hd, H = args.head_dim, args.hidden
    n = lambda *s: rng.standard_normal(s) * scale
    w = {"tok_embeddings": rng.standard_normal((args.vocab_size, args.dim)),
         "norm": 1 + n(args.dim), "output": n(args.vocab_size, args.dim), "layers": []}
    for _ in range(args.n_layers):
        w["layers"].append({
            "attention_norm": 1 + n(args.dim), "wq": n(args.n_heads * hd, args.dim),
            "wk": n(args.n_kv_heads * hd, args.dim), "wv": n(args.n_kv_heads * hd, args.dim),
            "wo": n(args.dim, args.n_heads * hd), "ffn_norm": 1 + n(args.dim),
            "w1": n(H, args.dim), "w2": n(args.dim, H), "w3": n(H, args.dim)})
    return w


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split(":", 1)
                out[k.strip()] = v.strip()
    return out


# --------------------------------------------------------------------------- sizes

def test_hidden_dim_rule_matches_stated_widths():
    """Admin Guide §8.4 FeedForward rule vs the stated widths (catches a dropped
    2/3 factor, a missing multiplier, rounding down instead of up)."""
    g = _golden("sizes.txt")
    for key in ("hidden_tiny", "hidden_7b", "hidden_13b", "hidden_70b", "hidden_70b_mo256",
                "hidden_70b_nomult"):
        m = re.match(r"dim=(\d+) multiple_of=(\d+) mult=([\d.]+) -> (\d+)", g[key])
        dim, mo, mult, want = int(m[1]), int(m[2]), float(m[3]), int(m[4])
        assert O.ffn_hidden_dim(dim, mo, mult if mult > 0 else None) == want, key


def test_workload_widths_agree_with_rule():
    from workloads import WORKLOADS
    for name, wl in WORKLOADS.items():
        s = wl["shape"]
        assert O.ffn_hidden_dim(s.dim, s.multiple_of, s.ffn_dim_multiplier) == s.hidden, name


def test_kv_cache_bytes_match_admin_guide():
    """Admin Guide §6.2: 64 MB per tensor per layer (7B b4 s2048 fp16), ~4 GB total,
    3 MB per tensor per layer per rank for 70B MP=8 b6 s2048."""
    g = _golden("sizes.txt")
    per = O.kv_cache_bytes_per_tensor(4, 2048, 32, 128, 2)
    assert per == int(g["kv_7b_b4_s2048_per_tensor_bytes"])
    assert per * 2 * 32 == int(g["kv_7b_b4_s2048_all_layers_k_and_v_bytes"])
    assert O.kv_cache_bytes_per_tensor(6, 2048, 1, 128, 2) == int(g["kv_70b_mp8_b6_s2048_per_tensor_bytes"])


def test_parameter_count_7b_shape():
    """The 7B shape has ~6.74e9 parameters ("7B"); exact value from the closed form."""
    g = _golden("sizes.txt")
    n = O.parameter_count(4096, 32, 32, 32, 32000, 11008)
    assert n == int(g["params_7b"])
    assert 6.5e9 < n < 7.0e9


# --------------------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector_closed_form():
    """x = c*1 gives c/sqrt(c^2+eps)*w (catches a missing eps, sqrt or mean)."""
    for c in (0.3, -2.0, 7.5):
        for eps in (1e-5, 0.25):
            x = np.full((3, 8), c)
            w = np.linspace(0.5, 2.0, 8)
            want = c / math.sqrt(c * c + eps) * w
            np.testing.assert_allclose(O.rms_norm(x, w, eps), np.broadcast_to(want, (3, 8)), rtol=1e-14)


def test_rmsnorm_unit_rms_and_row_independence():
    """eps=0: mean((y/w)^2) = 1 for every row; rows normalise independently
    (catches a norm over the wrong axis, a mean subtraction)."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 64)) * np.arange(1, 6)[:, None] + 3.0
    w = 1 + 0.1 * rng.standard_normal(64)
    y = O.rms_norm(x, w, 0.0)
    np.testing.assert_allclose(np.mean((y / w) ** 2, axis=-1), np.ones(5), rtol=1e-13)
    # y / w is proportional to x row by row (no mean subtraction)
    ratio = (y / w) / x
    np.testing.assert_allclose(ratio, np.broadcast_to(ratio[:, :1], ratio.shape), rtol=1e-12)


# --------------------------------------------------------------------------- RoPE

def test_rope_two_dim_is_a_rotation_by_position():
    """head_dim 2 has freq_0 = 1: (1,0) -> (cos p, sin p), (0,1) -> (-sin p, cos p).
    Pins the complex multiplication's sign and the adjacent-pair view
    (Admin Guide §8.4, apply_rotary_emb)."""
    for p in (0, 1, 5, 37):
        v = np.array([[[1.0, 0.0], [0.0, 1.0]]])  # T=1, two heads
        out = O.apply_rope(v, [p], 10000.0)
        np.testing.assert_allclose(out[0, 0], [math.cos(p), math.sin(p)], atol=1e-15)
        np.testing.assert_allclose(out[0, 1], [-math.sin(p), math.cos(p)], atol=1e-15)


def test_rope_frequency_schedule_textbook():
    """theta=100, head_dim=4: freq_1 = 100^(-2/4) = 0.1; e_2 at position 3 rotates by 0.3.
    The pairs are (0,1) and (2,3) (adjacent), not (0,2)/(1,3)."""
    v = np.zeros((1, 1, 4))
    v[0, 0, 2] = 1.0
    out = O.apply_rope(v, [3], 100.0)
    np.testing.assert_allclose(out[0, 0], [0, 0, math.cos(0.3), math.sin(0.3)], atol=1e-15)
    np.testing.assert_allclose(O.rope_frequencies(8, 10000.0), [1, 0.1, 0.01, 0.001], rtol=1e-14)


def test_rope_preserves_pair_norms_and_identity_at_zero():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((6, 3, 16))
    pos = np.arange(6) * 113
    out = O.apply_rope(v, pos, 10000.0)
    n_in = v[..., 0::2] ** 2 + v[..., 1::2] ** 2
    n_out = out[..., 0::2] ** 2 + out[..., 1::2] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)
    np.testing.assert_array_equal(O.apply_rope(v, np.zeros(6), 10000.0), v)


def test_rope_dot_product_depends_on_relative_position_only():
    """<R_m q, R_n k> = <R_{m+s} q, R_{n+s} k> (source tour: relative positions)."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, 32))
    k = rng.standard_normal((1, 1, 32))
    for m, n, s in ((5, 2, 100), (0, 17, 1000), (40, 40, 3)):
        a = np.sum(O.apply_rope(q, [m], 1e4) * O.apply_rope(k, [n], 1e4))
        b = np.sum(O.apply_rope(q, [m + s], 1e4) * O.apply_rope(k, [n + s], 1e4))
        assert abs(a - b) < 1e-12


# --------------------------------------------------------------------------- softmax / mask

def test_softmax_rows_sum_to_one_and_shift_invariant():
    rng = np.random.default_rng(4)
    s = rng.standard_normal((7, 33)) * 10
    p = O.softmax(s)
    np.testing.assert_allclose(p.sum(-1), np.ones(7), rtol=1e-14)
    np.testing.assert_allclose(O.softmax(s + 123.0), p, rtol=1e-12)
    s[:, 5] = -np.inf
    assert np.all(O.softmax(s)[:, 5] == 0)


def test_causal_mask_shape_and_values():
    """Admin Guide §8.4 NOTE: (seqlen, start_pos+seqlen), -inf above the diagonal
    of the new-token block only."""
    m = O.causal_mask(3, 2)
    ni = -np.inf
    want = np.array([[0, 0, 0, ni, ni], [0, 0, 0, 0, ni], [0, 0, 0, 0, 0]])
    np.testing.assert_array_equal(m, want)


# --------------------------------------------------------------------------- attention

def _brute_attention(q, keys, values, start_pos, n_rep):
    """Scalar loops: explicit dot products, explicit visibility test j <= start_pos+t,
    explicit exp and normalisation."""
    T, nh, hd = q.shape
    out = np.zeros((T, nh, hd))
    for t in range(T):
        for h in range(nh):
            g = h // n_rep
            vis = [j for j in range(keys.shape[0]) if j <= start_pos + t]
            sc = [sum(q[t, h, d] * keys[j, g, d] for d in range(hd)) / math.sqrt(hd) for j in vis]
            mx = max(sc)
            ex = [math.exp(s - mx) for s in sc]
            z = sum(ex)
            for d in range(hd):
                out[t, h, d] = sum(ex[i] * values[j, g, d] for i, j in enumerate(vis)) / z
    return out


@pytest.mark.parametrize("start_pos,T,nh,nkv", [(0, 4, 4, 2), (3, 2, 4, 1), (5, 1, 2, 2), (0, 1, 8, 2)])
def test_attention_matches_brute_force(start_pos, T, nh, nkv):
    rng = np.random.default_rng(5 + start_pos)
    hd = 6
    q = rng.standard_normal((T, nh, hd))
    keys = rng.standard_normal((start_pos + T, nkv, hd))
    values = rng.standard_normal((start_pos + T, nkv, hd))
    got = O.attention(q, keys, values, start_pos, nh // nkv)
    np.testing.assert_allclose(got, _brute_attention(q, keys, values, start_pos, nh // nkv),
                               rtol=1e-12, atol=1e-14)


def test_attention_zero_query_averages_visible_values():
    """q = 0 gives uniform weights: output t is the mean of values 0..start_pos+t
    (catches an off-by-one in the mask, a wrong KV head)."""
    rng = np.random.default_rng(6)
    T, start, nkv, hd = 3, 4, 2, 5
    values = rng.standard_normal((start + T, nkv, hd))
    keys = rng.standard_normal((start + T, nkv, hd))
    out = O.attention(np.zeros((T, 4, hd)), keys, values, start, 2)
    for t in range(T):
        for h in range(4):
            np.testing.assert_allclose(out[t, h], values[:start + t + 1, h // 2].mean(0), rtol=1e-13)


def test_attention_scale_is_inverse_sqrt_head_dim():
    """Two keys, scores differ by exactly sqrt(hd)*a/sqrt(hd) = a: weight ratio e^a."""
    hd = 16
    q = np.zeros((1, 1, hd))
    q[0, 0, 0] = 2.0
    keys = np.zeros((2, 1, hd))
    keys[1, 0, 0] = math.sqrt(hd) * 0.75 / 2.0   # score difference 0.75
    values = np.zeros((2, 1, hd))
    values[1, 0, 3] = 1.0
    out = O.attention(q, keys, values, 1, 1)
    want = math.exp(0.75) / (1 + math.exp(0.75))
    assert abs(out[0, 0, 3] - want) < 1e-14


# --------------------------------------------------------------------------- SwiGLU

def test_silu_values():
    np.testing.assert_allclose(O.silu(np.array([0.0, 1.0, -1.0])),
                               [0.0, 0.7310585786300049, -0.2689414213699951], rtol=1e-15)
    # large |z|: silu(z) -> z and silu(-z) -> 0 (sigmoid saturates)
    np.testing.assert_allclose(O.silu(np.array([40.0, -40.0])), [40.0, 0.0], atol=1e-15)


def test_feed_forward_orientation_and_gate():
    """w2(silu(w1 x) * w3 x) with nn.Linear orientation y = x W^T (catches a
    transposed operand, swapped w1/w3, a missing gate)."""
    a, b = 0.7, -1.3
    x = np.array([[a, b]])
    w1 = np.array([[1.0, 0.0], [0.0, 0.0]])   # gate reads x0
    w3 = np.array([[0.0, 2.0], [0.0, 0.0]])   # up reads x1
    w2 = np.array([[0.0, 0.0], [3.0, 0.0]])   # out1 = 3 * hidden0
    out = O.feed_forward(x, w1, w2, w3)
    want = 3.0 * (a / (1 + math.exp(-a))) * (2.0 * b)
    np.testing.assert_allclose(out, [[0.0, want]], rtol=1e-14, atol=1e-15)


# --------------------------------------------------------------------------- whole model

def test_block_is_identity_when_wo_and_w2_are_zero():
    """Pre-norm residual: with wo = w2 = 0 each block returns its input, so the
    logits are output(norm(embedding)) (catches a missing residual, a missing final
    norm, a wrong embedding row)."""
    args = _tiny_args()
    w = _rand_weights(args, seed=7)
    for lw in w["layers"]:
        lw["wo"] = np.zeros_like(lw["wo"])
        lw["w2"] = np.zeros_like(lw["w2"])
    toks = [3, 17, 0, 39, 5]
    logits = O.forward(args, w, toks, 0, O.new_cache(args))
    x = w["tok_embeddings"][toks]
    want = (x / np.sqrt(np.mean(x ** 2, -1, keepdims=True) + 1e-5) * w["norm"]) @ w["output"].T
    np.testing.assert_allclose(logits, want, rtol=1e-12)


def test_linear_orientation_in_attention_output():
    """wo with a single entry wo[i, j] = 1 adds o[j] to x[i] (y = x W^T)."""
    args = _tiny_args(n_layers=1)
    w = _rand_weights(args, seed=8)
    lw = w["layers"][0]
    lw["w2"] = np.zeros_like(lw["w2"])
    lw["wo"] = np.zeros_like(lw["wo"])
    lw["wo"][5, 9] = 1.0
    cache = O.new_cache(args)
    x = w["tok_embeddings"][[4]]
    h = O.layer_forward(args, lw, x, cache, 0, 0)
    delta = h - x
    # T=1, start 0: attention output is v of the only key; head of dim 9 reads KV head (9//hd)//n_rep
    y = O.rms_norm(x, lw["attention_norm"], args.norm_eps)
    v = (y @ lw["wv"].T).reshape(args.n_kv_heads, args.head_dim)
    hq = 9 // args.head_dim
    expect = v[hq // args.n_rep, 9 % args.head_dim]
    assert abs(delta[0, 5] - expect) < 1e-13
    assert np.count_nonzero(np.abs(np.delete(delta[0], 5)) > 0) == 0


def test_gqa_equals_mha_with_repeated_kv_heads():
    """A GQA model equals the MHA model whose wk/wv head blocks are repeated n_rep
    times (repeat_kv; source tour "One model.py").  Also n_kv_heads == n_heads
    makes the repeat an identity."""
    g_args = _tiny_args(n_heads=4, n_kv_heads=2)
    m_args = _tiny_args(n_heads=4, n_kv_heads=4)
    w = _rand_weights(g_args, seed=9)
    hd = g_args.head_dim
    wm = {k: w[k] for k in ("tok_embeddings", "norm", "output")}
    wm["layers"] = []
    for lw in w["layers"]:
        m = dict(lw)
        for name in ("wk", "wv"):
            blocks = lw[name].reshape(g_args.n_kv_heads, hd, g_args.dim)
            m[name] = np.repeat(blocks, g_args.n_rep, axis=0).reshape(-1, g_args.dim)
        wm["layers"].append(m)
    toks = [1, 2, 3, 4, 5, 6, 7]
    a = O.forward(g_args, w, toks, 0, O.new_cache(g_args))
    b = O.forward(m_args, wm, toks, 0, O.new_cache(m_args))
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_causality_prefix_logits_unchanged_by_later_tokens():
    args = _tiny_args()
    w = _rand_weights(args, seed=10)
    t1 = [5, 9, 2, 33, 8, 1, 14]
    t2 = t1[:4] + [0, 0, 39]
    a = O.forward(args, w, t1, 0, O.new_cache(args))
    b = O.forward(args, w, t2, 0, O.new_cache(args))
    np.testing.assert_array_equal(a[:4], b[:4])
    assert np.max(np.abs(a[4:] - b[4:])) > 1e-6


def test_kv_cache_prefill_then_decode_equals_full_forward():
    """Prefill T1 tokens, then one token at a time (and a second prefill chunk)
    equals a single full-sequence forward (Admin Guide §8.4 mask NOTE)."""
    args = _tiny_args()
    w = _rand_weights(args, seed=11)
    toks = [7, 3, 22, 19, 0, 31, 8, 8, 2, 11, 25]
    full = O.forward(args, w, toks, 0, O.new_cache(args))
    cache = O.new_cache(args)
    got = [O.forward(args, w, toks[:6], 0, cache)]
    for i in range(6, 9):
        got.append(O.forward(args, w, toks[i:i + 1], i, cache))
    got.append(O.forward(args, w, toks[9:], 9, cache))   # chunked prefill at start_pos 9
    np.testing.assert_allclose(np.concatenate(got), full, rtol=1e-11, atol=1e-12)


def test_logits_positions_subset():
    args = _tiny_args(n_layers=1)
    w = _rand_weights(args, seed=12)
    toks = [1, 2, 3, 4, 5]
    full = O.forward(args, w, toks, 0, O.new_cache(args))
    part = O.forward(args, w, toks, 0, O.new_cache(args), logits_positions=[4, 1])
    np.testing.assert_allclose(part, full[[4, 1]], rtol=1e-13)


# --------------------------------------------------------------------------- sampling

def _parse_top_p_cases():
    cases = []
    with open(os.path.join(GOLDEN, "top_p_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, draws = line.split(";")
            m = re.match(r"p=([\d.,]+) top_p=([\d.]+) -> kept=([\d,]+)", lhs.strip())
            p = [float(v) for v in m[1].split(",")]
            kept = [int(v) for v in m[3].split(",")]
            ds = [(float(a[2:]), int(b)) for a, b in (d.split(":") for d in draws.split())]
            cases.append((p, float(m[2]), kept, ds))
    return cases


@pytest.mark.parametrize("case", _parse_top_p_cases())
def test_top_p_hand_worked_cases(case):
    p, top_p, kept, draws = case
    logits = np.log(np.array(p, dtype=np.float32)).astype(np.float32)
    assert O.top_p_kept(logits, 1.0, top_p) == kept
    for u, tok in draws:
        assert O.sample_top_p(logits, 1.0, top_p, u) == tok, (u, tok)


def test_top_p_limits():
    """top_p -> 0+ is the argmax; top_p = 1 keeps every token; T=0 is greedy."""
    rng = np.random.default_rng(13)
    l = rng.standard_normal(1000).astype(np.float32)
    assert O.top_p_kept(l, 0.7, 1e-9) == [int(np.argmax(l))]
    for u in (0.0, 0.3, 0.99):
        assert O.sample_top_p(l, 0.7, 1e-9, u) == int(np.argmax(l))
    assert len(O.top_p_kept(l, 0.7, 1.0)) == 1000
    assert O.sample_top_p(l, 0.0, 0.9, 0.5) == int(np.argmax(l))


def test_top_p_temperature_divides_logits():
    """softmax(l / T): T = 0.5 on l equals T = 1 on 2l (catches multiplying by T)."""
    rng = np.random.default_rng(14)
    l = rng.standard_normal(300).astype(np.float32)
    np.testing.assert_allclose(O.top_p_probs(l, 0.5), O.top_p_probs(2 * l.astype(np.float64), 1.0),
                               rtol=1e-12)


def test_greedy_ties_go_to_lowest_id():
    l = np.array([0.1, 3.0, -2.0, 3.0, 3.0], dtype=np.float32)
    assert O.greedy(l) == 1
    order = O.sampling_order(l)
    assert list(order[:3]) == [1, 3, 4]


def test_top_p_stratified_draw_frequencies_are_exact():
    """With u on a regular grid the number of draws of each kept token is
    N*p/Z up to one (the inverse-CDF draw is exact), and unkept tokens never appear."""
    rng = np.random.default_rng(15)
    l = (rng.standard_normal(50) * 2).astype(np.float32)
    T, top_p, N = 0.8, 0.75, 20000
    p = O.top_p_probs(l, T)
    kept = O.top_p_kept(l, T, top_p)
    Z = sum(p[k] for k in kept)
    counts = {}
    for i in range(N):
        tok = O.sample_top_p(l, T, top_p, (i + 0.5) / N)
        counts[tok] = counts.get(tok, 0) + 1
    assert set(counts) <= set(kept)
    for k in kept:
        assert abs(counts.get(k, 0) - N * p[k] / Z) <= 1.0 + 1e-9


def test_top_p_random_draws_chi_square():
    """Random uniforms: chi-square of draw counts against p/Z stays below the
    0.999 quantile (catches a draw from the unrenormalised or unsorted mass)."""
    from scipy.stats import chi2
    rng = np.random.default_rng(16)
    l = rng.standard_normal(12).astype(np.float32)
    T, top_p, N = 1.0, 0.8, 40000
    p = O.top_p_probs(l, T)
    kept = O.top_p_kept(l, T, top_p)
    Z = sum(p[k] for k in kept)
    us = rng.random(N)
    counts = np.zeros(len(l))
    for u in us:
        counts[O.sample_top_p(l, T, top_p, u)] += 1
    exp = np.array([N * p[k] / Z for k in kept])
    stat = float(np.sum((counts[kept] - exp) ** 2 / exp))
    assert stat < chi2.ppf(0.999, len(kept) - 1)
    assert counts.sum() == counts[kept].sum()


def test_sample_margins_flags_boundary_draws_only():
    """A draw right at a cumulative boundary has margin ~0; a draw in the
    middle of a bin has a margin of about half the bin's share."""
    p = [0.5, 0.3, 0.15, 0.05]
    l = np.log(np.array(p, dtype=np.float32))
    assert O.sample_margins(l, 1.0, 1.0, 0.5) < 1e-6          # target 0.5 = C_0
    assert abs(O.sample_margins(l, 1.0, 1.0, 0.25) - 0.25) < 1e-6
    # tail tokens of negligible mass near top_p = 1 do not make a mid-bin draw ambiguous
    l2 = np.concatenate([l, np.full(5, -60.0, dtype=np.float32)])
    assert O.sample_margins(l2, 1.0, 1.0, 0.25) > 0.2
    # but a draw that lands on such a token is flagged
    assert O.sample_margins(l2, 1.0, 1.0, 0.9999999999999) < 1e-9


# --------------------------------------------------------------------------- 16-bit storage error model

def test_round_bf16_closed_forms():
    """bfloat16 keeps 8 significant bits: 1 + 2^-7 is exact, 1 + 2^-8 lies
    halfway between 1 and 1 + 2^-7 and goes to the even neighbour 1, and
    1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6 and goes to the
    even 1 + 2^-6.  Catches truncation instead of rounding, ties away from
    zero, and a wrong count of kept bits."""
    x = np.array([1.0, 1 + 2 ** -7, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, 3 - 2 ** -9, 0.0])
    want = np.array([1.0, 1 + 2 ** -7, 1.0, 1 + 2 ** -6, 1 + 2 ** -7, 3.0, 0.0])
    np.testing.assert_array_equal(O.round_bf16(x), want)
    np.testing.assert_array_equal(O.round_bf16(-x), -want)
    np.testing.assert_array_equal(O.round_bf16(x * 2.0 ** 40), want * 2.0 ** 40)   # exponent untouched


def test_round_bf16_bounds_and_idempotence():
    """Half-ulp bound |r(x) - x| <= 2^-8 |x| for normal x, the low 16 bits of
    every result's binary32 word are zero, and r(r(x)) = r(x)."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))
    r = O.round_bf16(x)
    assert np.all(np.abs(r - x) <= 2.0 ** -8 * np.abs(x) * (1 + 1e-7))
    assert np.all((r.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)
    np.testing.assert_array_equal(O.round_bf16(r), r)


def test_round_f16_closed_forms():
    """binary16 keeps 11 significant bits: ties at 1 + 2^-11 and 1 + 3*2^-11
    go to the even neighbours 1 and 1 + 2^-9; 65504 is the largest finite."""
    x = np.array([1.0, 1 + 2 ** -10, 1 + 2 ** -11, 1 + 3 * 2 ** -11, 65504.0, -0.5])
    want = np.array([1.0, 1 + 2 ** -10, 1.0, 1 + 2 ** -9, 65504.0, -0.5])
    np.testing.assert_array_equal(O.round_f16(x), want)


def test_storage_hook_identity_is_the_exact_forward():
    """With an identity `store` the forward is bit-identical to the plain
    definition: the hook adds no arithmetic of its own."""
    args = _tiny_args()
    w = _rand_weights(args, seed=21)
    toks = [3, 1, 4, 1, 5, 9, 2, 6]
    a = O.forward(args, w, toks, 0, O.new_cache(args))
    b = O.forward(args, w, toks, 0, O.new_cache(args), store=lambda v: np.array(v, dtype=np.float64))
    np.testing.assert_array_equal(a, b)


def test_storage_hook_rounds_the_cache_and_stays_close():
    """With 16-bit storage the cache holds only 16-bit values, the logits
    move from the exact ones by an amount of the format's precision, and
    bfloat16 (8 significant bits) moves them further than binary16 (11):
    catches a hook that never reaches the cache, or one that rounds nothing
    or everything."""
    args = _tiny_args(dim=64, n_heads=4, n_kv_heads=2, vocab=50)
    w = _rand_weights(args, seed=22, scale=0.1)
    toks = [7, 3, 22, 19, 0, 31, 8, 8, 2, 11, 25, 40]
    exact = O.forward(args, w, toks, 0, O.new_cache(args))
    errs = {}
    for name, fn in (("bf16", O.round_bf16), ("f16", O.round_f16)):
        cache = O.new_cache(args)
        got = O.forward(args, w, toks, 0, cache, store=fn)
        for l in range(args.n_layers):
            for t in (cache.k[l][:len(toks)], cache.v[l][:len(toks)]):
                np.testing.assert_array_equal(fn(t), t)
        errs[name] = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    assert 0 < errs["f16"] < 2e-3 and 0 < errs["bf16"] < 2e-2
    assert errs["bf16"] > 3 * errs["f16"]


def test_storage_error_fixture_is_complete():
    """tests/golden/storage_error_7b.txt (written by make_storage_error.py
    from the oracle) holds one record per row of the 4-row batch, each a
    bf16-sized error: above the two-layer figure and far below O(1)."""
    rows = []
    with open(os.path.join(GOLDEN, "storage_error_7b.txt")) as f:
        for line in f:
            if line.startswith("row"):
                rows.append(dict(item.split("=") for item in line.split(":", 1)[1].split()))
    assert len(rows) == 4
    for r in rows:
        assert 1e-2 < float(r["rel_l2"]) < 1e-1
        assert 0 < float(r["rms_abs"]) < 0.1 * float(r["logits_rms"])


def test_storage_error_script_rows_on_a_tiny_model():
    """make_storage_error.py's per-row routine (prefill, then one token per
    step through the cache) on a tiny model: its exact logits equal one
    full-sequence forward at the same positions, and its bf16-storage logits
    differ from them by a bf16-sized amount."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_storage_error",
                                                  os.path.join(GOLDEN, "make_storage_error.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    args = _tiny_args(dim=64, n_heads=4, n_kv_heads=2, vocab=50)
    w = _rand_weights(args, seed=23, scale=0.1)
    prompt, after = [4, 8, 15, 16, 23], [42, 7]
    exact = mod.run_row(args, w, prompt, after, None)
    full = O.forward(args, w, prompt + after, 0, O.new_cache(args), logits_positions=[4, 5, 6])
    np.testing.assert_allclose(exact, full, rtol=1e-11, atol=1e-12)
    rounded = mod.run_row(args, w, prompt, after, O.round_bf16)
    rel = np.linalg.norm(rounded - exact) / np.linalg.norm(exact)
    assert 1e-4 < rel < 2e-2
