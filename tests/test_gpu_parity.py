"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Tolerances: logits relative L2 <= 1e-4 for the fp32
model and <= 2e-2 for bf16 models; greedy ids identical wherever the oracle's
top-2 logit gap exceeds 1e-2; single kernels much tighter (stated per test)."""
import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import build_model, check_greedy, oracle_args, rel_l2
from workloads import (L7B_LAYER, TINY, ModelShape, make_normal, make_tokens, make_uniforms, make_weights,
                       to_numpy_f64_weights, token_seed, uniform_seed, weight_seed)

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def llb(cuda_device):
    import decoder_only_transformer_llama_b200 as m
    return m


# ----------------------------------------------------------------------------- single kernels

@pytest.mark.parametrize("M,dim", [(1, 256), (5, 4096), (33, 5120), (3, 8192)])
def test_rmsnorm_kernel(llb, M, dim):
    g = torch.Generator().manual_seed(M * dim)
    x = torch.randn(M, dim, generator=g) * 3 + 0.5
    w = 1 + 0.02 * torch.randn(dim, generator=g)
    want = O.rms_norm(x.double().numpy(), w.double().numpy(), 1e-5)
    out32 = torch.empty(M, dim, device="cuda")
    llb.op_rmsnorm(x.cuda(), w.cuda(), 1e-5, out32)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out32.cpu().double().numpy(), want, rtol=2e-6, atol=1e-6)
    out16 = torch.empty(M, dim, device="cuda", dtype=torch.bfloat16)
    llb.op_rmsnorm(x.cuda(), w.cuda(), 1e-5, out16)
    torch.cuda.synchronize()
    got = out16.cpu().double().numpy()
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8 + 1e-6)
    outh = torch.empty(M, dim, device="cuda", dtype=torch.float16)
    llb.op_rmsnorm(x.cuda(), w.cuda(), 1e-5, outh)
    torch.cuda.synchronize()
    got = outh.cpu().double().numpy()
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -11 + 1e-6)


@pytest.mark.parametrize("M,N,K", [(1, 384, 256), (70, 1000, 768), (130, 130, 64), (2, 2048, 96)])
def test_linear_f32_kernel(llb, M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g)
    W = torch.randn(N, K, generator=g) * 0.05
    out = torch.empty(M, N, device="cuda")
    llb.op_linear(A.cuda(), W.cuda(), out)
    torch.cuda.synchronize()
    want = A.double().numpy() @ W.double().numpy().T
    assert rel_l2(out.cpu().numpy(), want) < 1e-6


@pytest.mark.parametrize("M,N,K", [
    (1, 256, 256), (7, 1000, 4096), (16, 4096, 256), (17, 384, 4160), (33, 512, 200), (64, 12288, 4096),
    (48, 640, 512),
    (65, 256, 256), (128, 1000, 4096), (300, 768, 1024), (2048, 512, 64),
    (300, 4224, 4096), (7, 1003, 512), (130, 1003, 512), (300, 5003, 4096)])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_linear_16bit_tcgen05_kernel(llb, M, N, K, dt):
    """tcgen05 GEMM in both orientations (M <= 64: weights as the 128-row
    operand; else activations, on one SM per tile or, for at least 256 rows
    and more than 4096 x 4096 weights, on CTA pairs), with ragged M, N and K
    tails (N = 1003 and 5003: fp32 rows that are not 16-byte aligned, stored
    element by element), for both 16-bit operand types."""
    g = torch.Generator().manual_seed(7 * M + N + K)
    A = torch.randn(M, K, generator=g).to(dt)
    W = (torch.randn(N, K, generator=g) * 0.05).to(dt)
    out = torch.full((M, N), float("nan"), device="cuda")
    llb.op_linear(A.cuda(), W.cuda(), out)
    torch.cuda.synchronize()
    want = A.double().numpy() @ W.double().numpy().T
    got = out.cpu().double().numpy()
    assert np.isfinite(got).all()
    assert rel_l2(got, want) < 2e-5
    np.testing.assert_allclose(got, want, atol=1e-3 + 1e-4 * np.abs(want).max())


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [
    (512, 9472, 256),      # 148 tiles: one full wave, whole tiles only
    (2048, 2560, 1024),    # 160 tiles: all split along K over the SMs (stream-K)
    (2048, 4864, 512),     # 304 tiles: one wave of whole tiles, then a stream-K run
    (256, 35584, 256),     # 278 tiles: last wave 88 % full, whole tiles only
    (1000, 1000, 4160),    # ragged M, N and K, 32 tiles split up to 4 ways
    # CTA pairs (256 x 256 tiles, 74 pairs on a 148-SM B200)
    (512, 18944, 1024),    # 148 pair tiles: two full waves, whole tiles only
    (2048, 5120, 4096),    # 160 pair tiles: two waves, then 12 tiles stream-K over 48 runs
    (1000, 4160, 4160),    # ragged M, N and K, 68 pair tiles all split (the last half-tile partly past M)
    (384, 16384, 1088),    # the second pair tile's upper half lies wholly past M
])
def test_linear_bf16_prefill_work_split(llb, M, N, K):
    """The persistent prefill projection under each of its work splits, with
    and without the split-tile workspace; split results are bit-identical
    from run to run (partials added in a fixed order)."""
    g = torch.Generator().manual_seed(11 * M + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16).cuda()
    want = A.cpu().double().numpy() @ W.cpu().double().numpy().T
    outs = []
    for ws in (None, False, None):
        out = torch.full((M, N), float("nan"), device="cuda")
        if ws is False:
            llb.op_linear_whole_tiles(A, W, out)
        else:
            llb.op_linear(A, W, out)
        torch.cuda.synchronize()
        got = out.cpu().double().numpy()
        assert np.isfinite(got).all()
        assert rel_l2(got, want) < 2e-5
        np.testing.assert_allclose(got, want, atol=1e-3 + 1e-4 * np.abs(want).max())
        outs.append(out.cpu())
    assert torch.equal(outs[0], outs[2])


@pytest.mark.gpu
def test_linear_bf16_prefill_7b_qkv_sampled(llb):
    """7B wq/wk/wv shape at 4 x 512 prompt tokens (2048 x 12288 x 4096),
    checked on 64 sampled token rows against fp64."""
    M, N, K = 2048, 12288, 4096
    g = torch.Generator().manual_seed(77)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    out = torch.empty((M, N), device="cuda")
    llb.op_linear(A.cuda(), W.cuda(), out)
    torch.cuda.synchronize()
    rows = torch.randperm(M, generator=g)[:64].sort().values
    want = A[rows].double().numpy() @ W.double().numpy().T
    got = out.cpu()[rows].double().numpy()
    assert rel_l2(got, want) < 2e-5
    np.testing.assert_allclose(got, want, atol=1e-3 + 1e-4 * np.abs(want).max())


# ----------------------------------------------------------------------------- sampling

def test_greedy_sampler_ties_and_values(llb):
    V = 32000
    g = torch.Generator().manual_seed(5)
    lg = torch.randn(6, V, generator=g)
    lg[1, 100] = lg[1, 2000] = 50.0       # tie: lowest id wins
    lg[2, :] = 0.0                        # all equal: id 0
    lg[3, V - 1] = 99.0
    out = torch.empty(6, dtype=torch.int32, device="cuda")
    llb.sample(lg.cuda(), 0.0, 0.9, None, out)
    torch.cuda.synchronize()
    want = [O.greedy(r) for r in lg.numpy()]
    assert out.cpu().tolist() == want
    assert want[1] == 100 and want[2] == 0 and want[3] == V - 1


@pytest.mark.parametrize("V,T,p,scale", [(32000, 0.6, 0.9, 1.0), (32000, 0.6, 0.9, 8.0), (512, 1.0, 0.5, 3.0),
                                         (1000, 0.3, 0.99, 1.0), (32000, 1.0, 1.0, 2.0), (50, 0.8, 1e-6, 1.0),
                                         (5, 0.7, 0.9, 1.0), (128256, 0.6, 0.9, 1.5), (150000, 0.7, 0.9, 1.0)])
def test_top_p_sampler_matches_oracle(llb, V, T, p, scale):
    """Indices identical to the oracle's for every draw whose margin to a
    decision boundary exceeds 1e-9 (no draw is expected to be that close).
    Vocabularies up to about 137k run on a cluster of CTAs per row (5: some
    CTAs own no slice; 128256: the largest slices), larger ones on one CTA
    per row."""
    B, draws = (4, 8) if V > 100000 else (8, 16)
    g = torch.Generator().manual_seed(V + int(100 * T))
    base = torch.randn(B, V, generator=g) * scale
    lg = base.repeat_interleave(draws, 0).contiguous()
    u = make_uniforms((B * draws,), 3000 + V)
    out = torch.empty(B * draws, dtype=torch.int32, device="cuda")
    llb.sample(lg.cuda(), T, p, u.cuda(), out)
    torch.cuda.synchronize()
    got = out.cpu().tolist()
    ambiguous = 0
    for i in range(B * draws):
        row = lg[i].numpy()
        if O.sample_margins(row, T, p, float(u[i])) < 1e-9:
            ambiguous += 1
            assert got[i] in O.top_p_kept(row, T, p)
            continue
        assert got[i] == O.sample_top_p(row, T, p, float(u[i])), i
    assert ambiguous == 0


@pytest.mark.parametrize("V", [1000, 32000])
def test_top_p_sampler_with_tied_logits(llb, V):
    """Logits on a 0.25 grid (thousands of exact ties, which the select
    resolves on the id digits of its key, across the slices of the CTAs that
    share a row), a row of equal logits and a row with -inf entries: indices
    identical to the oracle's (ties: lowest id first)."""
    B, draws = 6, 12
    g = torch.Generator().manual_seed(77 + V)
    base = torch.round(torch.randn(B, V, generator=g) * 4.0) / 4.0
    base[1, :] = 0.0
    base[2, ::3] = float("-inf")
    lg = base.repeat_interleave(draws, 0).contiguous()
    u = make_uniforms((B * draws,), 4100 + V)
    T, p = 0.7, 0.9003
    out = torch.empty(B * draws, dtype=torch.int32, device="cuda")
    llb.sample(lg.cuda(), T, p, u.cuda(), out)
    torch.cuda.synchronize()
    got = out.cpu().tolist()
    for i in range(B * draws):
        row = lg[i].numpy()
        assert O.sample_margins(row, T, p, float(u[i])) >= 1e-9, i
        assert got[i] == O.sample_top_p(row, T, p, float(u[i])), i


# ----------------------------------------------------------------------------- whole model

def _tiny_run(llb, shape, weights, B, T, steps, lens=None):
    """Prefill (lens per row) then greedy decode `steps` tokens; returns the
    GPU's tokens per row and its logits (prefill last position, then each step)."""
    m = build_model(shape, weights)
    toks = make_tokens(shape.vocab_size, (B, T), token_seed(0)).cuda()
    lens = lens or [T] * B
    logits = torch.empty(B, shape.vocab_size, device="cuda")
    m.prefill(toks, lens=lens, logits=logits)
    seq = [toks[b, :lens[b]].cpu().tolist() for b in range(B)]
    all_logits = [[logits[b].cpu().numpy().copy()] for b in range(B)]
    cur = torch.tensor([O.greedy(all_logits[b][0]) for b in range(B)], dtype=torch.int32)
    # greedy from the GPU's own logits (the kernel argmax is checked separately)
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    first = nxt.clone()
    llb.sample(logits, 0.0, 0.9, None, first)
    assert first.cpu().tolist() == cur.tolist()
    cur = cur.cuda()
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for _ in range(steps):
        for b in range(B):
            seq[b].append(int(cur[b]))
        step_logits = torch.empty(B, shape.vocab_size, device="cuda")
        m.decode_step(cur, pos, temperature=0.0, next_tokens=nxt, logits=step_logits)
        torch.cuda.synchronize()
        for b in range(B):
            all_logits[b].append(step_logits[b].cpu().numpy().copy())
        cur = nxt.clone()
        pos += 1
    assert m.status() == 0
    m.close()
    return seq, all_logits


def _oracle_check(shape, weights, seq, gpu_logits, lens, tol):
    args = oracle_args(shape)
    w64 = to_numpy_f64_weights(weights)
    worst = 0.0
    for b, s in enumerate(seq):
        L = lens[b]
        want = O.forward(args, w64, s, 0, O.new_cache(args))   # teacher-forced full sequence
        want = want[L - 1:]                                    # logits after the prompt, then each step
        got = np.stack(gpu_logits[b][:want.shape[0]])
        err = rel_l2(got, want)
        worst = max(worst, err)
        assert err <= tol, (b, err)
        # greedy ids: the token after position i is seq[L + i]
        gen = s[L:]
        check_greedy(gen, want[:len(gen)])
    return worst


def test_tiny_f32_model_prefill_and_greedy_decode(llb):
    """Tiny fp32 workload: batch 2, prefill 64 random ids, 16 greedy steps,
    max_seq_len 128.  Logits rel-L2 <= 1e-4 at every step."""
    w = make_weights(TINY, weight_seed(0))
    seq, gl = _tiny_run(llb, TINY, w, B=2, T=64, steps=16)
    _oracle_check(TINY, w, seq, gl, [64, 64], F32_TOL)


def test_tiny_f32_all_position_logits_and_chunked_prefill(llb):
    """logits_mode 1 returns every position's logits; a prefill split in two
    chunks (start_pos > 0) gives the same cache and logits as one call."""
    w = make_weights(TINY, weight_seed(0))
    args = oracle_args(TINY)
    w64 = to_numpy_f64_weights(w)
    toks = make_tokens(TINY.vocab_size, (2, 40), 77).cuda()
    m = build_model(TINY, w)
    allg = torch.empty(80, TINY.vocab_size, device="cuda")
    m.prefill(toks[:, :25].contiguous(), logits=allg[:50], all_logits=True)
    m.prefill(toks[:, 25:].contiguous(), start_pos=25, logits=allg[50:], all_logits=True)
    torch.cuda.synchronize()
    got = allg.cpu().numpy()
    for b in range(2):
        want = O.forward(args, w64, toks[b].cpu().tolist(), 0, O.new_cache(args))
        g_b = np.concatenate([got[b * 25:(b + 1) * 25], got[50 + b * 15:50 + (b + 1) * 15]])
        assert rel_l2(g_b, want) <= F32_TOL
    m.close()


SMALL_BF16 = ModelShape(dim=256, n_layers=2, n_heads=2, n_kv_heads=1, vocab_size=512, max_seq_len=160,
                        max_batch_size=3, dtype="bf16", hidden=768)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_small_bf16_gqa_ragged_prefill_and_decode(llb, dtype):
    """16-bit path (tcgen05 projections, head_dim 128, n_rep 2) with ragged
    prompt lengths and per-row decode positions, in bf16 and in the
    reference's own fp16."""
    shape = SMALL_BF16.replace(dtype=dtype)
    w = make_weights(shape, 99)
    lens = [37, 64, 5]
    seq, gl = _tiny_run(llb, shape, w, B=3, T=64, steps=12, lens=lens)
    _oracle_check(shape, w, seq, gl, lens, BF16_TOL)


def test_small_bf16_decode_with_top_p_sampling(llb):
    """Decode steps that sample in the step itself (temperature 0.6, top-p 0.9,
    one seeded uniform per row and step): every sampled id equals the oracle's
    nucleus draw on the step's own logits with the same uniform (or, for a draw
    within rounding of a boundary, lies in the kept set), and the logits of the
    sampled sequence match the oracle's teacher-forced forward pass."""
    T_, P_ = 0.6, 0.9
    w = make_weights(SMALL_BF16, 98)
    m = build_model(SMALL_BF16, w)
    B, T, steps = 3, 48, 8
    lens = [48, 17, 30]
    toks = make_tokens(SMALL_BF16.vocab_size, (B, T), token_seed(5)).cuda()
    logits = torch.empty(B, SMALL_BF16.vocab_size, device="cuda")
    m.prefill(toks, lens=lens, logits=logits)
    uni = make_uniforms((steps + 1, B), 3100)
    cur = torch.empty(B, dtype=torch.int32, device="cuda")
    llb.sample(logits, T_, P_, uni[0].cuda(), cur)
    seq = [toks[b, :lens[b]].cpu().tolist() for b in range(B)]
    gl = [[logits[b].cpu().numpy().copy()] for b in range(B)]
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    ambiguous = 0
    for i in range(steps):
        for b in range(B):
            seq[b].append(int(cur[b]))
        step_logits = torch.empty(B, SMALL_BF16.vocab_size, device="cuda")
        u = uni[i + 1]
        m.decode_step(cur, pos, temperature=T_, top_p=P_, uniforms=u.cuda(), next_tokens=nxt, logits=step_logits)
        torch.cuda.synchronize()
        got = nxt.cpu().tolist()
        for b in range(B):
            row = step_logits[b].cpu().numpy().astype(np.float64)
            gl[b].append(row.copy())
            if O.sample_margins(row, T_, P_, float(u[b])) < 1e-9:
                ambiguous += 1
                assert got[b] in O.top_p_kept(row, T_, P_)
            else:
                assert got[b] == O.sample_top_p(row, T_, P_, float(u[b])), (i, b)
        cur = nxt.clone()
        pos += 1
    assert ambiguous == 0
    assert m.status() == 0
    m.close()
    args = oracle_args(SMALL_BF16)
    w64 = to_numpy_f64_weights(w)
    for b in range(B):
        want = O.forward(args, w64, seq[b], 0, O.new_cache(args))[lens[b] - 1:]
        got = np.stack(gl[b][:want.shape[0]])
        assert rel_l2(got, want) <= BF16_TOL, (b, rel_l2(got, want))


@pytest.mark.parametrize("B,L,dtype", [(B, L, "bf16") for B in (1, 8, 32) for L in (128, 1024, 4096)] +
                         [(8, 1024, "f16")])
def test_7b_layer_decode_against_oracle(llb, B, L, dtype):
    """One 7B-shaped layer (bf16, fp32 norms), KV cache filled with N(0,1) for
    positions [0, L), one decode step at position L; oracle on sampled rows.
    Every (batch, context) point of the decode microbenchmark grid, B in
    {1, 8, 32} x L in {128, 1024, 4096}, plus an fp16 repeat."""
    s = L7B_LAYER.replace(dtype=dtype)
    w = make_weights(s, weight_seed(1), device="cuda")
    m = build_model(s, w)
    kview, vview = m.kv_tensors(0)
    fillk = make_normal((B, L, s.n_kv_heads, s.head_dim), 11, device="cuda", dtype=kview.dtype)
    fillv = make_normal((B, L, s.n_kv_heads, s.head_dim), 12, device="cuda", dtype=kview.dtype)
    kview[:B, :L].copy_(fillk)
    vview[:B, :L].copy_(fillv)
    torch.cuda.synchronize()
    toks = make_tokens(s.vocab_size, (B,), token_seed(1)).cuda()
    pos = torch.full((B,), L, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, s.vocab_size, device="cuda")
    m.decode_step(toks, pos, logits=logits)
    torch.cuda.synchronize()
    assert m.status() == 0
    got = logits.cpu().numpy()
    args = oracle_args(s)
    w64 = to_numpy_f64_weights(w)
    rows = sorted(set([0, B - 1, B // 2]))
    fk = fillk.cpu().double().numpy()
    fv = fillv.cpu().double().numpy()
    for b in rows:
        cache = O.new_cache(args)
        cache.k[0][:L] = fk[b]
        cache.v[0][:L] = fv[b]
        want = O.forward(args, w64, [int(toks[b])], L, cache)[0]
        assert rel_l2(got[b], want) <= BF16_TOL, (b, rel_l2(got[b], want))
    m.close()
