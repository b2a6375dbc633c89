"""Edge cases of the CUDA path against the oracle: the last cache position,
one-token prompts at full batch, and inputs that the kernels' own range checks
turn into a device status code (a position past max_seq_len, a token id
outside the vocabulary) while the other rows of the batch stay exact."""
import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import build_model, oracle_args, rel_l2
from workloads import ModelShape, TINY, make_tokens, make_weights, to_numpy_f64_weights, token_seed

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
SMALL = ModelShape(dim=256, n_layers=2, n_heads=2, n_kv_heads=1, vocab_size=512, max_seq_len=96,
                   max_batch_size=4, dtype="bf16", hidden=768)


@pytest.fixture(scope="module")
def llb(cuda_device):
    import decoder_only_transformer_llama_b200 as m
    return m


def _oracle_logits(shape, w64, seq):
    args = oracle_args(shape)
    return O.forward(args, w64, seq, 0, O.new_cache(args))


@pytest.mark.parametrize("shape,tol", [(TINY, 1e-4), (SMALL, BF16_TOL)])
def test_decode_at_the_last_cache_position(llb, shape, tol):
    """Prefill max_seq_len - 1 tokens, then one decode step at position
    max_seq_len - 1: the step fills the cache exactly and matches the oracle."""
    S = shape.max_seq_len
    w = make_weights(shape, 41)
    m = build_model(shape, w)
    B, T = 2, S - 1
    toks = make_tokens(shape.vocab_size, (B, T), token_seed(7)).cuda()
    logits = torch.empty(B, shape.vocab_size, device="cuda")
    m.prefill(toks, logits=logits)
    nxt_tok = make_tokens(shape.vocab_size, (B,), token_seed(8)).cuda()
    pos = torch.full((B,), S - 1, dtype=torch.int32, device="cuda")
    step = torch.empty(B, shape.vocab_size, device="cuda")
    m.decode_step(nxt_tok, pos, logits=step)
    torch.cuda.synchronize()
    assert m.status() == 0
    w64 = to_numpy_f64_weights(w)
    for b in range(B):
        seq = toks[b].cpu().tolist() + [int(nxt_tok[b])]
        want = _oracle_logits(shape, w64, seq)[-1]
        assert rel_l2(step[b].cpu().numpy(), want) <= tol, b
    m.close()


def test_one_token_prompts_at_full_batch(llb):
    """max_batch_size rows whose prompts are 1, 2, 1 and 5 tokens long."""
    w = make_weights(SMALL, 42)
    m = build_model(SMALL, w)
    B, T = SMALL.max_batch_size, 5
    lens = [1, 2, 1, 5]
    toks = make_tokens(SMALL.vocab_size, (B, T), token_seed(9)).cuda()
    logits = torch.empty(B, SMALL.vocab_size, device="cuda")
    m.prefill(toks, lens=lens, logits=logits)
    torch.cuda.synchronize()
    assert m.status() == 0
    w64 = to_numpy_f64_weights(w)
    for b in range(B):
        want = _oracle_logits(SMALL, w64, toks[b, :lens[b]].cpu().tolist())[-1]
        assert rel_l2(logits[b].cpu().numpy(), want) <= BF16_TOL, b
    m.close()


def test_position_past_the_cache_sets_capacity_status(llb):
    """Row 1 asks for position max_seq_len: the kernels skip it and report
    LLAMA_ERR_CAPACITY; rows 0 and 2 are computed as usual."""
    S = SMALL.max_seq_len
    w = make_weights(SMALL, 43)
    m = build_model(SMALL, w)
    B, T = 3, 10
    toks = make_tokens(SMALL.vocab_size, (B, T), token_seed(10)).cuda()
    logits = torch.empty(B, SMALL.vocab_size, device="cuda")
    m.prefill(toks, logits=logits)
    nxt_tok = make_tokens(SMALL.vocab_size, (B,), token_seed(11)).cuda()
    pos = torch.tensor([T, S, T], dtype=torch.int32, device="cuda")
    step = torch.empty(B, SMALL.vocab_size, device="cuda")
    m.decode_step(nxt_tok, pos, logits=step)
    torch.cuda.synchronize()
    assert m.status() == llb.LLAMA_ERR_CAPACITY
    w64 = to_numpy_f64_weights(w)
    for b in (0, 2):
        seq = toks[b].cpu().tolist() + [int(nxt_tok[b])]
        want = _oracle_logits(SMALL, w64, seq)[-1]
        assert rel_l2(step[b].cpu().numpy(), want) <= BF16_TOL, b
    m.close()


def test_token_outside_the_vocabulary_sets_token_range_status(llb):
    """A prompt token id equal to vocab_size: its embedding row reads as zero
    and the model reports LLAMA_ERR_TOKEN_RANGE; the other row is exact."""
    w = make_weights(SMALL, 44)
    m = build_model(SMALL, w)
    B, T = 2, 6
    toks = make_tokens(SMALL.vocab_size, (B, T), token_seed(12))
    toks[1, 3] = SMALL.vocab_size
    logits = torch.empty(B, SMALL.vocab_size, device="cuda")
    m.prefill(toks.cuda(), logits=logits)
    torch.cuda.synchronize()
    assert m.status() == llb.LLAMA_ERR_TOKEN_RANGE
    want = _oracle_logits(SMALL, to_numpy_f64_weights(w), toks[0].tolist())[-1]
    assert rel_l2(logits[0].cpu().numpy(), want) <= BF16_TOL
    m.close()


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_prefix_reuse_across_prefill_calls(llb, dtype):
    """A prefix prefilled once, then two different continuations prefilled at
    start_pos = len(prefix) one after the other (the second overwrites the
    first's cache entries): every position's logits equal the oracle's on
    prefix + continuation.  Continuation lengths put the projections on both
    kernels (<= 64 token rows: the weight-streaming kernel; more: the
    128 x 256-tile kernel) and the prefill attention on start_pos > 0."""
    shape = SMALL.replace(max_seq_len=192, dtype=dtype)
    w = make_weights(shape, 45)
    m = build_model(shape, w)
    w64 = to_numpy_f64_weights(w)
    B, P = 2, 40
    prefix = make_tokens(shape.vocab_size, (B, P), token_seed(13)).cuda()
    m.prefill(prefix, logits=torch.empty(B, shape.vocab_size, device="cuda"))
    for T, seed in ((30, 14), (100, 15)):
        cont = make_tokens(shape.vocab_size, (B, T), token_seed(seed)).cuda()
        lg = torch.empty(B, T, shape.vocab_size, device="cuda")
        m.prefill(cont, start_pos=P, logits=lg, all_logits=True)
        torch.cuda.synchronize()
        assert m.status() == 0
        for b in range(B):
            seq = prefix[b].cpu().tolist() + cont[b].cpu().tolist()
            want = _oracle_logits(shape, w64, seq)[P:]
            assert rel_l2(lg[b].cpu().numpy(), want) <= BF16_TOL, (T, b)
    m.close()


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_decode_wider_than_the_fused_chain(llb, dtype):
    """A 16-bit decode step of more than 64 rows runs the un-fused sequence
    (one RMSNorm kernel per norm, the 128 x 256-tile projections) instead of
    the fused chain, whose weight-streaming projection takes at most 64 token
    columns: 72 rows prefilled and decoded twice, in bf16 and fp16, sampled
    rows against the oracle, greedy tokens written back on the device.  Row 13
    asks for a position past the cache in both steps: the step reports
    LLAMA_ERR_CAPACITY for it and the other rows stay exact."""
    shape = SMALL.replace(max_batch_size=72, max_seq_len=32, dtype=dtype)
    S = shape.max_seq_len
    w = make_weights(shape, 46)
    m = build_model(shape, w)
    B, T, bad = 72, 6, 13
    toks = make_tokens(shape.vocab_size, (B, T), token_seed(16)).cuda()
    logits = torch.empty(B, shape.vocab_size, device="cuda")
    m.prefill(toks, logits=logits)
    cur = torch.empty(B, dtype=torch.int32, device="cuda")
    llb.sample(logits, 0.0, 0.9, None, cur)
    pos = torch.full((B,), T, dtype=torch.int32, device="cuda")
    pos[bad] = S
    seqs = [toks[b].cpu().tolist() for b in range(B)]
    steps = []
    for _ in range(2):
        for b in range(B):
            seqs[b].append(int(cur[b]))
        lg = torch.empty(B, shape.vocab_size, device="cuda")
        m.decode_step(cur, pos, temperature=0.0, next_tokens=cur, logits=lg, advance=True)
        torch.cuda.synchronize()
        steps.append(lg.cpu().numpy())
    assert m.status() == llb.LLAMA_ERR_CAPACITY
    want_pos = [T + 2] * B
    want_pos[bad] = S + 2
    assert pos.cpu().tolist() == want_pos
    w64 = to_numpy_f64_weights(w)
    for b in (0, 40, 71):
        want = _oracle_logits(shape, w64, seqs[b])[T:]
        got = np.stack([steps[0][b], steps[1][b]])
        assert rel_l2(got, want) <= BF16_TOL, b
        if O.sample_margins(want[1], 0.0, 0.9, 0.0) > 1e-2:
            assert int(cur[b]) == O.greedy(want[1]), b
    m.close()
