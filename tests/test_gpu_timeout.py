"""The device-side timeout path, exercised without a GPU fault.

Every wait of a kernel on another agent (the TMA/MMA rings of the decode
and prefill projections, single-SM and CTA-pair, the bulk-copy ring of the
decode attention) is bounded.  A test
arms a one-shot stalled producer (llama_debug_stall): in the next launch of
the chosen kernel, CTA 0 never issues the copies of one pipeline stage nor the
barrier signal that would announce them, and that launch's waits give up after
1 ms.  The step must come back (the stream synchronises), the device status
word must read LLAMA_ERR_DEVICE_TIMEOUT, and the next step, at the same
positions, must again match the oracle (the failed step's partly counted split
tiles and attention pairs are reset by the status read).  Admin Guide §8.8
("Code patterns and conventions": errors are reported, not ignored)."""
import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import build_model, oracle_args, rel_l2
from workloads import ModelShape, make_tokens, make_weights, to_numpy_f64_weights, token_seed

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
# Sized so that CTA 0 of the first decode launches owns several pipeline
# stages: wq/wk/wv is 32 weight tiles x 32 K-slices = 1024 units over 148
# CTAs (6 for CTA 0); the attention at batch 8, context 601 is 8 rows x 8 KV
# heads x 10 blocks of 64 keys = 640 units over at most 296 CTAs (2 for CTA 0).
SHAPE = ModelShape(dim=2048, n_layers=2, n_heads=16, n_kv_heads=8, vocab_size=512, max_seq_len=640,
                   max_batch_size=8, dtype="bf16", hidden=5632)


@pytest.fixture(scope="module")
def llb(cuda_device):
    import decoder_only_transformer_llama_b200 as m
    return m


@pytest.mark.parametrize("which,unit", [("projection", 0), ("projection", 2), ("attention", 0), ("attention", 1)])
def test_stalled_producer_times_out_and_the_next_step_is_exact(llb, which, unit):
    s = SHAPE
    w = make_weights(s, 71)
    m = build_model(s, w)
    B, T = 8, 600
    toks = make_tokens(s.vocab_size, (B, T), token_seed(21)).cuda()
    logits = torch.empty(B, s.vocab_size, device="cuda")
    m.prefill(toks, logits=logits)
    nxt = make_tokens(s.vocab_size, (B,), token_seed(22)).cuda()
    pos = torch.full((B,), T, dtype=torch.int32, device="cuda")
    assert m.status() == 0

    m.debug_stall(which, unit=unit, wait_limit_ns=1_000_000)
    bad = torch.empty(B, s.vocab_size, device="cuda")
    m.decode_step(nxt, pos, logits=bad)
    torch.cuda.synchronize()                      # the stalled launch returned
    assert m.status() == llb.LLAMA_ERR_DEVICE_TIMEOUT

    good = torch.empty(B, s.vocab_size, device="cuda")
    m.decode_step(nxt, pos, logits=good)          # the same step again, nothing armed
    torch.cuda.synchronize()
    assert m.status() == 0
    w64 = to_numpy_f64_weights(w)
    args = oracle_args(s)
    got = good.cpu().numpy()
    for b in (0, B - 1):
        seq = toks[b].cpu().tolist() + [int(nxt[b])]
        want = O.forward(args, w64, seq, 0, O.new_cache(args))[-1]
        assert rel_l2(got[b], want) <= BF16_TOL, (which, unit, b, rel_l2(got[b], want))
    m.close()


def test_stall_arguments_are_checked(llb):
    m = build_model(SHAPE, make_weights(SHAPE, 72))
    with pytest.raises(llb.LlamaError):
        m.debug_stall("projection", unit=-1)
    with pytest.raises(llb.LlamaError):
        m.debug_stall("attention", unit=0, wait_limit_ns=10)
    m.debug_stall("projection", unit=0)
    m.debug_stall("none")                         # disarmed before any launch took it
    assert m.status() == 0
    m.close()


# wq/wk/wv of this shape (6144 x 4096 weights) runs on CTA pairs: 300 tokens
# make 2 x 24 pair tiles, all split along K over the 74 pairs (41 or 42
# stages each); the SHAPE above runs its wq/wk/wv (4096 x 2048) on single SMs
# (4800 tokens: 38 x 16 tiles, 4 waves and a stream-K tail).
PAIR_SHAPE = ModelShape(dim=4096, n_layers=1, n_heads=32, n_kv_heads=8, vocab_size=512, max_seq_len=320,
                        max_batch_size=1, dtype="bf16", hidden=11008)


@pytest.mark.parametrize("shape,B,T,unit", [(SHAPE, 8, 600, 0), (SHAPE, 8, 600, 2), (PAIR_SHAPE, 1, 300, 0),
                                            (PAIR_SHAPE, 1, 300, 3)])
def test_stalled_prefill_projection_times_out_and_the_next_prefill_is_exact(llb, shape, B, T, unit):
    """The same for the prefill projections: the stall takes the first 16-bit
    projection launch, which is the prefill's wq/wk/wv."""
    s = shape
    w = make_weights(s, 73)
    m = build_model(s, w)
    toks = make_tokens(s.vocab_size, (B, T), token_seed(23)).cuda()
    m.debug_stall("projection", unit=unit, wait_limit_ns=1_000_000)
    bad = torch.empty(B, s.vocab_size, device="cuda")
    m.prefill(toks, logits=bad)
    torch.cuda.synchronize()
    assert m.status() == llb.LLAMA_ERR_DEVICE_TIMEOUT

    good = torch.empty(B, s.vocab_size, device="cuda")
    m.prefill(toks, logits=good)
    torch.cuda.synchronize()
    assert m.status() == 0
    w64 = to_numpy_f64_weights(w)
    args = oracle_args(s)
    for b in (0, B - 1):
        want = O.forward(args, w64, toks[b].cpu().tolist(), 0, O.new_cache(args))[-1]
        assert rel_l2(good[b].cpu().numpy(), want) <= BF16_TOL, (unit, b)
    m.close()
