"""The generation driver on the GPU (prefill, decode steps, sampling and
log-probability kernels) against the oracle: every generated token is the
oracle's choice on the same prefix (where the choice is not within rounding
of a tie or a nucleus boundary), prompt tokens are kept, log-probabilities
match the oracle's log-softmax, and EOS ends a row."""
import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import build_model, oracle_args
from workloads import TINY, ModelShape, make_tokens, make_uniforms, make_weights, to_numpy_f64_weights

pytestmark = pytest.mark.gpu

SMALL = ModelShape(dim=256, n_layers=2, n_heads=2, n_kv_heads=1, vocab_size=512, max_seq_len=64,
                   max_batch_size=3, dtype="bf16", hidden=768)


@pytest.fixture(scope="module")
def gen(cuda_device):
    import decoder_only_transformer_llama_b200.generate as g
    return g


def _prompts(s, lens, seed):
    t = make_tokens(s.vocab_size, (len(lens), max(lens)), seed)
    return [t[b, :n].tolist() for b, n in enumerate(lens)]


@pytest.mark.parametrize("shape,tol", [(TINY, 1e-4), (SMALL, 2e-2)])
def test_greedy_generation_with_logprobs(gen, shape, tol):
    """Greedy generation with log-probabilities.  `tol` is the model's logit
    bound (relative L2).  A log-probability moves by the chosen logit's error
    minus the softmax-weighted mean of all the row's logit errors, each about
    tol x RMS(logits); each position's log-probability must lie within
    4 x tol x RMS of that row's oracle logits of the oracle's."""
    w = make_weights(shape, 61)
    m = build_model(shape, w)
    prompts = _prompts(shape, [5, 12], 62)
    out, lps = gen.generate(m, prompts, max_gen_len=10, temperature=0.0, logprobs=True, echo=True)
    m.close()
    args, w64 = oracle_args(shape), to_numpy_f64_weights(w)
    for b, p in enumerate(prompts):
        seq = out[b]
        assert seq[:len(p)] == p and len(seq) == len(p) + 10
        lg = O.forward(args, w64, seq[:-1], 0, O.new_cache(args))      # row i predicts position i + 1
        want_lp = O.token_logprobs(lg, seq[1:])
        assert lps[b][0] == 0.0
        lp_tol = 4.0 * tol * np.sqrt(np.mean(lg ** 2, axis=1))
        diff = np.abs(np.asarray(lps[b][1:], dtype=np.float64) - want_lp)
        assert np.all(diff <= lp_tol), (b, float(np.max(diff / lp_tol)))
        for pos in range(len(p), len(seq)):
            row = lg[pos - 1]
            if O.sample_margins(row, 0.0, 0.9, 0.0) > 1e-2:
                assert seq[pos] == O.greedy(row), (b, pos)


def test_sampled_generation_and_eos(gen):
    s = TINY
    w = make_weights(s, 63)
    m = build_model(s, w)
    prompts = _prompts(s, [4, 7], 64)
    uni = make_uniforms((s.max_seq_len, 2), 65).cuda()
    out, _ = gen.generate(m, prompts, max_gen_len=8, temperature=0.8, top_p=0.9, uniforms=uni, echo=True)
    args, w64 = oracle_args(s), to_numpy_f64_weights(w)
    u = uni.cpu().numpy()
    for b, p in enumerate(prompts):
        seq = out[b]
        lg = O.forward(args, w64, seq[:-1], 0, O.new_cache(args))
        for pos in range(len(p), len(seq)):
            row = lg[pos - 1]
            assert seq[pos] in O.top_p_kept(row, 0.8, 0.9), (b, pos)
            if O.sample_margins(row, 0.8, 0.9, float(u[pos][b])) > 1e-4:
                assert seq[pos] == O.sample_top_p(row, 0.8, 0.9, float(u[pos][b])), (b, pos)
    # EOS: the first token row 0 generated ends row 0 at once
    eos = out[0][len(prompts[0])]
    cut, _ = gen.generate(m, prompts, max_gen_len=8, temperature=0.8, top_p=0.9, uniforms=uni, eos_id=eos)
    assert cut[0] == []
    gen_1 = out[1][len(prompts[1]):]
    assert cut[1] == (gen_1[:gen_1.index(eos)] if eos in gen_1 else gen_1)
    m.close()
