"""The generation driver's host logic on the CPU: a stand-in model answers
prefill / decode_step with the oracle's forward pass, and the stand-in
sampling and log-probability calls use the oracle's functions, so the
driver's own part (the lock-step schedule, keeping prompt tokens, EOS and the
early exit, slicing, echo, log-probability alignment) must reproduce the
oracle's generate exactly."""
import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import oracle_args
from workloads import TINY, make_tokens, make_uniforms, make_weights, to_numpy_f64_weights


class _Arena:
    device = torch.device("cpu")


class FakeModel:
    """prefill / decode_step through the oracle, one KV cache per row."""

    def __init__(self, shape, w64):
        self.shape = shape
        self.oargs = oracle_args(shape)
        self.w = w64
        self.args = type("A", (), {"max_seq_len": shape.max_seq_len, "vocab_size": shape.vocab_size,
                                   "max_batch_size": shape.max_batch_size})()
        self.arena = _Arena()
        self.caches = None
        self.calls = []

    def prefill(self, tokens, lens=None, start_pos=0, logits=None, all_logits=False, stream=None):
        assert start_pos == 0 and lens is None
        self.calls.append(("prefill", tokens.shape[1]))
        self.caches = [O.new_cache(self.oargs) for _ in range(tokens.shape[0])]
        for b in range(tokens.shape[0]):
            lg = O.forward(self.oargs, self.w, tokens[b].tolist(), 0, self.caches[b])
            if all_logits:
                logits[b].copy_(torch.from_numpy(lg))
            else:
                logits[b].copy_(torch.from_numpy(lg[-1]))
        return logits

    def decode_step(self, tokens, pos, logits=None, **kw):
        self.calls.append(("decode", int(pos[0])))
        assert len(set(pos.tolist())) == 1   # all rows at one position
        for b in range(tokens.shape[0]):
            lg = O.forward(self.oargs, self.w, [int(tokens[b])], int(pos[b]), self.caches[b])
            logits[b].copy_(torch.from_numpy(lg[-1]))

    def status(self):
        return 0


def _fake_sample(logits, temperature, top_p, uniforms, out, stream=None):
    for b in range(logits.shape[0]):
        row = logits[b].numpy().astype(np.float64)
        out[b] = O.greedy(row) if temperature == 0 else O.sample_top_p(row, temperature, top_p, float(uniforms[b]))
    return out


def _fake_logprobs(logits, tokens, out, stream=None):
    out.copy_(torch.from_numpy(O.token_logprobs(logits.numpy().astype(np.float64), tokens.numpy()).astype(np.float32)))
    return out


@pytest.fixture(scope="module")
def setup():
    s = TINY.replace(n_layers=1, max_seq_len=20, max_batch_size=3)
    w = make_weights(s, 55)
    return s, to_numpy_f64_weights(w)


@pytest.fixture
def gen(monkeypatch):
    import decoder_only_transformer_llama_b200.generate as g
    monkeypatch.setattr(g, "sample", _fake_sample)
    monkeypatch.setattr(g, "token_logprobs", _fake_logprobs)
    return g


def _prompts(s, lens, seed):
    t = make_tokens(s.vocab_size, (len(lens), max(lens)), seed)
    return [t[b, :n].tolist() for b, n in enumerate(lens)]


@pytest.mark.parametrize("lens,max_gen,temp,echo,logprobs", [
    ([3, 5, 1], 6, 0.0, True, True),
    ([4, 4], 5, 0.7, False, True),
    ([2, 9, 6], 30, 0.0, False, False),     # total_len capped by max_seq_len 20
    ([5, 5, 5], 0, 0.0, True, True),        # nothing to generate
])
def test_driver_reproduces_the_oracle_loop(setup, gen, lens, max_gen, temp, echo, logprobs):
    s, w64 = setup
    prompts = _prompts(s, lens, 21 + sum(lens))
    uni = make_uniforms((s.max_seq_len, len(lens)), 31)
    m = FakeModel(s, w64)
    got_t, got_l = gen.generate(m, prompts, max_gen_len=max_gen, temperature=temp, top_p=0.8,
                                uniforms=uni if temp > 0 else None, logprobs=logprobs, echo=echo)
    want_t, want_l = O.generate(m.oargs, w64, prompts, max_gen_len=max_gen, temperature=temp, top_p=0.8,
                                uniforms=uni.numpy(), logprobs=logprobs, echo=echo)
    assert got_t == want_t
    if logprobs:
        for g_, w_ in zip(got_l, want_l):
            np.testing.assert_allclose(g_, w_, atol=1e-5)
    else:
        assert got_l is None
    # one prefill of the shortest prompt, then one decode step per later position
    if min(lens) < min(s.max_seq_len, max_gen + max(lens)):
        assert m.calls[0] == ("prefill", min(lens))
        assert [c[1] for c in m.calls[1:]] == list(range(min(lens), min(lens) + len(m.calls) - 1))


def test_driver_eos_and_early_exit(setup, gen):
    s, w64 = setup
    prompts = _prompts(s, [3, 3], 41)
    m = FakeModel(s, w64)
    free, _ = gen.generate(m, prompts, max_gen_len=8, temperature=0.0)
    eos = free[1][1]
    m = FakeModel(s, w64)
    got, _ = gen.generate(m, prompts, max_gen_len=8, temperature=0.0, eos_id=eos)
    want, _ = O.generate(m.oargs, w64, prompts, max_gen_len=8, temperature=0.0, eos_id=eos)
    assert got == want
    m = FakeModel(s, w64)
    got, _ = gen.generate(m, [prompts[0]], max_gen_len=8, temperature=0.0, eos_id=free[0][0])
    assert got == [[]] and len(m.calls) == 1


def test_driver_argument_checks(setup, gen):
    s, w64 = setup
    m = FakeModel(s, w64)
    with pytest.raises(ValueError):
        gen.generate(m, [[1, 2]], temperature=0.5)                       # no uniforms
    with pytest.raises(ValueError):
        gen.generate(m, [[1]] * (s.max_batch_size + 1), temperature=0.0)  # too many rows
    with pytest.raises(ValueError):
        gen.generate(m, [[]], temperature=0.0)                            # empty prompt
