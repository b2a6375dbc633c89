"""Pins of the oracle's generation loop (Admin Guide §8.5, source tour "The
decode loop in generate") against what the loop must equal without its
machinery: each row recomputed from scratch (a fresh forward over the whole
prefix, no KV cache, no lock-step schedule), prompt tokens never overwritten,
EOS cutting a row and stopping the loop once every row has it, and
log-probabilities equal to the log-softmax of freshly computed logits."""
import numpy as np
import pytest

from oracle import llama_oracle as O
from tests.helpers import oracle_args
from workloads import TINY, make_tokens, make_uniforms, make_weights, to_numpy_f64_weights

pytestmark = pytest.mark.filterwarnings("ignore")


@pytest.fixture(scope="module")
def model():
    s = TINY.replace(n_layers=1, max_seq_len=24)
    w = make_weights(s, 77)
    return s, oracle_args(s), to_numpy_f64_weights(w)


def _prompts(s, lens, seed):
    t = make_tokens(s.vocab_size, (len(lens), max(lens)), seed)
    return [t[b, :n].tolist() for b, n in enumerate(lens)]


def _fresh_logits(args, w, seq):
    """Logits predicting the position after seq, from scratch."""
    return O.forward(args, w, seq, 0, O.new_cache(args))[-1]


def test_greedy_generation_equals_per_row_recomputation(model):
    s, args, w = model
    prompts = _prompts(s, [3, 5, 1], 11)
    out, _ = O.generate(args, w, prompts, max_gen_len=6, temperature=0.0, echo=True)
    for b, p in enumerate(prompts):
        seq = list(p)
        while len(seq) < len(p) + 6:
            seq.append(O.greedy(_fresh_logits(args, w, seq)))
        assert out[b] == seq, b


def test_sampled_generation_equals_per_row_recomputation(model):
    s, args, w = model
    prompts = _prompts(s, [2, 4], 12)
    uni = make_uniforms((s.max_seq_len, 2), 12).numpy()
    out, _ = O.generate(args, w, prompts, max_gen_len=5, temperature=0.8, top_p=0.7, uniforms=uni, echo=False)
    for b, p in enumerate(prompts):
        seq = list(p)
        for pos in range(len(p), len(p) + 5):
            seq.append(O.sample_top_p(_fresh_logits(args, w, seq), 0.8, 0.7, float(uni[pos][b])))
        assert out[b] == seq[len(p):], b


def test_longer_prompts_are_kept_and_results_are_sliced(model):
    s, args, w = model
    prompts = _prompts(s, [2, 7], 13)
    echo, _ = O.generate(args, w, prompts, max_gen_len=3, temperature=0.0, echo=True)
    plain, _ = O.generate(args, w, prompts, max_gen_len=3, temperature=0.0, echo=False)
    for b, p in enumerate(prompts):
        assert echo[b][:len(p)] == p
        assert len(echo[b]) == len(p) + 3 and echo[b][len(p):] == plain[b]


def test_total_length_is_capped_by_max_seq_len(model):
    s, args, w = model
    prompts = _prompts(s, [20, 4], 14)
    out, _ = O.generate(args, w, prompts, max_gen_len=100, temperature=0.0, echo=True)
    # total_len = min(24, 100 + 20) = 24: every row is filled to position 24
    assert [len(t) for t in out] == [24, 24]


def test_eos_cuts_a_row_and_ends_the_loop(model, monkeypatch):
    s, args, w = model
    prompts = _prompts(s, [3, 3], 15)
    free, _ = O.generate(args, w, prompts, max_gen_len=6, temperature=0.0, echo=False)
    eos = free[0][2]                     # row 0's third generated token
    cut, _ = O.generate(args, w, prompts, max_gen_len=6, temperature=0.0, echo=False, eos_id=eos)
    for b in range(2):
        want = free[b][:free[b].index(eos)] if eos in free[b] else free[b]
        assert cut[b] == want, b
    # one row whose first generated token is EOS: one forward, empty result
    calls = []
    real = O.forward
    monkeypatch.setattr(O, "forward", lambda *a, **k: calls.append(1) or real(*a, **k))
    first = free[1][0]
    out, _ = O.generate(args, w, [prompts[1]], max_gen_len=6, temperature=0.0, eos_id=first)
    assert out == [[]] and len(calls) == 1


def test_logprobs_are_log_softmax_of_fresh_logits(model):
    s, args, w = model
    prompts = _prompts(s, [2, 4], 16)
    out, lps = O.generate(args, w, prompts, max_gen_len=4, temperature=0.0, echo=True, logprobs=True)
    for b in range(2):
        seq = out[b]
        assert lps[b][0] == 0.0 and len(lps[b]) == len(seq)
        for p in range(1, len(seq)):
            lg = _fresh_logits(args, w, seq[:p])
            want = lg[seq[p]] - (lg.max() + np.log(np.exp(lg - lg.max()).sum()))
            assert abs(lps[b][p] - want) < 1e-9, (b, p)
            if p >= len(prompts[b]):          # greedy picks: the row's largest log-probability
                assert abs(lps[b][p] - (lg.max() - (lg.max() + np.log(np.exp(lg - lg.max()).sum())))) < 1e-9


def test_no_position_left_to_generate(model):
    s, args, w = model
    prompts = _prompts(s, [5, 5], 17)
    out, lps = O.generate(args, w, prompts, max_gen_len=0, temperature=0.0, echo=True, logprobs=True)
    assert out == prompts
    for b, p in enumerate(prompts):
        lg = O.forward(args, w, p, 0, O.new_cache(args))
        assert np.allclose(lps[b][1:], O.token_logprobs(lg[:-1], p[1:]), atol=1e-12)
    none, _ = O.generate(args, w, prompts, max_gen_len=0, temperature=0.0, echo=False)
    assert none == [[], []]


def test_token_logprobs_closed_form():
    lg = np.array([[0.0, 0.0, 0.0, 0.0], [1.0, 2.0, 3.0, 4.0]])
    got = O.token_logprobs(lg, [2, 3])
    assert got[0] == pytest.approx(-np.log(4.0), abs=1e-15)
    assert got[1] == pytest.approx(4.0 - np.log(np.exp([1.0, 2.0, 3.0, 4.0]).sum()), abs=1e-14)
