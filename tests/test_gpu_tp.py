"""Tensor parallelism on one GPU: every rank of a group runs on cuda:0
(llama_tp_prefill_all / llama_tp_decode_step_all), each holding the weight
slices decoder_only_transformer_llama_b200.tp gives it -- column-parallel
wq/wk/wv, w1/w3 and the vocabulary projection, row-parallel wo and w2 (Admin
Guide §1.3 NOTE, §4.2; source tour, "One model.py") -- with the two
reductions per layer and the gathered logits done by the library's kernels.
The group's logits must match the unsharded oracle at the same tolerance as
the unsharded model: ragged prompts, greedy decode steps at per-row
positions, all-position logits of a prefill continued at start_pos > 0."""
import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import oracle_args, rel_l2
from workloads import ModelShape, make_tokens, make_weights, to_numpy_f64_weights, token_seed

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
# 8 query heads over 4 KV heads (n_rep 2), FFN 1536, vocabulary 1024: splits
# over 2 ranks (4 query heads, 2 KV heads, 768 features, 512 vocabulary rows
# each) and over 4 (2, 1, 384, 256)
SHAPE = ModelShape(dim=512, n_layers=2, n_heads=8, n_kv_heads=4, vocab_size=1024, max_seq_len=112,
                   max_batch_size=3, dtype="bf16", hidden=1536)


@pytest.fixture(scope="module")
def llb(cuda_device):
    import decoder_only_transformer_llama_b200 as m
    return m


def _group(llb, s, w, tp):
    g = llb.TPGroup(llb.args_from_shape(s), tp, device="cuda")
    g.load({"tok_embeddings": w["tok_embeddings"].cuda(), "norm": w["norm"].cuda(), "output": w["output"].cuda(),
            "layers": [{k: v.cuda() for k, v in layer.items()} for layer in w["layers"]]}, s)
    return g


@pytest.mark.parametrize("tp,dtype", [(2, "bf16"), (4, "bf16"), (2, "f16")])
def test_group_prefill_and_decode_match_the_oracle(llb, tp, dtype):
    s = SHAPE.replace(dtype=dtype)
    w = make_weights(s, 91)
    g = _group(llb, s, w, tp)
    B, T, steps = 3, 64, 6
    lens = [37, 64, 5]
    toks = make_tokens(s.vocab_size, (B, T), token_seed(31)).cuda()
    logits = torch.empty(B, s.vocab_size, device="cuda")
    g.prefill(toks, lens=lens, logits=logits)
    cur = torch.empty(B, dtype=torch.int32, device="cuda")
    llb.sample(logits, 0.0, 0.9, None, cur)
    seq = [toks[b, :lens[b]].cpu().tolist() for b in range(B)]
    got = [[logits[b].cpu().numpy().copy()] for b in range(B)]
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for _ in range(steps):
        for b in range(B):
            seq[b].append(int(cur[b]))
        lg = torch.empty(B, s.vocab_size, device="cuda")
        g.decode_step(cur, pos, temperature=0.0, next_tokens=cur, logits=lg, advance=True)
        torch.cuda.synchronize()
        for b in range(B):
            got[b].append(lg[b].cpu().numpy().copy())
    assert g.status() == 0
    assert pos.cpu().tolist() == [n + steps for n in lens]
    g.close()
    args = oracle_args(s)
    w64 = to_numpy_f64_weights(w)
    for b in range(B):
        want = O.forward(args, w64, seq[b], 0, O.new_cache(args))[lens[b] - 1:]
        err = rel_l2(np.stack(got[b]), want)
        assert err <= BF16_TOL, (tp, dtype, b, err)
        # the group's greedy pick is the argmax of its gathered logits
        for i in range(steps):
            assert seq[b][lens[b] + i] == O.greedy(got[b][i]), (b, i)


def test_group_all_position_logits_after_a_prefix(llb):
    """A prefix, then a continuation prefilled at start_pos > 0 with every
    position's logits: each rank fills its vocabulary slice of the rows."""
    s = SHAPE
    w = make_weights(s, 92)
    g = _group(llb, s, w, 2)
    B, P, T = 2, 20, 30
    prefix = make_tokens(s.vocab_size, (B, P), token_seed(32)).cuda()
    cont = make_tokens(s.vocab_size, (B, T), token_seed(33)).cuda()
    g.prefill(prefix)
    lg = torch.empty(B * T, s.vocab_size, device="cuda")
    g.prefill(cont, start_pos=P, logits=lg, all_logits=True)
    torch.cuda.synchronize()
    assert g.status() == 0
    g.close()
    args = oracle_args(s)
    w64 = to_numpy_f64_weights(w)
    got = lg.cpu().numpy()
    for b in range(B):
        seq = prefix[b].cpu().tolist() + cont[b].cpu().tolist()
        want = O.forward(args, w64, seq, 0, O.new_cache(args))[P:]
        assert rel_l2(got[b * T:(b + 1) * T], want) <= BF16_TOL, b


def test_shard_arguments_are_checked(llb):
    a = llb.args_from_shape(SHAPE)
    with pytest.raises(llb.LlamaError):
        llb.model_bytes(a, 0, 3)                  # 8 heads do not split over 3 ranks
    with pytest.raises(llb.LlamaError):
        llb.model_bytes(a, 2, 2)                  # rank outside the group
    sizes = llb.model_bytes(a, 1, 4)
    assert sizes["hidden"] == SHAPE.hidden // 4
    m = llb.Model(a, device="cuda", tp_rank=0, tp_size=2)
    tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(llb.LlamaError):
        m.decode_step(tok, pos)                   # a shard alone, never bound to its group
    m.close()
