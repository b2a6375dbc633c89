"""Parity at the workloads' full layer dimensions (7B, 13B with ragged
prompts, 70B GQA slice), with the model truncated to two layers so that the
fp64 oracle can recompute sampled rows in seconds, and the full 32-layer 7B
model on one sampled row.  The GPU runs the same
launch configuration as the benchmark (batched prefill, then batched decode
steps at per-row positions); the oracle recomputes one or two rows from
scratch, teacher-forced on the GPU's greedy tokens."""
import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import build_model, check_greedy, oracle_args, rel_l2
from workloads import (L7B, L13B, L70B_SLICE, LazyF64Weights, make_lengths, make_normal, make_tokens,
                       make_weights, token_seed, weight_seed)

pytestmark = pytest.mark.gpu
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def llb(cuda_device):
    import decoder_only_transformer_llama_b200 as m
    return m


def _run(llb, shape, B, T, lens, steps, rows, seed_idx, start_pos=0, tol=BF16_TOL, gap=1e-2,
         storage_bound=False, storage_gap=False):
    """Prefill B prompts (right-padded to T, real lengths `lens`), then `steps`
    greedy decode steps at per-row positions; the oracle recomputes `rows`
    teacher-forced on the GPU's tokens.  With `storage_bound`, the oracle runs
    each row a second time with bfloat16 storage (store=round_bf16) and the
    bounds become that storage error's on these very weights and tokens:
    rel-L2 <= 1.5 x rel-L2(rounded, exact), greedy ids equal where the top-2
    gap exceeds 8 x the RMS of (rounded - exact).  With `storage_gap` only the
    greedy gap is taken from it (the rel-L2 bound stays `tol`)."""
    s = shape
    w = make_weights(s, weight_seed(seed_idx), device="cuda")
    m = build_model(s, w)
    toks = make_tokens(s.vocab_size, (B, T), token_seed(seed_idx)).cuda()
    logits = torch.empty(B, s.vocab_size, device="cuda")
    m.prefill(toks, lens=lens, logits=logits)
    cur = torch.empty(B, dtype=torch.int32, device="cuda")
    llb.sample(logits, 0.0, 0.9, None, cur)
    got = [[logits[b].cpu().numpy().copy()] for b in range(B)]
    seqs = [toks[b, :lens[b]].cpu().tolist() for b in range(B)]
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for _ in range(steps):
        for b in range(B):
            seqs[b].append(int(cur[b]))
        lg = torch.empty(B, s.vocab_size, device="cuda")
        m.decode_step(cur, pos, temperature=0.0, next_tokens=cur, logits=lg, advance=True)
        torch.cuda.synchronize()
        for b in range(B):
            got[b].append(lg[b].cpu().numpy().copy())
    assert m.status() == 0
    m.close()
    args = oracle_args(s)
    lw = LazyF64Weights({k: (v.cpu() if k != "layers" else [{n: t.cpu() for n, t in l.items()} for l in v])
                         for k, v in w.items()})
    del w
    for b in rows:
        L = lens[b]
        positions = list(range(L - 1, L + steps))
        want = O.forward(args, lw, seqs[b], 0, O.new_cache(args), logits_positions=positions)
        g = np.stack(got[b])
        if storage_bound or storage_gap:
            rounded = O.forward(args, lw, seqs[b], 0, O.new_cache(args), logits_positions=positions,
                                store=O.round_bf16)
            storage = rel_l2(rounded, want)
            if storage_bound:
                tol = 1.5 * storage
            gap = 8.0 * float(np.sqrt(np.mean((rounded - want) ** 2)))
            print(f"row {b}: bf16 storage error of the oracle {storage:.3e}; GPU to the bf16-storage oracle "
                  f"{rel_l2(g, rounded):.3e}")
        err = rel_l2(g, want)
        print(f"{s.n_layers} layers, dim {s.dim}, {s.dtype}: row {b} rel-L2 {err:.3e} (bound {tol:.3e})")
        assert err <= tol, (b, err)
        check_greedy(seqs[b][L:], want[:steps], gap)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_7b_dims_prefill_4x512_then_decode(llb, dtype):
    """7B layer dimensions, batch 4 x 512 prefill (the benchmark's launch
    configuration), 3 greedy decode steps; oracle on rows 0 and 3; bf16 and
    the reference's own fp16."""
    s = L7B.replace(n_layers=2, dtype=dtype)
    _run(llb, s, B=4, T=512, lens=[512] * 4, steps=3, rows=[0, 3], seed_idx=2)


@pytest.mark.slow
def test_7b_full_depth_benchmark_configuration(llb):
    """The whole 32-layer 7B model in the benchmark's launch configuration
    (4 x 512 prefill, then batched decode steps); the oracle recomputes row 2
    (514 tokens through 32 layers) exactly and again with bfloat16 storage.

    Over 32 layers the rounding of bfloat16 activation storage compounds
    past the 2e-2 that holds at two layers (tests/golden/storage_error_7b.txt
    records 4.3e-2 to 4.6e-2 on four rows of host-drawn weights).  The bounds
    here are therefore the storage error of the oracle itself on the very
    weights and tokens under test: relative L2 within 1.5 x rel-L2(bf16-storage
    oracle, exact oracle), greedy ids identical wherever the exact oracle's
    top-2 gap exceeds 8 x the RMS element-wise storage error."""
    _run(llb, L7B, B=4, T=512, lens=[512] * 4, steps=2, rows=[2], seed_idx=5, storage_bound=True)


def test_13b_dims_ragged_prefill_then_decode(llb):
    """13B layer dimensions, 16 prompts of seeded lengths in [64, 1024]
    right-padded to a rectangle, then the workload's 128 greedy decode steps
    at per-row positions; oracle on the shortest and the longest row.  Logits
    within rel-L2 2e-2 at every step.  Over 128 teacher-forced steps some
    oracle top-2 gaps fall below what bf16 storage of the cache and
    activations can resolve (RMS logit error ~1.6e-2 here, so gaps of a few
    hundredths can flip), so greedy ids must agree where the gap exceeds
    8 x the RMS of the oracle's own bf16-storage error on these rows."""
    s = L13B.replace(n_layers=2)
    lens = make_lengths(16, 64, 1024, token_seed(3))
    T = max(lens)
    order = sorted(range(16), key=lambda b: lens[b])
    _run(llb, s, B=16, T=T, lens=lens, steps=128, rows=[order[0], order[-1]], seed_idx=3, storage_gap=True)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_70b_gqa_dims_prefill_then_decode(llb, dtype):
    """70B layer dimensions (64 query heads over 8 KV heads, hidden 28672),
    batch 8 x 256 prefill, 2 decode steps; oracle on row 5; bf16 and fp16."""
    s = L70B_SLICE.replace(n_layers=2, max_tokens=8 * 256, dtype=dtype)
    _run(llb, s, B=8, T=256, lens=[256] * 8, steps=2, rows=[5], seed_idx=4)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_70b_gqa_decode_at_long_context(llb, dtype):
    """70B layer dimensions (64 query heads over 8 KV heads: n_rep 8), two
    layers, max_seq_len 4096.  Both layers' caches are filled through
    llama_get_kv with N(0, 1) values for positions [0, 4095), then one decode
    step at per-row positions: 4095 (the last cache position, 4096 keys) for
    most rows, shorter contexts for others, so rows of different lengths share
    one split-KV plan and the 8-head query groups are merged across splits at
    4096 keys.  The oracle recomputes four rows from the same cache contents."""
    s = L70B_SLICE.replace(n_layers=2, max_tokens=64, dtype=dtype)
    w = make_weights(s, weight_seed(4), device="cuda")
    m = build_model(s, w)
    B, S = 8, s.max_seq_len
    pos_l = [S - 1, S - 1, 3000, 2049, S - 1, 64, S - 2, S - 1]
    fills = []
    for l in range(s.n_layers):
        kview, vview = m.kv_tensors(l)
        fk = make_normal((B, S - 1, s.n_kv_heads, s.head_dim), 21 + 2 * l, device="cuda", dtype=kview.dtype)
        fv = make_normal((B, S - 1, s.n_kv_heads, s.head_dim), 22 + 2 * l, device="cuda", dtype=kview.dtype)
        kview[:B, :S - 1].copy_(fk)
        vview[:B, :S - 1].copy_(fv)
        fills.append((fk.cpu(), fv.cpu()))
    toks = make_tokens(s.vocab_size, (B,), token_seed(4)).cuda()
    pos = torch.tensor(pos_l, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, s.vocab_size, device="cuda")
    m.decode_step(toks, pos, logits=logits)
    torch.cuda.synchronize()
    assert m.status() == 0
    got = logits.cpu().numpy()
    m.close()
    args = oracle_args(s)
    lw = LazyF64Weights({k: (v.cpu() if k != "layers" else [{n: t.cpu() for n, t in l.items()} for l in v])
                         for k, v in w.items()})
    del w
    for b in (0, 2, 5, 6):
        p = pos_l[b]
        cache = O.new_cache(args)
        for l in range(s.n_layers):
            cache.k[l][:p] = fills[l][0][b, :p].double().numpy()
            cache.v[l][:p] = fills[l][1][b, :p].double().numpy()
        want = O.forward(args, lw, [int(toks[b])], p, cache)[0]
        err = rel_l2(got[b], want)
        print(f"70B dims, {dtype}, row {b} at position {p}: rel-L2 {err:.3e}")
        assert err <= BF16_TOL, (b, p, err)
