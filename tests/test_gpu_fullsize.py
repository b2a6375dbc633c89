"""Parity at the workloads' full layer dimensions (7B, 13B with ragged
prompts, 70B GQA slice), with the model truncated to two layers so that the
fp64 oracle can recompute sampled rows in seconds, and the full 32-layer 7B
model on one sampled row.  The GPU runs the same
launch configuration as the benchmark (batched prefill, then batched decode
steps at per-row positions); the oracle recomputes one or two rows from
scratch, teacher-forced on the GPU's greedy tokens."""
import os

import numpy as np
import pytest
import torch

from oracle import llama_oracle as O
from tests.helpers import build_model, check_greedy, oracle_args, rel_l2
from workloads import (L7B, L13B, L70B_SLICE, LazyF64Weights, make_lengths, make_tokens, make_weights,
                       token_seed, weight_seed)

pytestmark = pytest.mark.gpu
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def llb(cuda_device):
    import decoder_only_transformer_llama_b200 as m
    return m


def _run(llb, shape, B, T, lens, steps, rows, seed_idx, start_pos=0, tol=BF16_TOL, gap=1e-2):
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
        err = rel_l2(np.stack(got[b]), want)
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


def _storage_error_7b():
    """Per-row figures of tests/golden/storage_error_7b.txt (written by
    make_storage_error.py from the oracle alone)."""
    rows = []
    with open(os.path.join(os.path.dirname(__file__), "golden", "storage_error_7b.txt")) as f:
        for line in f:
            if line.startswith("row"):
                kv = dict(item.split("=") for item in line.split(":", 1)[1].split())
                rows.append({k: float(v) for k, v in kv.items()})
    assert len(rows) == 4
    return rows


def test_7b_full_depth_benchmark_configuration(llb):
    """The whole 32-layer 7B model in the benchmark's launch configuration
    (4 x 512 prefill, then batched decode steps); the oracle recomputes row 2
    (514 tokens through 32 layers, about a minute on the host).

    Over 32 layers the rounding of bfloat16 activation storage compounds
    past the 2e-2 that holds at two layers: the oracle with bf16 storage
    (round_bf16 at its storage points) is 4.3e-2 to 4.6e-2 from the exact
    oracle at this depth, on each of the batch's four rows.  The bounds are therefore that storage error's, from
    tests/golden/storage_error_7b.txt: relative L2 within 1.5 x the largest
    per-row figure, and greedy ids identical wherever the oracle's top-2 gap
    exceeds 8 x the largest RMS element-wise difference."""
    err = _storage_error_7b()
    tol = 1.5 * max(r["rel_l2"] for r in err)
    gap = 8.0 * max(r["rms_abs"] for r in err)
    _run(llb, L7B, B=4, T=512, lens=[512] * 4, steps=2, rows=[2], seed_idx=5, tol=tol, gap=gap)


def test_13b_dims_ragged_prefill_then_decode(llb):
    """13B layer dimensions, 16 prompts of seeded lengths in [64, 1024]
    right-padded to a rectangle, 2 decode steps; oracle on the two shortest rows."""
    s = L13B.replace(n_layers=2)
    lens = make_lengths(16, 64, 1024, token_seed(3))
    T = max(lens)
    order = sorted(range(16), key=lambda b: lens[b])
    _run(llb, s, B=16, T=T, lens=lens, steps=2, rows=order[:2], seed_idx=3)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_70b_gqa_dims_prefill_then_decode(llb, dtype):
    """70B layer dimensions (64 query heads over 8 KV heads, hidden 28672),
    batch 8 x 256 prefill, 2 decode steps; oracle on row 5; bf16 and fp16."""
    s = L70B_SLICE.replace(n_layers=2, max_tokens=8 * 256, dtype=dtype)
    _run(llb, s, B=8, T=256, lens=[256] * 8, steps=2, rows=[5], seed_idx=4)
