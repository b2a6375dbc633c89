"""Writes storage_error_7b.txt: the error that bfloat16 activation storage
alone causes in the full 32-layer 7B model, the scale the full-depth parity
test's bounds are taken from.

For each row of the 4 x 512 prompt batch (tokens of the benchmark's seeded
generator, weights drawn from the same distribution on the host), the oracle
runs the row exactly in fp64 and again with `store=round_bf16` (16-bit
storage at the points listed in the oracle's layer_forward), at the last
prompt position and two greedy decode positions (the exact run's own
tokens).  Recorded per row: the relative L2 distance of the two logit sets
and the RMS of their element-wise difference.  Only the oracle and the
seeded input generators are used; nothing comes from the CUDA path.

Run from the repository root:  python tests/golden/make_storage_error.py
(about 2 minutes per row on 8 cores).
"""
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import llama_oracle as O  # noqa: E402
from workloads import L7B, LazyF64Weights, make_tokens, make_weights, token_seed, weight_seed  # noqa: E402

SEED_INDEX = 5          # the full-depth test's weight and token seeds
B, T, STEPS = 4, 512, 2
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "storage_error_7b.txt")


def oracle_args(s):
    return O.Args(dim=s.dim, n_layers=s.n_layers, n_heads=s.n_heads, n_kv_heads=s.n_kv_heads,
                  vocab_size=s.vocab_size, multiple_of=s.multiple_of, ffn_dim_multiplier=s.ffn_dim_multiplier,
                  norm_eps=s.norm_eps, rope_theta=s.rope_theta, max_seq_len=s.max_seq_len)


def run_row(args, w, prompt, tokens_after, store):
    """Logits at the last prompt position and at each later token, one row,
    through the KV cache (prefill, then one token per step)."""
    cache = O.new_cache(args)
    out = [O.forward(args, w, prompt, 0, cache, logits_positions=[len(prompt) - 1], store=store)[0]]
    for i, tok in enumerate(tokens_after):
        out.append(O.forward(args, w, [tok], len(prompt) + i, cache, store=store)[0])
    return np.stack(out)


def main():
    s = L7B
    args = oracle_args(s)
    w = LazyF64Weights(make_weights(s, weight_seed(SEED_INDEX)))
    prompts = make_tokens(s.vocab_size, (B, T), token_seed(SEED_INDEX))
    lines = []
    for b in range(B):
        t0 = time.time()
        prompt = prompts[b].tolist()
        cache = O.new_cache(args)
        lg = O.forward(args, w, prompt, 0, cache, logits_positions=[T - 1])[0]
        toks = []
        for i in range(STEPS):          # the exact run's greedy continuation
            toks.append(O.greedy(lg))
            lg = O.forward(args, w, [toks[-1]], T + i, cache)[0]
        exact = run_row(args, w, prompt, toks, None)
        rounded = run_row(args, w, prompt, toks, O.round_bf16)
        rel = np.linalg.norm(rounded - exact) / np.linalg.norm(exact)
        rms = np.sqrt(np.mean((rounded - exact) ** 2))
        lines.append(f"row{b}: rel_l2={rel:.6e} rms_abs={rms:.6e} logits_rms={np.sqrt(np.mean(exact ** 2)):.6e}")
        print(lines[-1], f"({time.time() - t0:.0f} s)", flush=True)
    with open(OUT, "w") as f:
        f.write("# bfloat16 storage error of the full 32-layer 7B model (dim 4096, 32 heads, hidden 11008,\n"
                "# vocab 32000): oracle with store=round_bf16 against the exact fp64 oracle, logits at the\n"
                f"# last prompt position and {STEPS} greedy decode positions, prompts 4 x 512 from the seeded\n"
                f"# token generator (seed index {SEED_INDEX}), weights N(0, 0.02) bf16-rounded, norms 1 + N(0, 0.02)\n"
                "# drawn on the host.  Written by tests/golden/make_storage_error.py (oracle only).\n")
        for ln in lines:
            f.write(ln + "\n")


if __name__ == "__main__":
    main()
