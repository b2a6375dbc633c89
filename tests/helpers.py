"""Shared test plumbing: build a model through the C ABI from a seeded weight
dict, and compare GPU outputs with the oracle's."""
from __future__ import annotations

import numpy as np
import torch

from oracle import llama_oracle as O
from workloads import ModelShape, make_weights, to_numpy_f64_weights


def oracle_args(s: ModelShape, n_layers=None) -> O.Args:
    return O.Args(dim=s.dim, n_layers=s.n_layers if n_layers is None else n_layers, n_heads=s.n_heads,
                  n_kv_heads=s.n_kv_heads, vocab_size=s.vocab_size, multiple_of=s.multiple_of,
                  ffn_dim_multiplier=s.ffn_dim_multiplier, norm_eps=s.norm_eps, rope_theta=s.rope_theta,
                  max_seq_len=s.max_seq_len)


def build_model(s: ModelShape, weights: dict, device="cuda"):
    import decoder_only_transformer_llama_b200 as llb
    m = llb.Model(llb.args_from_shape(s), device=device)
    dev_w = {"tok_embeddings": weights["tok_embeddings"].to(device), "norm": weights["norm"].to(device),
             "output": weights["output"].to(device),
             "layers": [{k: v.to(device) for k, v in layer.items()} for layer in weights["layers"]]}
    m.load(dev_w)
    return m


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def top2_gap(logits) -> float:
    l = np.sort(np.asarray(logits, dtype=np.float64))[::-1]
    return float(l[0] - l[1])


def check_greedy(gpu_tokens, oracle_logits, gap=1e-2):
    """Greedy ids must agree wherever the oracle's top-2 gap exceeds `gap`.
    Returns (checked, skipped)."""
    checked = skipped = 0
    for tok, lg in zip(gpu_tokens, oracle_logits):
        if top2_gap(lg) > gap:
            assert int(tok) == O.greedy(lg), (int(tok), O.greedy(lg), top2_gap(lg))
            checked += 1
        else:
            skipped += 1
    return checked, skipped
