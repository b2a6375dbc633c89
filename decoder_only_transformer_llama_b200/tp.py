"""Tensor-parallel sharding plan of the decoder (host side, data slicing only).

The reference's only model-parallel strategy (Admin Guide §1.3 NOTE on
fairscale, §4.2 "Single-host, multi-GPU", §6.1 "Hot path"; source tour, "One
model.py"): every matrix that produces heads or hidden features is split by
output rows (column-parallel: wq, wk, wv, w1, w3 and the vocabulary
projection), every matrix that consumes them is split by input columns
(row-parallel: wo, w2), so each rank computes whole attention heads and whole
SwiGLU features on its own and the two row-parallel products leave partial
sums of the residual update that the ranks add together (two all-reduces per
layer).  The vocabulary projection leaves each rank the logits of its slice of
the vocabulary (gathered across ranks).  The token embedding and the three
RMSNorm weights are replicated.

Query head h reads KV head h // n_rep (repeat_kv), so giving rank r the query
heads [r * nh/tp, (r+1) * nh/tp) and the KV heads [r * nkv/tp, (r+1) * nkv/tp)
keeps every query group on the rank that holds its KV head: the plan needs
n_kv_heads % tp == 0.

This module only decides which rows and columns each rank holds and cuts
the weight tensors accordingly; no arithmetic of the forward pass happens
here.
"""
from __future__ import annotations

import dataclasses
from typing import Dict


@dataclasses.dataclass(frozen=True)
class ShardPlan:
    """Index ranges [begin, end) that rank `rank` of `tp` holds."""
    rank: int
    tp: int
    heads: tuple
    kv_heads: tuple
    hidden: tuple
    vocab: tuple
    head_dim: int

    @property
    def q_rows(self) -> tuple:
        return (self.heads[0] * self.head_dim, self.heads[1] * self.head_dim)

    @property
    def kv_rows(self) -> tuple:
        return (self.kv_heads[0] * self.head_dim, self.kv_heads[1] * self.head_dim)


def _split(n: int, tp: int, r: int, what: str) -> tuple:
    if n % tp:
        raise ValueError(f"{what} = {n} is not divisible by the tensor-parallel size {tp}")
    k = n // tp
    return (r * k, (r + 1) * k)


def shard_plan(n_heads: int, n_kv_heads: int, head_dim: int, hidden: int, vocab: int, rank: int,
               tp: int) -> ShardPlan:
    if tp < 1 or not 0 <= rank < tp:
        raise ValueError(f"rank {rank} outside a tensor-parallel group of {tp}")
    return ShardPlan(rank=rank, tp=tp, heads=_split(n_heads, tp, rank, "n_heads"),
                     kv_heads=_split(n_kv_heads, tp, rank, "n_kv_heads"),
                     hidden=_split(hidden, tp, rank, "the FFN hidden width"),
                     vocab=_split(vocab, tp, rank, "vocab_size"), head_dim=head_dim)


def plan_for(shape, rank: int, tp: int) -> ShardPlan:
    """The plan of a workloads.ModelShape-like object (fields n_heads,
    n_kv_heads, head_dim, hidden, vocab_size)."""
    return shard_plan(shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.hidden, shape.vocab_size, rank, tp)


def shard_layer(layer: Dict, plan: ShardPlan) -> Dict:
    """One layer's weights (nn.Linear layout [out, in]) cut for `plan`'s rank."""
    q0, q1 = plan.q_rows
    k0, k1 = plan.kv_rows
    h0, h1 = plan.hidden
    return {
        "attention_norm": layer["attention_norm"],
        "wq": layer["wq"][q0:q1],
        "wk": layer["wk"][k0:k1],
        "wv": layer["wv"][k0:k1],
        "wo": layer["wo"][:, q0:q1],
        "ffn_norm": layer["ffn_norm"],
        "w1": layer["w1"][h0:h1],
        "w2": layer["w2"][:, h0:h1],
        "w3": layer["w3"][h0:h1],
    }


def shard_weights(w: Dict, plan: ShardPlan) -> Dict:
    """A whole weight dict (workloads layout) cut for `plan`'s rank: sliced
    views of the same tensors or arrays (call .contiguous() / np.ascontiguousarray
    before handing them to a kernel)."""
    v0, v1 = plan.vocab
    return {"tok_embeddings": w["tok_embeddings"], "norm": w["norm"], "output": w["output"][v0:v1],
            "layers": [shard_layer(layer, plan) for layer in w["layers"]]}
