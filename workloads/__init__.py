"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds the five Llama-2-shaped workloads and the random number
draws that feed them: weights, token ids, prompt lengths and the uniforms
that drive top-p sampling.  It contains none of the method's arithmetic:
no normalisation, projection, attention or sampling happens here.  Both
sides of every parity test receive the very same tensors from here.

Shapes follow the model configuration table of "Llama 2 Reference
Implementation — Administrator & Developer Guide", §3.3 (ModelArgs) and
§8.4 (the model architecture in detail); the weights are random because the
real checkpoints are licence-gated (same guide, §7.1).

Draw order (fixed, documented): tok_embeddings; then per layer
attention_norm, wq, wk, wv, wo, ffn_norm, w1, w2, w3; then norm; output.
Matrices are N(0, 0.02); RMSNorm weights are 1 + N(0, 0.02) stored fp32.
16-bit models (bf16, f16) round each matrix to that type once, right after its draw.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

LAYER_WEIGHTS = ("attention_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w2", "w3")
NORM_WEIGHTS = ("attention_norm", "ffn_norm", "norm")


@dataclasses.dataclass(frozen=True)
class ModelShape:
    """Structural configuration (the pages' ModelArgs plus a storage dtype)."""
    dim: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    vocab_size: int
    multiple_of: int = 256
    ffn_dim_multiplier: Optional[float] = None
    norm_eps: float = 1e-5
    rope_theta: float = 10000.0
    max_seq_len: int = 2048
    max_batch_size: int = 32
    max_tokens: int = 0
    dtype: str = "bf16"  # "f32", "bf16" or "f16"
    hidden: int = 0  # FFN width as the workload states it (checked against the oracle's rule)

    @property
    def head_dim(self) -> int:
        return self.dim // self.n_heads

    @property
    def n_rep(self) -> int:
        return self.n_heads // self.n_kv_heads

    def replace(self, **kw) -> "ModelShape":
        return dataclasses.replace(self, **kw)


# --- The five workloads -----------------------------------------------------
# index 0: tiny fp32 parity model; 1: one 7B layer, decode microbench;
# 2: full 7B shape; 3: 13B shape, ragged batch; 4: 70B-shaped GQA slice.

TINY = ModelShape(dim=256, n_layers=2, n_heads=8, n_kv_heads=2, vocab_size=512,
                  max_seq_len=128, max_batch_size=2, dtype="f32", hidden=768)
L7B_LAYER = ModelShape(dim=4096, n_layers=1, n_heads=32, n_kv_heads=32, vocab_size=32000,
                       max_seq_len=4160, max_batch_size=32, max_tokens=64, hidden=11008)
L7B = ModelShape(dim=4096, n_layers=32, n_heads=32, n_kv_heads=32, vocab_size=32000,
                 max_seq_len=4096, max_batch_size=4, max_tokens=2048, hidden=11008)
L13B = ModelShape(dim=5120, n_layers=40, n_heads=40, n_kv_heads=40, vocab_size=32000,
                  max_seq_len=1152, max_batch_size=16, max_tokens=16 * 1024, hidden=13824)
L70B_SLICE = ModelShape(dim=8192, n_layers=16, n_heads=64, n_kv_heads=8, vocab_size=32000,
                        multiple_of=4096, ffn_dim_multiplier=1.3,
                        max_seq_len=4096, max_batch_size=8, max_tokens=8 * 2048, hidden=28672)

WORKLOADS: Dict[str, dict] = {
    "tiny_f32": dict(index=0, shape=TINY, batch=2, prompt_len=64, decode_steps=16),
    "7b_layer_decode": dict(index=1, shape=L7B_LAYER, batches=(1, 8, 32), contexts=(128, 1024, 4096)),
    "7b": dict(index=2, shape=L7B, batch=4, prompt_len=512, decode_steps=256,
               temperature=0.6, top_p=0.9),
    "13b_ragged": dict(index=3, shape=L13B, batch=16, min_len=64, max_len=1024, decode_steps=128),
    "70b_slice": dict(index=4, shape=L70B_SLICE, batch=8, prompt_len=2048, decode_to=4096),
    # the full 7B shape at batch 1 (same weights and prompt seed as "7b"): the
    # single-sequence decode case that a 7B roofline target is quoted on
    "7b_batch1": dict(index=2, shape=L7B, batch=1, prompt_len=512, decode_steps=256),
}


def weight_seed(index: int) -> int:
    return 1000 + index


def token_seed(index: int) -> int:
    return 2000 + index


def uniform_seed(index: int) -> int:
    return 3000 + index


def weight_shapes(s: ModelShape) -> Dict[str, tuple]:
    hd, H = s.head_dim, s.hidden
    return {
        "tok_embeddings": (s.vocab_size, s.dim),
        "attention_norm": (s.dim,),
        "wq": (s.n_heads * hd, s.dim),
        "wk": (s.n_kv_heads * hd, s.dim),
        "wv": (s.n_kv_heads * hd, s.dim),
        "wo": (s.dim, s.n_heads * hd),
        "ffn_norm": (s.dim,),
        "w1": (H, s.dim),
        "w2": (s.dim, H),
        "w3": (H, s.dim),
        "norm": (s.dim,),
        "output": (s.vocab_size, s.dim),
    }


def _draw(name: str, shape: tuple, gen: torch.Generator, device, dtype: str) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * 0.02
    if name in NORM_WEIGHTS:
        return t + 1.0  # fp32 norm weights
    half = {"bf16": torch.bfloat16, "f16": torch.float16}.get(dtype)
    return t.to(half) if half is not None else t


def make_weights(s: ModelShape, seed: int, device="cpu", n_layers: Optional[int] = None) -> dict:
    """All weights of a model as torch tensors on `device`, drawn in the fixed order.

    `n_layers` (<= s.n_layers) draws only the first layers; the draws of layer
    l do not depend on how many layers follow, so a truncated model holds the
    same first layers as the full one but a different `norm`/`output`.
    """
    L = s.n_layers if n_layers is None else n_layers
    shapes = weight_shapes(s)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    w = {"tok_embeddings": _draw("tok_embeddings", shapes["tok_embeddings"], gen, device, s.dtype),
         "layers": []}
    for _ in range(L):
        layer = {}
        for name in LAYER_WEIGHTS:
            layer[name] = _draw(name, shapes[name], gen, device, s.dtype)
        w["layers"].append(layer)
    w["norm"] = _draw("norm", shapes["norm"], gen, device, s.dtype)
    w["output"] = _draw("output", shapes["output"], gen, device, s.dtype)
    return w


def make_tokens(vocab: int, shape, seed: int, device="cpu") -> torch.Tensor:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randint(0, vocab, tuple(shape), generator=gen, dtype=torch.int32).to(device)


def make_lengths(batch: int, lo: int, hi: int, seed: int) -> List[int]:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return [int(v) for v in torch.randint(lo, hi + 1, (batch,), generator=gen)]


def make_uniforms(shape, seed: int, device="cpu") -> torch.Tensor:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.rand(tuple(shape), generator=gen, dtype=torch.float32).to(device)


def make_normal(shape, seed: int, device="cpu", dtype=torch.bfloat16, std: float = 1.0) -> torch.Tensor:
    """N(0, std) values, e.g. for a KV cache filled before a decode microbench."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return (torch.randn(tuple(shape), generator=gen, device=device, dtype=torch.float32) * std).to(dtype)


def to_numpy_f64_weights(w: dict) -> dict:
    """Upcast a weight dict to float64 numpy arrays (exact for bf16, fp16 and fp32)."""
    out = {"tok_embeddings": w["tok_embeddings"].detach().cpu().double().numpy(),
           "norm": w["norm"].detach().cpu().double().numpy(),
           "output": w["output"].detach().cpu().double().numpy(),
           "layers": []}
    for layer in w["layers"]:
        out["layers"].append({k: v.detach().cpu().double().numpy() for k, v in layer.items()})
    return out


class LazyF64Weights:
    """Dict-like view that upcasts one tensor at a time (for 7B+ shapes).

    Holding a 7B model in float64 takes ~54 GB; this view converts each
    matrix when the oracle reads it and keeps nothing.
    """

    def __init__(self, w: dict):
        self._w = w

    def __getitem__(self, key):
        if key == "layers":
            return [_LazyLayer(layer) for layer in self._w["layers"]]
        return _to_np(self._w[key])


class _LazyLayer:
    def __init__(self, layer: dict):
        self._layer = layer

    def __getitem__(self, key):
        return _to_np(self._layer[key])


def _to_np(t: torch.Tensor):
    return t.detach().cpu().float().numpy()  # exact for bf16; oracle upcasts to f64
