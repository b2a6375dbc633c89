"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the headers declare, sizes the arena as the Admin Guide's KV
footprint fixes, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

llb = pytest.importorskip("decoder_only_transformer_llama_b200",
                          reason="library not built (run decoder_only_transformer_llama_b200/build.py)")
from oracle import llama_oracle as O  # noqa: E402
from workloads import WORKLOADS  # noqa: E402


def _declared_symbols():
    names = set()
    for h in ("llama_b200.h", "llama_b200_ops.h"):
        with open(os.path.join(ROOT, "include", h)) as f:
            names |= set(re.findall(r"LLAMA_API\s+[\w\s\*]+?\b(llama_\w+)\s*\(", f.read()))
    return names


def test_library_exports_every_declared_symbol():
    names = _declared_symbols()
    assert len(names) >= 16
    for n in names:
        assert hasattr(llb.lib(), n), n
    assert set(llb.EXPORTED) == names


def test_struct_layout_matches_header():
    # 13 four-byte fields, no padding
    assert ctypes.sizeof(llb.ModelArgs) == 13 * 4
    assert ctypes.sizeof(llb.Sampling) == 8


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_model_bytes_for_every_workload(name):
    s = WORKLOADS[name]["shape"]
    sz = llb.model_bytes(llb.args_from_shape(s))
    assert sz["hidden"] == s.hidden == O.ffn_hidden_dim(s.dim, s.multiple_of, s.ffn_dim_multiplier)
    esz = 4 if s.dtype == "f32" else 2
    per_tensor = O.kv_cache_bytes_per_tensor(s.max_batch_size, s.max_seq_len, s.n_kv_heads, s.head_dim, esz)
    # the cache is two tensors per layer; each region is padded to 256 bytes at most once
    assert 2 * s.n_layers * per_tensor <= sz["kv"] <= 2 * s.n_layers * per_tensor + 512
    n_params = O.parameter_count(s.dim, s.n_layers, s.n_heads, s.n_kv_heads, s.vocab_size, s.hidden)
    n_norm = (2 * s.n_layers + 1) * s.dim
    expect = (n_params - n_norm) * esz + n_norm * 4
    assert expect <= sz["weights"] <= expect + 256 * (8 * s.n_layers + 4)
    assert sz["total"] == sz["weights"] + sz["kv"] + sz["workspace"]


def test_kv_bytes_match_admin_guide_figure():
    """7B, max_batch_size 4, max_seq_len 2048, 16-bit cache: 64 MiB per tensor per layer."""
    a = llb.make_args(4096, 32, 32, 32, 32000, max_seq_len=2048, max_batch_size=4, max_tokens=16)
    assert llb.model_bytes(a)["kv"] == 2 * 32 * 64 * 1024 * 1024


@pytest.mark.parametrize("kw,code", [
    (dict(dim=0), llb.LLAMA_ERR_INVALID_ARG),
    (dict(n_heads=3), llb.LLAMA_ERR_INVALID_ARG),              # dim % n_heads
    (dict(n_kv_heads=3), llb.LLAMA_ERR_INVALID_ARG),           # n_heads % n_kv_heads
    (dict(dim=512, n_heads=2), llb.LLAMA_ERR_INVALID_ARG),     # head_dim 256 unsupported
    (dict(max_batch_size=1000), llb.LLAMA_ERR_INVALID_ARG),
    (dict(max_seq_len=0), llb.LLAMA_ERR_INVALID_ARG),
    (dict(dtype="fp8"), None),
])
def test_model_bytes_rejects_bad_args(kw, code):
    base = dict(dim=256, n_layers=2, n_heads=8, n_kv_heads=2, vocab_size=512, max_seq_len=128, max_batch_size=2,
                dtype="f32")
    fp8 = kw.get("dtype") == "fp8"
    base.update({k: v for k, v in kw.items() if k != "dtype"})
    a = llb.make_args(**base)
    if fp8:
        a.dtype = 7   # no such dtype: the library itself must reject it
        code = llb.LLAMA_ERR_INVALID_ARG
    with pytest.raises(llb.LlamaError) as ei:
        llb.model_bytes(a)
    assert ei.value.code == code
    assert llb.last_error()


def test_create_rejects_null_and_small_arena_without_gpu():
    a = llb.make_args(256, 2, 8, 2, 512, max_seq_len=128, max_batch_size=2, dtype="f32")
    lib = llb.lib()
    h = ctypes.c_void_p()
    assert lib.llama_model_create(ctypes.byref(a), None, 1 << 30, None, ctypes.byref(h)) == llb.LLAMA_ERR_INVALID_ARG
    # misaligned arena pointer is refused before any device access
    assert lib.llama_model_create(ctypes.byref(a), 0x1001, 1 << 30, None, ctypes.byref(h)) == llb.LLAMA_ERR_INVALID_ARG
    total = llb.model_bytes(a)["total"]
    assert lib.llama_model_create(ctypes.byref(a), 0x100000, total - 1, None, ctypes.byref(h)) == llb.LLAMA_ERR_CAPACITY
    assert h.value is None


def test_calls_reject_null_model_and_bad_sizes():
    lib = llb.lib()
    assert lib.llama_prefill(None, 0x1000, None, 1, 1, 0, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_decode_step(None, 0x1000, 0x1000, 1, None, None, None, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_sample(None, 1, 10, 0.0, 0.9, None, 0x1000, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_sample(0x1000, 0, 10, 0.0, 0.9, None, 0x1000, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_sample(0x1000, 1, 10, 0.7, 0.9, None, 0x1000, None) == llb.LLAMA_ERR_INVALID_ARG  # no uniforms
    assert lib.llama_sample(0x1000, 1, 10, -1.0, 0.9, 0x1000, 0x1000, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_model_status(None, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_op_linear(None, 0x1000, 1, 1, 8, 1, 0x1000, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_op_linear(0x1000, 0x1000, 1, 1, 7, 1, 0x1000, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG  # K % 8
    # decode-shaped bf16 needs the scratch workspace
    assert lib.llama_op_linear(0x1000, 0x1000, 4, 128, 64, 1, 0x1000, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    # fp16 takes the same rules; an unknown dtype code is rejected
    assert lib.llama_op_linear(0x1000, 0x1000, 1, 1, 7, llb.LLAMA_F16, 0x1000, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_op_linear(0x1000, 0x1000, 4, 128, 64, llb.LLAMA_F16, 0x1000, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_op_linear(0x1000, 0x1000, 4, 128, 64, 7, 0x1000, None, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_op_linear_workspace_bytes() > 0
    assert lib.llama_op_rmsnorm(0x1000, 0x1000, 1, 6, 1e-5, 0x1000, 0, None) == llb.LLAMA_ERR_INVALID_ARG
    assert lib.llama_get_kv(None, 0, None, None, None) == llb.LLAMA_ERR_INVALID_ARG


def test_op_bindings_reject_mismatched_tensors():
    """The Python op wrappers check dtypes and shapes before the C call: a
    float16 operand never reaches the fp32 kernel, and mixed operand types,
    a non-fp32 output or an unsupported type raise ValueError."""
    import torch
    A16 = torch.zeros(4, 64, dtype=torch.float16)
    W16 = torch.zeros(128, 64, dtype=torch.float16)
    Wb = torch.zeros(128, 64, dtype=torch.bfloat16)
    out = torch.zeros(4, 128)
    with pytest.raises(ValueError):
        llb.op_linear(A16, Wb, out)                                   # mixed 16-bit types
    with pytest.raises(ValueError):
        llb.op_linear(A16, W16, torch.zeros(4, 128, dtype=torch.float16))   # output not fp32
    with pytest.raises(ValueError):
        llb.op_linear(A16, W16, torch.zeros(4, 127))                  # output shape
    with pytest.raises(ValueError):
        llb.op_linear(A16.to(torch.float64), W16.to(torch.float64), out)
    with pytest.raises(ValueError):
        llb.op_linear(A16, W16.t().contiguous().t(), out)             # W not contiguous
    with pytest.raises(ValueError):
        llb.op_linear_noalloc(A16, W16, out)                          # bf16 only
    with pytest.raises(ValueError):
        llb.op_linear_whole_tiles(torch.zeros(80, 64), torch.zeros(128, 64), torch.zeros(80, 128))
    x = torch.zeros(2, 64)
    with pytest.raises(ValueError):
        llb.op_rmsnorm(x, torch.zeros(64), 1e-5, torch.zeros(2, 64, dtype=torch.int32))
    with pytest.raises(ValueError):
        llb.op_rmsnorm(x.to(torch.bfloat16), torch.zeros(64), 1e-5, torch.zeros(2, 64))


class _FakeCudaTensor:
    """Stands in for a CUDA tensor on a machine without one: the binding's
    checks read its device, dtype, contiguity and size; asking for its
    address means a call got past them to the library."""
    is_cuda = True

    def __init__(self, shape, dtype, contiguous=True, device="cuda:0"):
        import torch
        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def contiguous(self):
        return self

    def numel(self):
        n = 1
        for d in self.shape:
            n *= d
        return n

    def data_ptr(self):
        raise RuntimeError("reached the library")


def _fake_model(dtype="bf16"):
    import torch
    m = object.__new__(llb.Model)
    m.args = llb.make_args(256, 2, 8, 2, 512, max_seq_len=64, max_batch_size=4, dtype=dtype)
    m.sizes = llb.model_bytes(m.args)
    m.arena = _FakeCudaTensor((m.sizes["total"],), torch.uint8)
    m.handle = None
    return m


def test_kernel_wrappers_refuse_host_mistyped_and_short_tensors():
    """Every wrapper that hands a kernel a pointer checks the tensor first:
    a host tensor, a wrong dtype, a non-contiguous view, a buffer shorter
    than the call writes, or a tensor on another GPU raises ValueError; a
    well-formed call passes the checks (and here reaches the stub)."""
    import torch
    F = _FakeCudaTensor
    V = 512
    with pytest.raises(ValueError):
        llb.sample(torch.zeros(2, V), 0.0, 0.9, None, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError):
        llb.token_logprobs(torch.zeros(3, V), torch.zeros(3, dtype=torch.int32), torch.zeros(3))
    with pytest.raises(ValueError):
        llb.sample(F((2, V), torch.float32), 0.0, 0.9, None, F((1,), torch.int32))       # out too short
    with pytest.raises(RuntimeError, match="reached the library"):
        llb.sample(F((2, V), torch.float32), 0.7, 0.9, F((2,), torch.float32), F((2,), torch.int32))

    m = _fake_model()
    tok = F((2, 5), torch.int32)
    with pytest.raises(ValueError):
        m.prefill(F((2, 5), torch.int64))                                               # token dtype
    with pytest.raises(ValueError):
        m.prefill(tok, lens=[3])                                                         # one len per row
    with pytest.raises(ValueError):
        m.prefill(tok, logits=F((2, V - 1), torch.float32))                              # last-token logits
    with pytest.raises(ValueError):
        m.prefill(tok, lens=[5, 4], logits=F((8, V), torch.float32), all_logits=True)    # 9 rows needed
    with pytest.raises(ValueError):
        m.prefill(F((2, 5), torch.int32, device="cuda:1"))                               # other GPU
    with pytest.raises(RuntimeError, match="reached the library"):
        m.prefill(tok, lens=[5, 4], logits=F((9, V), torch.float32), all_logits=True)

    t1, p1 = F((2,), torch.int32), F((2,), torch.int32)
    with pytest.raises(ValueError):
        m.decode_step(t1, F((2,), torch.int64))                                          # positions int32
    with pytest.raises(ValueError):
        m.decode_step(t1, p1, temperature=0.0, next_tokens=F((2,), torch.int32, contiguous=False))
    with pytest.raises(ValueError):
        m.decode_step(t1, p1, temperature=0.7, uniforms=F((2,), torch.float64), next_tokens=t1)
    with pytest.raises(ValueError):
        m.decode_step(t1, p1, logits=F((1, V), torch.float32))
    with pytest.raises(RuntimeError, match="reached the library"):
        m.decode_step(t1, p1, temperature=0.7, uniforms=F((2,), torch.float32), next_tokens=t1,
                      logits=F((2, V), torch.float32))

    with pytest.raises(ValueError):
        m.set_weight(-1, "norm", F((256,), torch.bfloat16))                              # norms are fp32
    with pytest.raises(ValueError):
        m.set_weight(0, "wq", F((256, 255), torch.bfloat16))                             # short matrix
    with pytest.raises(ValueError):
        _fake_model("f16").set_weight(0, "wk", F((64, 256), torch.bfloat16))             # model is fp16
    with pytest.raises(RuntimeError, match="reached the library"):
        m.set_weight(0, "w2", F((256, m.sizes["hidden"]), torch.bfloat16))
