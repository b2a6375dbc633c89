"""Python binding of libllama_b200.so (argument marshalling only).

Every step of the forward pass and of sampling runs in the library's CUDA
kernels; this module only turns torch tensors into device pointers and
streams, and raises on non-zero status codes.  PyTorch provides device memory
(the model arena) and streams.  There is no CPU path: if the shared library
has not been built, importing this package raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libllama_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python decoder_only_transformer_llama_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

LLAMA_OK = 0
LLAMA_ERR_INVALID_ARG = 1
LLAMA_ERR_CAPACITY = 2
LLAMA_ERR_CUDA = 3
LLAMA_ERR_DEVICE_TIMEOUT = 4
LLAMA_ERR_TOKEN_RANGE = 5
LLAMA_F32 = 0
LLAMA_BF16 = 1
LLAMA_F16 = 2
LLAMA_DECODE_ADVANCE = 1

WEIGHT_IDS = {"tok_embeddings": 0, "norm": 1, "output": 2, "attention_norm": 3, "wq": 4, "wk": 5,
              "wv": 6, "wo": 7, "ffn_norm": 8, "w1": 9, "w2": 10, "w3": 11}

EXPORTED = ("llama_model_bytes", "llama_model_create", "llama_set_weight", "llama_get_kv",
            "llama_prefill", "llama_decode_step", "llama_sample", "llama_model_status",
            "llama_model_destroy", "llama_last_error", "llama_launch_count",
            "llama_op_rmsnorm", "llama_op_linear", "llama_op_linear_workspace_bytes", "llama_op_linear_noalloc",
            "llama_profile_start", "llama_profile_stop", "llama_token_logprobs", "llama_timeline_start",
            "llama_timeline_stop", "llama_debug_stall", "llama_model_bytes_tp", "llama_model_create_tp",
            "llama_tp_prefill_all", "llama_tp_decode_step_all", "llama_tp_buffers", "llama_tp_bind")
LLAMA_STALL_NONE, LLAMA_STALL_PROJECTION, LLAMA_STALL_ATTENTION = 0, 1, 2
TIMELINE_KINDS = {0: "embed", 1: "projection", 2: "attention", 3: "sample", 4: "rmsnorm"}


class LlamaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


_DTYPES = {"f32": LLAMA_F32, "bf16": LLAMA_BF16, "f16": LLAMA_F16}


class ModelArgs(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("vocab_size", ctypes.c_int32),
                ("multiple_of", ctypes.c_int32), ("ffn_dim_multiplier", ctypes.c_float),
                ("norm_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("max_seq_len", ctypes.c_int32), ("max_batch_size", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class Sampling(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("top_p", ctypes.c_float)]


_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t


def _sig(name, restype, argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = argtypes
    return fn


_sig("llama_model_bytes", _i, [ctypes.POINTER(ModelArgs), ctypes.POINTER(_sz), ctypes.POINTER(_sz),
                                ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(ctypes.c_int32)])
_sig("llama_model_create", _i, [ctypes.POINTER(ModelArgs), _vp, _sz, _vp, ctypes.POINTER(_vp)])
_sig("llama_set_weight", _i, [_vp, _i, _i, _vp, _vp])
_sig("llama_get_kv", _i, [_vp, _i, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(ctypes.c_int64)])
_sig("llama_prefill", _i, [_vp, _vp, ctypes.POINTER(ctypes.c_int32), _i, _i, _i, _vp, _i, _vp])
_sig("llama_decode_step", _i, [_vp, _vp, _vp, _i, ctypes.POINTER(Sampling), _vp, _vp, _vp, _i, _vp])
_sig("llama_sample", _i, [_vp, _i, _i, _f, _f, _vp, _vp, _vp])
_sig("llama_model_status", _i, [_vp, ctypes.POINTER(ctypes.c_int)])
_sig("llama_model_destroy", _i, [_vp])
_sig("llama_last_error", ctypes.c_char_p, [])
_sig("llama_launch_count", ctypes.c_uint64, [])
_sig("llama_op_rmsnorm", _i, [_vp, _vp, _i, _i, _f, _vp, _i, _vp])
_sig("llama_op_linear", _i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp])
_sig("llama_op_linear_workspace_bytes", _sz, [])
_sig("llama_token_logprobs", _i, [_vp, _vp, _i, _i, _vp, _vp])
_sig("llama_op_linear_noalloc", _i, [_vp, _vp, _i, _i, _i, _vp, _vp])
_sig("llama_timeline_start", _i, [_vp, _vp])
_sig("llama_timeline_stop", _i, [_vp, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_int32),
                                 ctypes.POINTER(ctypes.c_int64), _i, ctypes.POINTER(ctypes.c_int)])
_sig("llama_debug_stall", _i, [_vp, _i, _i, ctypes.c_int64])
_sig("llama_model_bytes_tp", _i, [ctypes.POINTER(ModelArgs), _i, _i, ctypes.POINTER(_sz), ctypes.POINTER(_sz),
                                  ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(ctypes.c_int32)])
_sig("llama_model_create_tp", _i, [ctypes.POINTER(ModelArgs), _i, _i, _vp, _sz, _vp, ctypes.POINTER(_vp)])
_sig("llama_tp_prefill_all", _i, [ctypes.POINTER(_vp), _i, _vp, ctypes.POINTER(ctypes.c_int32), _i, _i, _i, _vp, _i,
                                  _vp])
_sig("llama_tp_decode_step_all", _i, [ctypes.POINTER(_vp), _i, _vp, _vp, _i, ctypes.POINTER(Sampling), _vp, _vp, _vp,
                                      _i, _vp])
_sig("llama_tp_buffers", _i, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp)])
_sig("llama_tp_bind", _i, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp)])
_sig("llama_profile_start", _i, [_vp, _i])
_sig("llama_profile_stop", _i, [_vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int64),
                                ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32), _i,
                                ctypes.POINTER(ctypes.c_int)])


def lib():
    return _lib


def last_error() -> str:
    return (_lib.llama_last_error() or b"").decode()


def launch_count() -> int:
    return int(_lib.llama_launch_count())


def _check(rc: int):
    if rc != LLAMA_OK:
        raise LlamaError(rc, last_error())


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def make_args(dim, n_layers, n_heads, n_kv_heads, vocab_size, multiple_of=256, ffn_dim_multiplier=None,
              norm_eps=1e-5, rope_theta=10000.0, max_seq_len=2048, max_batch_size=32, max_tokens=0,
              dtype="bf16") -> ModelArgs:
    if dtype not in _DTYPES:
        raise ValueError(f"dtype must be one of {sorted(_DTYPES)}")
    return ModelArgs(dim, n_layers, n_heads, n_kv_heads or 0, vocab_size, multiple_of,
                     float(ffn_dim_multiplier or 0.0), norm_eps, rope_theta, max_seq_len,
                     max_batch_size, max_tokens, _DTYPES[dtype])


def args_from_shape(s) -> ModelArgs:
    """ModelArgs from any object with the ModelArgs field names (e.g. workloads.ModelShape)."""
    return make_args(s.dim, s.n_layers, s.n_heads, s.n_kv_heads, s.vocab_size, s.multiple_of,
                     s.ffn_dim_multiplier, s.norm_eps, s.rope_theta, s.max_seq_len, s.max_batch_size,
                     s.max_tokens, s.dtype)


def model_bytes(args: ModelArgs, tp_rank: int = 0, tp_size: int = 1) -> dict:
    """Arena sizes of a model, or of shard tp_rank of a tensor-parallel group
    of tp_size ranks ("hidden" is then the shard's FFN width)."""
    w, kv, ws, tot = _sz(), _sz(), _sz(), _sz()
    h = ctypes.c_int32()
    _check(_lib.llama_model_bytes_tp(ctypes.byref(args), tp_rank, tp_size, ctypes.byref(w), ctypes.byref(kv),
                                     ctypes.byref(ws), ctypes.byref(tot), ctypes.byref(h)))
    return {"weights": w.value, "kv": kv.value, "workspace": ws.value, "total": tot.value, "hidden": h.value}


def _dev(t, dtype: str, numel: int, name: str, device=None):
    """A tensor handed to a kernel: on a CUDA device (`device` if given),
    of torch dtype `dtype` (e.g. "int32"), contiguous, with at least `numel`
    elements.  Raises ValueError instead of passing a pointer a kernel would
    read out of bounds or from host memory."""
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the model on {device}")
    if str(t.dtype) != "torch." + dtype:
        raise ValueError(f"{name} must be {dtype}, not {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs {numel}")


class Model:
    """A model laid out in one torch-allocated device arena."""

    def __init__(self, args: ModelArgs, device="cuda", stream=None, tp_rank: int = 0, tp_size: int = 1):
        import torch
        self.args = args
        self.tp_rank, self.tp_size = tp_rank, tp_size
        self.sizes = model_bytes(args, tp_rank, tp_size)
        self.arena = torch.empty(self.sizes["total"], dtype=torch.uint8, device=device)
        h = _vp()
        _check(_lib.llama_model_create_tp(ctypes.byref(args), tp_rank, tp_size, self.arena.data_ptr(),
                                          self.sizes["total"], _stream(stream), ctypes.byref(h)))
        self.handle = h

    def close(self):
        if self.handle:
            _lib.llama_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_weight(self, layer: int, name: str, tensor, stream=None):
        t = tensor.contiguous()
        _dev(t, self._weight_dtype(name), self._weight_numel(name), name, self.arena.device)
        _check(_lib.llama_set_weight(self.handle, layer, WEIGHT_IDS[name], t.data_ptr(), _stream(stream)))
        return t  # keep alive until the stream passes the copy

    def _weight_dtype(self, name: str) -> str:
        if name in ("norm", "attention_norm", "ffn_norm"):
            return "float32"
        return {LLAMA_BF16: "bfloat16", LLAMA_F16: "float16"}.get(self.args.dtype, "float32")

    def _weight_numel(self, name: str) -> int:
        a = self.args
        t = getattr(self, "tp_size", 1)
        hd = a.dim // a.n_heads
        nh = a.n_heads // t
        nkv = (a.n_kv_heads or a.n_heads) // t
        H = self.sizes["hidden"]
        return {"tok_embeddings": a.vocab_size * a.dim, "output": a.vocab_size // t * a.dim, "norm": a.dim,
                "attention_norm": a.dim, "ffn_norm": a.dim, "wq": nh * hd * a.dim,
                "wk": nkv * hd * a.dim, "wv": nkv * hd * a.dim, "wo": a.dim * nh * hd,
                "w1": H * a.dim, "w2": a.dim * H, "w3": H * a.dim}[name]

    def load(self, weights: dict, stream=None):
        """Upload a weight dict in the workloads layout (torch tensors on the device)."""
        import torch
        keep = [self.set_weight(-1, "tok_embeddings", weights["tok_embeddings"], stream),
                self.set_weight(-1, "norm", weights["norm"], stream),
                self.set_weight(-1, "output", weights["output"], stream)]
        for l, layer in enumerate(weights["layers"]):
            for name, t in layer.items():
                keep.append(self.set_weight(l, name, t, stream))
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
        del keep

    def kv(self, layer: int):
        """(k, v, strides) of one layer: device addresses and element strides of
        the logical [batch_row][position][kv_head][d] index."""
        k, v = _vp(), _vp()
        st = (ctypes.c_int64 * 4)()
        _check(_lib.llama_get_kv(self.handle, layer, ctypes.byref(k), ctypes.byref(v), st))
        return k.value, v.value, tuple(st)

    def kv_tensors(self, layer: int):
        """Torch views of one layer's K and V caches, logical shape
        [max_batch_size, max_seq_len, n_kv_heads, head_dim] (strided)."""
        import torch
        k, v, st = self.kv(layer)
        a = self.args
        nkv = a.n_kv_heads or a.n_heads
        hd = a.dim // a.n_heads
        dt = {LLAMA_BF16: torch.bfloat16, LLAMA_F16: torch.float16}.get(a.dtype, torch.float32)
        esz = 4 if a.dtype == LLAMA_F32 else 2
        n = a.max_batch_size * a.max_seq_len * nkv * hd
        base = self.arena.data_ptr()
        out = []
        for addr in (k, v):
            flat = self.arena[addr - base: addr - base + n * esz].view(dt)
            out.append(torch.as_strided(flat, (a.max_batch_size, a.max_seq_len, nkv, hd), st))
        return out[0], out[1]

    def prefill(self, tokens, lens: Optional[Sequence[int]] = None, start_pos: int = 0, logits=None,
                all_logits: bool = False, stream=None):
        B, T = tokens.shape
        dev = self.arena.device
        _dev(tokens, "int32", B * T, "tokens", dev)
        lens_arr = None
        if lens is not None:
            if len(lens) != B:
                raise ValueError(f"lens has {len(lens)} entries for {B} rows")
            lens_arr = (ctypes.c_int32 * B)(*[int(v) for v in lens])
        if logits is not None:
            rows = (sum(int(v) for v in lens) if lens is not None else B * T) if all_logits else B
            _dev(logits, "float32", rows * self.args.vocab_size, "logits", dev)
        _check(_lib.llama_prefill(self.handle, tokens.data_ptr(), lens_arr, B, T, start_pos, _ptr(logits),
                                  1 if all_logits else 0, _stream(stream)))
        return logits

    def decode_step(self, tokens, pos, temperature: Optional[float] = None, top_p: float = 0.9,
                    uniforms=None, next_tokens=None, logits=None, advance: bool = False, stream=None):
        B = tokens.shape[0]
        dev = self.arena.device
        _dev(tokens, "int32", B, "tokens", dev)
        _dev(pos, "int32", B, "pos", dev)
        if uniforms is not None:
            _dev(uniforms, "float32", B, "uniforms", dev)
        if next_tokens is not None:
            _dev(next_tokens, "int32", B, "next_tokens", dev)
        if logits is not None:
            _dev(logits, "float32", B * self.args.vocab_size, "logits", dev)
        samp = None
        if temperature is not None:
            samp = Sampling(float(temperature), float(top_p))
        _check(_lib.llama_decode_step(self.handle, tokens.data_ptr(), pos.data_ptr(), B,
                                      ctypes.byref(samp) if samp is not None else None, _ptr(uniforms),
                                      _ptr(next_tokens), _ptr(logits),
                                      LLAMA_DECODE_ADVANCE if advance else 0, _stream(stream)))
        return next_tokens

    def profile_start(self, capacity: int):
        _check(_lib.llama_profile_start(self.handle, capacity))

    def profile_stop(self, max_records: int):
        """[(ms, algorithmic bytes, flops, token rows)] of the projection launches
        timed since profile_start."""
        ms = (ctypes.c_float * max_records)()
        by = (ctypes.c_int64 * max_records)()
        fl = (ctypes.c_int64 * max_records)()
        rw = (ctypes.c_int32 * max_records)()
        n = ctypes.c_int()
        _check(_lib.llama_profile_stop(self.handle, ms, by, fl, rw, max_records, ctypes.byref(n)))
        return [(ms[i], by[i], fl[i], rw[i]) for i in range(n.value)]

    def timeline_start(self, stream=None):
        _check(_lib.llama_timeline_start(self.handle, _stream(stream)))

    def timeline_stop(self, max_records: int = 8192):
        """[(end_ns, kind name, algorithmic bytes)] of the decode launches that
        took a timeline slot since timeline_start, in launch order."""
        en = (ctypes.c_uint64 * max_records)()
        kd = (ctypes.c_int32 * max_records)()
        by = (ctypes.c_int64 * max_records)()
        n = ctypes.c_int()
        _check(_lib.llama_timeline_stop(self.handle, en, kd, by, max_records, ctypes.byref(n)))
        return [(int(en[i]), TIMELINE_KINDS.get(kd[i], str(kd[i])), int(by[i])) for i in range(n.value)]

    def tp_buffers(self):
        """(partial sums phase 0, phase 1, flag words, logits) device addresses of a shard."""
        p0, p1, fl, lg = _vp(), _vp(), _vp(), _vp()
        _check(_lib.llama_tp_buffers(self.handle, ctypes.byref(p0), ctypes.byref(p1), ctypes.byref(fl),
                                     ctypes.byref(lg)))
        return p0.value, p1.value, fl.value, lg.value

    def tp_bind(self, part0, part1, flags, logits):
        """Bind every rank's buffers (lists indexed by rank, addresses mapped into this process)."""
        n = self.tp_size
        arr = [(_vp * n)(*[int(v) for v in t]) for t in (part0, part1, flags, logits)]
        _check(_lib.llama_tp_bind(self.handle, *arr))

    def debug_stall(self, which: str, unit: int = 0, wait_limit_ns: int = 1_000_000):
        """Arm a one-shot stalled producer in the next `which` launch
        ("projection", "attention" or "none"): tests of the device timeout."""
        code = {"none": LLAMA_STALL_NONE, "projection": LLAMA_STALL_PROJECTION,
                "attention": LLAMA_STALL_ATTENTION}[which]
        _check(_lib.llama_debug_stall(self.handle, code, int(unit), int(wait_limit_ns)))

    def status(self) -> int:
        s = ctypes.c_int()
        _check(_lib.llama_model_status(self.handle, ctypes.byref(s)))
        return s.value


def tp_bind_distributed(model: "Model", group=None, ipc=None):
    """Ranks of a tensor-parallel group on separate GPUs (one process per GPU,
    torch.distributed initialised, one rank per shard): shares this shard's
    buffers with the other ranks through a CUDA IPC handle of the allocation
    that holds its arena, maps theirs, and binds every rank's buffers
    (llama_tp_bind).  Call it on every rank, after creating the shard.
    `ipc` replaces the CUDA IPC calls (tests of the exchange on CPU): an
    object with base_of(ptr) -> (allocation base, handle bytes) and
    open(handle bytes) -> mapped base."""
    import torch.distributed as dist
    if ipc is None:
        ipc = _CudaIpc()
    bufs = model.tp_buffers()
    base, handle = ipc.base_of(bufs[0])
    mine = {"rank": model.tp_rank, "handle": handle, "offsets": [b - base for b in bufs]}
    world = dist.get_world_size(group)
    if world != model.tp_size:
        raise ValueError(f"process group of {world} ranks for a shard of a {model.tp_size}-rank group")
    everyone = [None] * world
    dist.all_gather_object(everyone, mine, group=group)
    tables = [[0] * model.tp_size for _ in range(4)]
    model._tp_mapped = []
    for entry in everyone:
        r = entry["rank"]
        mapped = base if r == model.tp_rank else ipc.open(entry["handle"])
        if r != model.tp_rank:
            model._tp_mapped.append(mapped)
        for i in range(4):
            tables[i][r] = mapped + entry["offsets"][i]
    model.tp_bind(*tables)
    return tables


class _CudaIpc:
    """CUDA IPC through cuda-python: the allocation base of a device pointer,
    its IPC handle, and the mapping of a peer's handle."""

    def __init__(self):
        from cuda.bindings import driver, runtime
        self._drv, self._rt = driver, runtime

    def base_of(self, ptr: int):
        err, base, _size = self._drv.cuMemGetAddressRange(ptr)
        if int(err) != 0:
            raise RuntimeError(f"cuMemGetAddressRange failed ({err})")
        err, h = self._rt.cudaIpcGetMemHandle(int(base))
        if int(err) != 0:
            raise RuntimeError(f"cudaIpcGetMemHandle failed ({err})")
        return int(base), bytes(h.reserved)

    def open(self, handle: bytes) -> int:
        h = self._rt.cudaIpcMemHandle_t()
        h.reserved = handle
        err, ptr = self._rt.cudaIpcOpenMemHandle(h, self._rt.cudaIpcMemLazyEnablePeerAccess)
        if int(err) != 0:
            raise RuntimeError(f"cudaIpcOpenMemHandle failed ({err})")
        return int(ptr)


class TPGroup:
    """Every rank of a tensor-parallel group on one GPU (llama_tp_*_all):
    shards[r] holds rank r's slices of the weights (decoder_only_transformer_llama_b200.tp)."""

    def __init__(self, args: ModelArgs, tp_size: int, device="cuda"):
        self.args = args
        self.tp_size = tp_size
        self.shards = [Model(args, device=device, tp_rank=r, tp_size=tp_size) for r in range(tp_size)]
        self.device = self.shards[0].arena.device
        self._h = (_vp * tp_size)(*[s.handle for s in self.shards])

    def load(self, weights: dict, shape):
        """Upload a whole (unsharded) weight dict, cut per rank by tp.shard_weights."""
        from . import tp as _tp
        for r, s in enumerate(self.shards):
            part = _tp.shard_weights(weights, _tp.plan_for(shape, r, self.tp_size))
            s.load({"tok_embeddings": part["tok_embeddings"].contiguous(), "norm": part["norm"].contiguous(),
                    "output": part["output"].contiguous(),
                    "layers": [{k: v.contiguous() for k, v in layer.items()} for layer in part["layers"]]})

    def prefill(self, tokens, lens=None, start_pos: int = 0, logits=None, all_logits: bool = False, stream=None):
        B, T = tokens.shape
        _dev(tokens, "int32", B * T, "tokens", self.device)
        lens_arr = (ctypes.c_int32 * B)(*[int(v) for v in lens]) if lens is not None else None
        if logits is not None:
            rows = (sum(int(v) for v in lens) if lens is not None else B * T) if all_logits else B
            _dev(logits, "float32", rows * self.args.vocab_size, "logits", self.device)
        _check(_lib.llama_tp_prefill_all(self._h, self.tp_size, tokens.data_ptr(), lens_arr, B, T, start_pos,
                                         _ptr(logits), 1 if all_logits else 0, _stream(stream)))
        return logits

    def decode_step(self, tokens, pos, temperature: Optional[float] = None, top_p: float = 0.9, uniforms=None,
                    next_tokens=None, logits=None, advance: bool = False, stream=None):
        B = tokens.shape[0]
        _dev(tokens, "int32", B, "tokens", self.device)
        _dev(pos, "int32", B, "pos", self.device)
        if uniforms is not None:
            _dev(uniforms, "float32", B, "uniforms", self.device)
        if next_tokens is not None:
            _dev(next_tokens, "int32", B, "next_tokens", self.device)
        if logits is not None:
            _dev(logits, "float32", B * self.args.vocab_size, "logits", self.device)
        samp = Sampling(float(temperature), float(top_p)) if temperature is not None else None
        _check(_lib.llama_tp_decode_step_all(self._h, self.tp_size, tokens.data_ptr(), pos.data_ptr(), B,
                                             ctypes.byref(samp) if samp is not None else None, _ptr(uniforms),
                                             _ptr(next_tokens), _ptr(logits),
                                             LLAMA_DECODE_ADVANCE if advance else 0, _stream(stream)))
        return next_tokens

    def status(self) -> int:
        codes = [s.status() for s in self.shards]
        return next((c for c in codes if c), 0)

    def close(self):
        for s in self.shards:
            s.close()


def sample(logits, temperature: float, top_p: float, uniforms, out, stream=None):
    B, V = logits.shape
    _dev(logits, "float32", B * V, "logits")
    _dev(out, "int32", B, "out", logits.device)
    if uniforms is not None:
        _dev(uniforms, "float32", B, "uniforms", logits.device)
    _check(_lib.llama_sample(logits.data_ptr(), B, V, float(temperature), float(top_p), _ptr(uniforms),
                             out.data_ptr(), _stream(stream)))
    return out


def token_logprobs(logits, tokens, out, stream=None):
    """out[i] = log_softmax(logits[i])[tokens[i]] (fp32 logits [N, V], int32 tokens [N])."""
    N, V = logits.shape
    _dev(logits, "float32", N * V, "logits")
    _dev(tokens, "int32", N, "tokens", logits.device)
    _dev(out, "float32", N, "out", logits.device)
    _check(_lib.llama_token_logprobs(logits.data_ptr(), tokens.data_ptr(), N, V, out.data_ptr(), _stream(stream)))
    return out


_TORCH_DTYPES = {"torch.float32": LLAMA_F32, "torch.bfloat16": LLAMA_BF16, "torch.float16": LLAMA_F16}


def _dtype_code(t, what: str) -> int:
    code = _TORCH_DTYPES.get(str(t.dtype))
    if code is None:
        raise ValueError(f"{what} must be float32, bfloat16 or float16, not {t.dtype}")
    return code


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _check_linear_operands(A, W, out):
    M, K = A.shape
    _need(W.dim() == 2 and W.dtype == A.dtype and W.shape[1] == K, "W must be [N, K] of A's dtype")
    _need(str(out.dtype) == "torch.float32" and tuple(out.shape) == (M, W.shape[0]), "out must be float32 [M, N]")
    _need(A.is_contiguous() and W.is_contiguous() and out.is_contiguous(), "tensors must be contiguous")


def op_rmsnorm(x, w, eps: float, out, stream=None):
    M, dim = x.shape
    _need(str(x.dtype) == "torch.float32" and str(w.dtype) == "torch.float32", "x and w must be float32")
    _need(tuple(out.shape) == (M, dim) and w.numel() == dim, "out must be [M, dim] and w [dim]")
    _need(x.is_contiguous() and w.is_contiguous() and out.is_contiguous(), "tensors must be contiguous")
    dt = _dtype_code(out, "out")
    _check(_lib.llama_op_rmsnorm(x.data_ptr(), w.data_ptr(), M, dim, float(eps), out.data_ptr(), dt,
                                 _stream(stream)))
    return out


_op_ws = {}


def op_linear_workspace(device):
    """A zero-filled scratch buffer for op_linear, cached per device."""
    import torch
    key = str(device)
    if key not in _op_ws:
        _op_ws[key] = torch.zeros(int(_lib.llama_op_linear_workspace_bytes()), dtype=torch.uint8, device=device)
    return _op_ws[key]


def op_linear_noalloc(A, W, out, stream=None):
    """bf16 projection out = A W^T (A: <= 16 rows) without any scratch from
    the caller: for callers that cannot allocate device memory."""
    M, K = A.shape
    N = W.shape[0]
    _check_linear_operands(A, W, out)
    _need(_dtype_code(A, "A") == LLAMA_BF16, "op_linear_noalloc takes bfloat16 operands")
    _check(_lib.llama_op_linear_noalloc(A.data_ptr(), W.data_ptr(), M, N, K, out.data_ptr(), _stream(stream)))
    return out


def op_linear_whole_tiles(A, W, out, stream=None):
    """16-bit projection with M > 64 and no workspace: every tile runs whole
    (no stream-K split of the last wave)."""
    M, K = A.shape
    N = W.shape[0]
    if M <= 64:
        raise ValueError("op_linear_whole_tiles takes M > 64 token rows")
    _check_linear_operands(A, W, out)
    dt = _dtype_code(A, "A")
    _need(dt != LLAMA_F32, "op_linear_whole_tiles takes bfloat16 or float16 operands")
    _check(_lib.llama_op_linear(A.data_ptr(), W.data_ptr(), M, N, K, dt, out.data_ptr(), None, 0,
                                _stream(stream)))
    return out


def op_linear(A, W, out, stream=None, workspace=None):
    """out = A W^T: A [M, K] and W [N, K] of one type (float32, bfloat16 or
    float16), out float32 [M, N]."""
    M, K = A.shape
    N = W.shape[0]
    dt = _dtype_code(A, "A")
    _check_linear_operands(A, W, out)
    ws = workspace if workspace is not None else (op_linear_workspace(A.device) if dt != LLAMA_F32 else None)
    _check(_lib.llama_op_linear(A.data_ptr(), W.data_ptr(), M, N, K, dt, out.data_ptr(), _ptr(ws),
                                0 if ws is None else ws.numel(), _stream(stream)))
    return out
