"""The tensor-parallel sharding plan on CPU: two and four gloo ranks stand in for
GPUs.  Each rank holds the weights decoder_only_transformer_llama_b200.tp
gives it, runs its share of every layer with the oracle's own steps (RMSNorm,
RoPE, attention over its query and KV heads, SwiGLU over its hidden slice),
and the ranks add the two row-parallel partial sums of each layer (wo and w2)
with an all-reduce and gather the vocabulary slices of the logits, as the
reference's model-parallel layers do (Admin Guide §1.3 NOTE, §4.2; source
tour, "One model.py").  The result must equal the unsharded oracle forward
pass to fp64 rounding, prefill and a decode step both, for multi-head and
grouped-query attention."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import llama_oracle as O
from workloads import ModelShape, make_tokens, make_weights, to_numpy_f64_weights

GQA = ModelShape(dim=256, n_layers=2, n_heads=8, n_kv_heads=4, vocab_size=512, max_seq_len=32,
                 max_batch_size=1, dtype="f32", hidden=768)
MHA = GQA.replace(n_kv_heads=8)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _all_reduce(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a))
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.numpy()


def _tp_forward(args, plan, w, tokens, start_pos, cache):
    """One rank's share of Transformer.forward over `tokens`, with the two
    all-reduces per layer and the gathered logits."""
    from decoder_only_transformer_llama_b200 import tp as TP  # noqa: F401  (plan already built)
    hd = args.head_dim
    nh_l = plan.heads[1] - plan.heads[0]
    nkv_l = plan.kv_heads[1] - plan.kv_heads[0]
    n_rep = args.n_rep
    x = np.asarray(w["tok_embeddings"][np.asarray(tokens)], dtype=np.float64)
    T = x.shape[0]
    pos = start_pos + np.arange(T)
    for l, lw in enumerate(w["layers"]):
        y = O.rms_norm(x, lw["attention_norm"], args.norm_eps)
        q = O.apply_rope((y @ np.asarray(lw["wq"], dtype=np.float64).T).reshape(T, nh_l, hd), pos, args.rope_theta)
        k = O.apply_rope((y @ np.asarray(lw["wk"], dtype=np.float64).T).reshape(T, nkv_l, hd), pos, args.rope_theta)
        v = (y @ np.asarray(lw["wv"], dtype=np.float64).T).reshape(T, nkv_l, hd)
        cache.k[l][start_pos:start_pos + T] = k
        cache.v[l][start_pos:start_pos + T] = v
        o = O.attention(q, cache.k[l][:start_pos + T], cache.v[l][:start_pos + T], start_pos, n_rep)
        x = x + _all_reduce(o.reshape(T, nh_l * hd) @ np.asarray(lw["wo"], dtype=np.float64).T)
        f = O.rms_norm(x, lw["ffn_norm"], args.norm_eps)
        x = x + _all_reduce(O.feed_forward(f, lw["w1"], lw["w2"], lw["w3"]))
    h = O.rms_norm(x, w["norm"], args.norm_eps)
    local = torch.from_numpy(np.ascontiguousarray(h @ np.asarray(w["output"], dtype=np.float64).T))
    parts = [torch.empty_like(local) for _ in range(dist.get_world_size())]
    dist.all_gather(parts, local)
    return torch.cat(parts, dim=1).numpy()


def _rank(rank, world, port, shape, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        from decoder_only_transformer_llama_b200 import tp as TP
        args = O.Args(dim=shape.dim, n_layers=shape.n_layers, n_heads=shape.n_heads, n_kv_heads=shape.n_kv_heads,
                      vocab_size=shape.vocab_size, max_seq_len=shape.max_seq_len)
        full = to_numpy_f64_weights(make_weights(shape, 81))
        plan = TP.plan_for(shape, rank, world)
        mine = TP.shard_weights(full, plan)
        toks = make_tokens(shape.vocab_size, (1, 13), 82)[0].tolist()
        cache = O.KVCache(args.n_layers, args.max_seq_len, plan.kv_heads[1] - plan.kv_heads[0], args.head_dim)
        got_prefill = _tp_forward(args, plan, mine, toks[:12], 0, cache)
        got_step = _tp_forward(args, plan, mine, toks[12:], 12, cache)
        dist.barrier()
        dist.destroy_process_group()
        if rank == 0:
            want = O.forward(args, full, toks, 0, O.new_cache(args))
            err = max(float(np.max(np.abs(got_prefill - want[:12]))), float(np.max(np.abs(got_step - want[12:]))))
            q.put((rank, err, None))
        else:
            q.put((rank, 0.0, None))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, None, repr(e)))


@pytest.mark.parametrize("shape,world", [(GQA, 2), (GQA, 4), (MHA, 2)])
def test_sharded_forward_equals_the_oracle(shape, world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, shape, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, err, exc in res:
        assert exc is None, (rank, exc)
        if rank == 0:
            assert err <= 1e-10, err


def test_plan_keeps_query_groups_with_their_kv_head():
    """Every query head a rank holds reads a KV head the same rank holds
    (h // n_rep), and the ranks' slices tile every dimension exactly once."""
    from decoder_only_transformer_llama_b200 import tp as TP
    for nh, nkv, tp in ((64, 8, 8), (64, 8, 2), (40, 40, 4), (32, 32, 8)):
        n_rep = nh // nkv
        plans = [TP.shard_plan(nh, nkv, 128, 28672, 32000, r, tp) for r in range(tp)]
        for p in plans:
            for h in range(*p.heads):
                assert p.kv_heads[0] <= h // n_rep < p.kv_heads[1]
        for attr, n in (("heads", nh), ("kv_heads", nkv), ("hidden", 28672), ("vocab", 32000)):
            covered = sorted(i for p in plans for i in range(*getattr(p, attr)))
            assert covered == list(range(n))
    with pytest.raises(ValueError):
        TP.shard_plan(64, 8, 128, 28672, 32000, 0, 16)   # 8 KV heads cannot split 16 ways


class _FakeShard:
    """Stands in for a shard on its own GPU: fixed buffer addresses inside a
    per-rank arena, and a record of what was bound."""

    def __init__(self, rank, tp):
        self.tp_rank, self.tp_size = rank, tp
        self.base = 0x10000000 * (rank + 1)
        self.bound = None

    def tp_buffers(self):
        b = self.base
        return b + 0x100 + self.tp_rank, b + 0x2000, b + 0x3000 + 8 * self.tp_rank, b + 0x4000

    def tp_bind(self, *tables):
        self.bound = [list(t) for t in tables]


class _FakeIpc:
    def __init__(self, shard):
        self.shard = shard

    def base_of(self, ptr):
        return self.shard.base, b"handle-of-rank-%d" % self.shard.tp_rank

    def open(self, handle):
        r = int(handle.decode().rsplit("-", 1)[1])
        return 0x90000000 + 0x1000000 * r      # where this process maps rank r's arena


def _bind_rank(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import decoder_only_transformer_llama_b200 as llb
        shard = _FakeShard(rank, world)
        llb.tp_bind_distributed(shard, ipc=_FakeIpc(shard))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, shard.bound, None))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, None, repr(e)))


def test_distributed_binding_maps_every_ranks_buffers():
    """Ranks on separate GPUs exchange their buffers' offsets and IPC handles;
    each binds, for every rank, that rank's mapped arena plus its offsets (its
    own arena for itself)."""
    world = 3
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bind_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, bound, exc in res:
        assert exc is None, (rank, exc)
        for r in range(world):
            owner = _FakeShard(r, world)
            mapped = owner.base if r == rank else 0x90000000 + 0x1000000 * r
            want = [mapped + (b - owner.base) for b in owner.tp_buffers()]
            assert [bound[i][r] for i in range(4)] == want, (rank, r)
