"""Benchmark of the Llama-2 7B-shaped forward pass on B200: prefill + greedy decode.

One step = the whole hot path over one batch: prefill of 4 x 512 random token
ids (all 32 layers, final norm, vocabulary projection, greedy pick of the
first token), then 256 greedy decode steps (contexts 513 .. 768), all through
the C ABI of libllama_b200.so.  Weights are random (seeded), bf16, with fp32
norm weights; data is synthetic.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is decode tokens/s of the whole job;
prefill tokens/s and both rooflines are extra keys.  With N > 1 (torchrun)
every rank runs an independent replica of the workload (batch rows never
interact, so there is nothing to exchange) and the job time is the max over
ranks.  `--impl reference` times the CPU oracle on a bounded sample of the
same workload on the host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import L7B, WORKLOADS, make_tokens, make_weights, token_seed, weight_seed  # noqa: E402

WL = WORKLOADS["7b"]
METRIC = "decode tok/s (% HBM peak) + prefill tok/s (% TC peak), 7B shape, 1 B200"
UNIT = "tok/s"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, path: str):
        self.index, self.path, self.proc = index, path, None

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- roofline bookkeeping

def bench_config(world):
    """The headline workload, as both arms print it (the reference arm times a
    bounded sample of it, described in its cpu_baseline.sample)."""
    return {"workload": "7b: Llama-2-7B shape, 32 layers, dim 4096, 32 heads (MHA), hidden 11008, "
                        "vocab 32000, max_seq_len 4096; prefill 4x512 then 256 greedy decode steps",
            "global_batch": WL["batch"] * world, "seq_len": WL["prompt_len"], "decode_steps": WL["decode_steps"],
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2: each decode step streams 13.5 GB of weights (L2 126 MB)"}


def max_over_ranks(vals, world):
    """Element-wise maximum of the float64 tensor `vals` over all ranks, in
    place: a replicated job ends when its slowest rank does."""
    if world > 1:
        torch.distributed.all_reduce(vals, op=torch.distributed.ReduceOp.MAX)
    return vals


def whole_job_rate(units_per_rank, world, ms):
    """Units that all `world` ranks processed, per second of the slowest rank's
    device time `ms` (every rank runs the same fixed work: weak scaling)."""
    return world * units_per_rank / (ms / 1e3)


def _traffic(kernel):
    """DRAM bytes per launch of `kernel` in this workload from the committed
    ncu record (profiles/dram_traffic_7b.json), or None when the kernel's
    sources no longer match the ones the counters were taken on."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic_7b.json")) as f:
            rec = json.load(f)[kernel]
        m = hashlib.sha256()
        for name in rec["source_files"]:
            with open(os.path.join(ROOT, "decoder_only_transformer_llama_b200", "csrc", name), "rb") as f:
                m.update(f.read())
        if m.hexdigest() != rec["source_sha256"]:
            return None
        return int(rec["bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def decode_step_bytes(s, B, ctx, logits=True):
    """Algorithmic bytes of one decode step of B rows at context ctx: every
    weight matrix once (bf16), the norm weights (fp32), B embedding rows, the
    K and V cache read over ctx positions and written at one, and the fp32
    logits when they are materialised (a greedy step picks its token inside
    the vocabulary projection and stores none)."""
    hd, nkv, L = s.head_dim, s.n_kv_heads, s.n_layers
    mats = L * (s.dim * (s.n_heads + 2 * nkv) * hd + s.dim * s.n_heads * hd + 3 * s.dim * s.hidden)
    mats += s.vocab_size * s.dim
    return (2 * mats + 4 * s.dim * (2 * L + 1) + 2 * B * s.dim
            + L * 2 * nkv * hd * 2 * ctx * B + L * 2 * nkv * hd * 2 * B + (4 * B * s.vocab_size if logits else 0))


# ----------------------------------------------------------------------------- our arm

def capture_graph(fn, dev, stream):
    """One call of `fn` (a decode step) captured as a CUDA graph on a side stream."""
    s_cap = torch.cuda.Stream(device=dev)
    s_cap.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s_cap):
        with torch.cuda.graph(g, stream=s_cap):
            fn()
    stream.wait_stream(s_cap)
    torch.cuda.synchronize()
    return g


def timeline_breakdown(recs, n_step):
    """Per-kind exclusive device time of one graph-replayed decode step from
    the library's timeline (see llama_timeline_start): the graph holds two
    decode steps of n_step launches each; launch i of the second step ran,
    exclusive of its predecessor, for end[i] - end[i-1], and these times sum
    to the second step's duration.  Returns (step ns, {kind: ns},
    {kind: algorithmic bytes})."""
    assert len(recs) == 2 * n_step, (len(recs), n_step)
    ends = [r[0] for r in recs]
    t_kind, b_kind = {}, {}
    for i in range(n_step, 2 * n_step):
        _, kind, byts = recs[i]
        t_kind[kind] = t_kind.get(kind, 0) + (ends[i] - ends[i - 1])
        b_kind[kind] = b_kind.get(kind, 0) + byts
    return ends[-1] - ends[n_step - 1], t_kind, b_kind


def run_ours(a, rank, world, local_rank):
    import decoder_only_transformer_llama_b200 as llb
    import tempfile

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm, tc_burst, tc_sust, peak_src = _peaks()
    s = L7B
    B, T, steps_dec = WL["batch"], WL["prompt_len"], WL["decode_steps"]
    w = make_weights(s, weight_seed(WL["index"]), device=dev)
    model = llb.Model(llb.args_from_shape(s), device=dev)
    model.load(w)
    del w
    torch.cuda.empty_cache()

    stream = torch.cuda.current_stream()
    prompt = make_tokens(s.vocab_size, (B, T), token_seed(WL["index"])).to(dev)
    prompt_host = prompt.cpu().pin_memory()
    prompt_dev = torch.empty_like(prompt)
    logits = torch.empty(B, s.vocab_size, device=dev)
    tok = torch.empty(B, dtype=torch.int32, device=dev)
    pos = torch.empty(B, dtype=torch.int32, device=dev)
    pos_init = torch.full((B,), T, dtype=torch.int32, device=dev)
    tok_host = torch.empty(B, dtype=torch.int32).pin_memory()

    def decode_direct():
        model.decode_step(tok, pos, temperature=0.0, next_tokens=tok, advance=True)

    graph = None

    def decode_once():
        if graph is not None:
            graph.replay()
        else:
            decode_direct()

    def start_request():
        model.prefill(prompt, logits=logits)
        llb.sample(logits, 0.0, 0.9, None, tok)
        pos.copy_(pos_init)

    def one_step():
        start_request()
        for _ in range(steps_dec):
            decode_once()

    for _ in range(a.warmup):
        one_step()
    torch.cuda.synchronize()
    assert model.status() == 0
    if not a.no_graph:
        # one decode step (tokens and positions advance on the device) as a CUDA graph
        graph = capture_graph(decode_direct, dev, stream)
        for _ in range(2):
            one_step()
        torch.cuda.synchronize()
        assert model.status() == 0

    # launches per bench step (exact count of this library's kernels, counted
    # on a step launched without the graph)
    c0 = llb.launch_count()
    start_request()
    for _ in range(steps_dec):
        decode_direct()
    torch.cuda.synchronize()
    launches_per_step = llb.launch_count() - c0

    # ---------------- timed region: prefill + first token + 256 decode steps per bench step
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(a.steps)]
    clocks = ClockSampler(local_rank, os.path.join(tempfile.gettempdir(), f"llama_b200_clocks_rank{rank}.csv"))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(a.steps):
        evs[i][0].record(stream)
        start_request()
        evs[i][1].record(stream)
        for _ in range(steps_dec):
            decode_once()
        evs[i][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    launches = launches_per_step * a.steps
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    prefill_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    decode_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    assert model.status() == 0

    # ---------------- batch 1: one 512-token prompt of the same model, 256 graph-replayed decode steps
    tok1 = torch.empty(1, dtype=torch.int32, device=dev)
    pos1 = torch.empty(1, dtype=torch.int32, device=dev)
    logits1 = torch.empty(1, s.vocab_size, device=dev)
    prompt1 = prompt[:1].contiguous()

    def start_b1():
        model.prefill(prompt1, logits=logits1)
        llb.sample(logits1, 0.0, 0.9, None, tok1)
        pos1.fill_(T)

    def decode_b1():
        model.decode_step(tok1, pos1, temperature=0.0, next_tokens=tok1, advance=True)

    start_b1()
    for _ in range(3):
        decode_b1()
    torch.cuda.synchronize()
    g1 = capture_graph(decode_b1, dev, stream) if not a.no_graph else None
    step_b1 = g1.replay if g1 is not None else decode_b1
    b1_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    b1_ms = 0.0
    clocks_b1 = ClockSampler(local_rank, os.path.join(tempfile.gettempdir(), f"llama_b200_clocks_b1_rank{rank}.csv"))
    torch.cuda.synchronize()
    clocks_b1.start()
    for _ in range(a.steps):
        start_b1()
        b1_ev[0].record(stream)
        for _ in range(steps_dec):
            step_b1()
        b1_ev[1].record(stream)
        torch.cuda.synchronize()
        b1_ms += b1_ev[0].elapsed_time(b1_ev[1])
    clk_b1 = clocks_b1.stop()
    assert model.status() == 0
    del g1

    # ---------------- in-graph timeline of the batch-4 decode step (outside the timed region):
    # a graph of two decode steps captured while the timeline records; every
    # replay re-stamps its slots, the last replay's stamps are read back
    start_request()
    torch.cuda.synchronize()

    def two_steps():
        decode_direct()
        decode_direct()

    model.timeline_start()
    if a.no_graph:
        two_steps()
    else:
        g_tl = capture_graph(two_steps, dev, stream)
        model.timeline_stop()          # slots are baked into the graph; stop handing out more
        for _ in range(8):
            g_tl.replay()
        del g_tl
    tl_recs = model.timeline_stop()    # the last execution's stamps
    n_step = len(tl_recs) // 2
    tl_step_ns, tl_kind_ns, tl_kind_bytes = timeline_breakdown(tl_recs, n_step)
    assert model.status() == 0

    # ---------------- SM clocks while prefills run back to back (outside the timed region): the
    # tensor-core-bound prefill runs under the 1 kW power cap, unlike the HBM-bound decode
    pre_clocks = ClockSampler(local_rank, os.path.join(tempfile.gettempdir(), f"llama_b200_clocks_pre_rank{rank}.csv"))
    pre_clocks.start()
    t_pc = time.time()
    while time.time() - t_pc < 0.8:
        start_request()
        torch.cuda.synchronize()
    pre_clk = pre_clocks.stop()

    # ---------------- serialised per-launch timing (outside the timed region): events around every
    # projection of one prefill and of 16 decode steps launched directly (programmatic dependent
    # launch off while timed, so each launch runs alone)
    PROF_DECODE = 16
    prof_cap = (5 * s.n_layers + 1) * (1 + PROF_DECODE)
    model.profile_start(prof_cap)
    start_request()
    for _ in range(PROF_DECODE):
        decode_direct()
    torch.cuda.synchronize()
    recs = model.profile_stop(prof_cap)
    assert model.status() == 0

    # ---------------- second run: top-p 0.9 at temperature 0.6, seeded uniforms
    # (one uniform per row per step; launched step by step, each with its row)
    from workloads import make_uniforms, uniform_seed
    uni = make_uniforms((steps_dec, B), uniform_seed(WL["index"])).to(dev)
    tp_ev0 = torch.cuda.Event(enable_timing=True)
    tp_ev1 = torch.cuda.Event(enable_timing=True)
    model.prefill(prompt, logits=logits)
    llb.sample(logits, WL["temperature"], WL["top_p"], uni[0], tok)
    pos.copy_(pos_init)
    torch.cuda.synchronize()
    tp_ev0.record(stream)
    for i in range(steps_dec):
        model.decode_step(tok, pos, temperature=WL["temperature"], top_p=WL["top_p"], uniforms=uni[i],
                          next_tokens=tok, advance=True)
    tp_ev1.record(stream)
    torch.cuda.synchronize()
    assert model.status() == 0
    top_p_tps = B * steps_dec / (tp_ev0.elapsed_time(tp_ev1) / 1e3)

    # ---------------- end to end through host buffers: one request per bench step, from the
    # prompt's copy out of pinned host memory to the host's read of the last generated token
    e2e_ev0 = torch.cuda.Event(enable_timing=True)
    e2e_ev1 = torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(a.steps):
        e2e_ev0.record(stream)
        prompt_dev.copy_(prompt_host, non_blocking=True)
        model.prefill(prompt_dev, logits=logits)
        llb.sample(logits, 0.0, 0.9, None, tok)
        tok_host.copy_(tok, non_blocking=True)
        pos.copy_(pos_init)
        stream.synchronize()
        for _ in range(steps_dec):
            model.decode_step(tok, pos, temperature=0.0, next_tokens=tok, advance=True)
            tok_host.copy_(tok, non_blocking=True)
            stream.synchronize()     # the host reads every generated token, like a serving loop
        e2e_ev1.record(stream)
        torch.cuda.synchronize()
        e2e_ms += e2e_ev0.elapsed_time(e2e_ev1)

    # ---------------- max over ranks
    vals = torch.tensor([total_ms, prefill_ms, decode_ms, e2e_ms, b1_ms], device=dev, dtype=torch.float64)
    total_ms, prefill_ms, decode_ms, e2e_ms, b1_ms = max_over_ranks(vals, world).tolist()

    value = whole_job_rate(a.steps * B * steps_dec, world, decode_ms)
    prefill_tps = whole_job_rate(a.steps * B * T, world, prefill_ms)
    e2e_value = whole_job_rate(a.steps * B * steps_dec, world, e2e_ms)
    b1_tps = whole_job_rate(a.steps * steps_dec, world, b1_ms)

    # serialised per-launch figures
    dec = [r for r in recs if r[0] > 0 and 0 < r[3] <= 64]
    pre = [r for r in recs if r[0] > 0 and r[3] > 64]
    dec_gbs_serial = sum(r[1] for r in dec) / (sum(r[0] for r in dec) / 1e3) / 1e9 if dec else 0.0
    pre_flops = sum(r[2] for r in pre)
    pre_ms_k = sum(r[0] for r in pre)
    pre_tfs = pre_flops / (pre_ms_k / 1e3) / 1e12 if pre_ms_k else 0.0
    # per projection kind (the layer's launch order: wq/wk/wv, wo, w1/w3, w2): mean
    # microseconds per launch and TFLOP/s
    pre_kinds = {}
    for i, r in enumerate(pre[:4 * s.n_layers]):
        k = ("wq/wk/wv", "wo", "w1/w3", "w2")[i % 4]
        acc = pre_kinds.setdefault(k, [0.0, 0, 0])
        acc[0] += r[0]
        acc[1] += r[2]
        acc[2] += 1
    pre_kind_line = {k: {"us_per_launch": round(v[0] * 1e3 / v[2], 1),
                         "TFLOP_s": round(v[1] / (v[0] / 1e3) / 1e12, 1)} for k, v in pre_kinds.items() if v[0] > 0}

    # in-graph: the projections' algorithmic bytes over their exclusive time in the replayed step
    proj_ns = tl_kind_ns.get("projection", 0)
    proj_bytes = tl_kind_bytes.get("projection", 0)
    n_proj = sum(1 for r in tl_recs[n_step:] if r[1] == "projection")
    dec_gbs = proj_bytes / proj_ns if proj_ns else 0.0    # bytes per ns = GB/s

    step_bytes = sum(decode_step_bytes(s, B, T + 1 + i, logits=False) for i in range(steps_dec))
    decode_gbs_path = step_bytes * world * a.steps / (decode_ms / 1e3) / 1e9
    b1_bytes = sum(decode_step_bytes(s, 1, T + 1 + i, logits=False) for i in range(steps_dec))
    b1_gbs = b1_bytes * world * a.steps / (b1_ms / 1e3) / 1e9

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": round(total_ms / a.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded random token ids, random-init bf16 weights, fp32 norm weights)",
        "config": bench_config(world),
        "prefill_tok_s": round(prefill_tps, 1),
        "decode_ms_per_token_step": round(decode_ms / (a.steps * steps_dec), 4),
        "decode_top_p_tok_s": round(top_p_tps * world, 2),
        "decode_top_p_what": "second run: temperature 0.6, top-p 0.9, seeded uniforms; steps launched one by one",
        "prefill_ms": round(prefill_ms / a.steps, 3),
        "roofline": {"bound": "hbm", "kernel": "linear_decode_kernel (decode projections: wq/wk/wv, wo, w1/w3, w2, output)",
                     "achieved": round(dec_gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(dec_gbs / hbm, 4), "peak_source": f"{peak_src} hbm_gbs",
                     "traffic": _traffic("linear_decode_kernel"), "launches": n_proj,
                     "what": "algorithmic bytes of one decode step's projection launches / their exclusive "
                             "device time inside the graph-replayed batch-4 step (each launch's end minus its "
                             "predecessor's end, from %globaltimer stamps; the parts sum to the step)",
                     "traffic_what": "DRAM bytes per launch, mean over one decode step's 129 projection launches "
                                     "(ncu record in profiles/dram_traffic_7b.json; null if the kernel changed since)"},
        "roofline_serialised": {"achieved": round(dec_gbs_serial, 1), "unit": "GB/s",
                                "frac": round(dec_gbs_serial / hbm, 4), "launches": len(dec),
                                "what": "the same kernel launched alone (events around each of the projection "
                                        "launches of 16 directly launched decode steps, no programmatic "
                                        "dependent launch): ramp and tail of every launch included"},
        "decode_step_breakdown_us": {k: round(v / 1e3, 2) for k, v in sorted(tl_kind_ns.items())},
        "decode_step_timeline_us": round(tl_step_ns / 1e3, 2),
        "roofline_prefill": {"bound": "tensor", "kernel": "linear_tcp_pair_kernel / linear_tcp_kernel (prefill projections: wq/wk/wv, w1/w3, w2 on CTA pairs with 256x256 tiles, wo on single SMs with 128x256 tiles; persistent)",
                             "achieved": round(pre_tfs, 1), "peak": tc_burst, "unit": "TFLOP/s",
                             "frac": round(pre_tfs / tc_burst, 4), "peak_source": f"{peak_src} bf16_tflops (burst)",
                             "sustained_peak": tc_sust, "frac_sustained": round(pre_tfs / tc_sust, 4),
                             "clocks": pre_clk,
                             "clocks_what": "SM clocks sampled while prefills run back to back: the power cap holds "
                                            "them below the maximum, which is what the sustained peak describes",
                             "traffic": _traffic("prefill_projections"), "launches": len(pre),
                             "per_kind": pre_kind_line,
                             "what": "2*M*N*K of one prefill's projection launches / their event-timed durations "
                                     "(prefill launches run one after another in the product path too)",
                             "traffic_what": "DRAM bytes per launch, mean over the 128 projection launches of one "
                                             "prefill (ncu record in profiles/dram_traffic_7b.json; null if the kernel changed since)"},
        "decode_path_hbm": {"achieved": round(decode_gbs_path, 1), "unit": "GB/s",
                            "frac": round(decode_gbs_path / hbm, 4),
                            "what": "all algorithmic bytes of a greedy decode step (weights, norms, embedding rows, "
                                    "KV read + write; no logits are stored) / decode time"},
        "decode_b1": {"tok_s": round(b1_tps, 2), "ms_per_token_step": round(b1_ms / (a.steps * steps_dec), 4),
                      "hbm": {"achieved": round(b1_gbs, 1), "unit": "GB/s", "frac": round(b1_gbs / hbm, 4)},
                      "clocks": clk_b1,
                      "what": "the same model at batch 1: row 0's 512-token prompt, then 256 graph-replayed "
                              "greedy decode steps (contexts 513..768), timed per bench step"},
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": B * T * 4,
                "d2h_bytes_per_step": B * 4 * (steps_dec + 1),
                "what": "decode tokens per second of whole requests through the Python API: each bench step "
                        "times the prompt's copy from pinned host memory, the prefill, the first token and 256 "
                        "directly launched decode steps, every generated token read back to the host and "
                        "synchronised on, as a serving loop does"},
        "gpu_launches": int(launches),
        "launches_per_step": int(launches_per_step),
        "decode_graph": graph is not None,
        "clocks": clk,
        "impl": "ours",
    }
    return line


# ----------------------------------------------------------------------------- oracle (CPU) sample

def oracle_sample(seconds: float = 12.0):
    """Times the oracle on a bounded sample of the 7B workload: decode of one
    token of one row at context 640 through `nl` layers (as many as fit the
    time budget, at least 1) plus the final norm, vocabulary projection and
    sampling, extrapolated to the 32-layer model.  Returns (tok_s, sample, cores)."""
    import numpy as np
    from oracle import llama_oracle as O
    from workloads import LazyF64Weights, make_normal

    try:
        from threadpoolctl import threadpool_info
    except Exception:  # pragma: no cover
        threadpool_info = lambda: []  # noqa: E731
    s = L7B
    nl = 2
    w = make_weights(s.replace(n_layers=nl), 4242, device="cpu")
    args = O.Args(dim=s.dim, n_layers=nl, n_heads=s.n_heads, n_kv_heads=s.n_kv_heads, vocab_size=s.vocab_size,
                  max_seq_len=1024)
    lw = LazyF64Weights(w)
    ctx = 640
    cache = O.new_cache(args)
    for l in range(nl):
        cache.k[l][:ctx] = make_normal((ctx, s.n_kv_heads, s.head_dim), 7 + l, dtype=torch.float32).double().numpy()
        cache.v[l][:ctx] = make_normal((ctx, s.n_kv_heads, s.head_dim), 9 + l, dtype=torch.float32).double().numpy()
    x = np.asarray(lw["tok_embeddings"][np.array([123])], dtype=np.float64)
    t0 = time.perf_counter()
    layers_done = 0
    while True:
        for l in range(nl):
            x = O.layer_forward(args, lw["layers"][l], x, cache, l, ctx)
            layers_done += 1
        if time.perf_counter() - t0 > seconds / 2 or layers_done >= 8:
            break
    t_layer = (time.perf_counter() - t0) / layers_done
    t1 = time.perf_counter()
    h = O.rms_norm(x, lw["norm"], args.norm_eps)
    logits = h @ np.asarray(lw["output"], dtype=np.float64).T
    O.greedy(logits[0])
    t_head = time.perf_counter() - t1
    t_tok = t_layer * s.n_layers + t_head
    cores = 0
    for info in threadpool_info():
        cores = max(cores, int(info.get("num_threads", 0)))
    cores = cores or (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())
    sample = (f"oracle (numpy fp64) decode of 1 token of 1 row at context {ctx}: {layers_done} 7B-shaped layer "
              f"passes timed ({t_layer * 1e3:.0f} ms each) plus final norm + 32000x4096 vocabulary projection + "
              f"argmax ({t_head * 1e3:.0f} ms), extrapolated to 32 layers")
    return 1.0 / t_tok, sample, cores


def run_reference(a, rank, world):
    if rank != 0:
        return None
    vals, walls = [], []
    sample = cores = None
    for i in range(a.warmup + a.steps):
        t0 = time.perf_counter()
        v, sample, cores = oracle_sample(seconds=6.0)
        if i >= a.warmup:
            vals.append(v)
            walls.append(time.perf_counter() - t0)
    value = statistics.mean(vals)
    # one step of this arm is one bounded oracle sample (its measured wall
    # time); the per-token time is an extrapolation to the 32-layer model
    return {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": round(1e3 * statistics.mean(walls), 1),
            "ms_per_token_extrapolated": round(1e3 / value, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(world),
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- single projection

def run_op_linear(a):
    """Times one bf16 projection (llama_op_linear) back to back: M token rows
    against an N x K weight, rotating over enough weight copies that the
    working set exceeds L2.  Prints a JSON line with GB/s and TFLOP/s."""
    import decoder_only_transformer_llama_b200 as llb
    M, N, K = (int(v) for v in a.op_linear.split(","))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm, tc_burst, _, peak_src = _peaks()
    wbytes = 2 * N * K
    copies = max(1, -(-3 * 126 * 2 ** 20 // wbytes))
    g = torch.Generator(device=dev).manual_seed(1)
    Ws = [(torch.randn(N, K, generator=g, device=dev) * 0.02).to(torch.bfloat16) for _ in range(copies)]
    A = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(M, N, device=dev)
    for i in range(3):
        llb.op_linear(A, Ws[i % copies], out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(a.iters):
        llb.op_linear(A, Ws[i % copies], out)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.iters
    byts = wbytes + 2 * M * K + 4 * M * N
    print(json.dumps({"op": "linear_bf16", "M": M, "N": N, "K": K, "us": round(ms * 1e3, 2),
                      "GB_s": round(byts / ms / 1e6, 1), "hbm_frac": round(byts / ms / 1e6 / hbm, 4),
                      "TFLOP_s": round(2 * M * N * K / ms / 1e9, 1),
                      "tc_frac": round(2 * M * N * K / ms / 1e9 / tc_burst, 4), "weight_copies": copies,
                      "peak_source": peak_src}), flush=True)


def run_op_sample(a):
    """Times top-p sampling (llama_sample, temperature 0.6, top-p 0.9) of B
    rows of V seeded N(0, 2.5) logits with seeded uniforms, back to back.
    Prints a JSON line with the time per call and the logit bytes it reads."""
    import decoder_only_transformer_llama_b200 as llb
    B, V = (int(v) for v in a.op_sample.split(","))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(B)
    logits = torch.randn(B, V, generator=g, device=dev) * 2.5
    uni = torch.rand(B, generator=g, device=dev)
    out = torch.empty(B, dtype=torch.int32, device=dev)
    for _ in range(3):
        llb.sample(logits, 0.6, 0.9, uni, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        llb.sample(logits, 0.6, 0.9, uni, out)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.iters
    print(json.dumps({"op": "sample_top_p", "B": B, "V": V, "temperature": 0.6, "top_p": 0.9,
                      "us": round(ms * 1e3, 2), "logit_bytes": 4 * B * V,
                      "picks": out[:8].tolist()}), flush=True)


# ----------------------------------------------------------------------------- other workloads

def _timed(fn, iters, stream, clocks=False):
    """Mean device time (ms) of one call of `fn` over `iters` calls, CUDA events
    on `stream`; with `clocks`, nvidia-smi clocks sampled during the region.
    Returns (ms, clocks or None)."""
    import tempfile
    sampler = ClockSampler(0, os.path.join(tempfile.gettempdir(), "llama_b200_clocks_workload.csv")) if clocks else None
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    return ms, (sampler.stop() if sampler else None)


def _reps_for(ms_once, min_ms=600.0):
    """Repetitions of a timed sequence that make the region last about min_ms
    (long enough for a few 200 ms clock samples)."""
    return max(1, int(min_ms / max(ms_once, 1e-3)) + 1)


LAYER_CHAIN = 8   # single-layer decode steps per graph replay in the 7b_layer_decode workload


def run_workload(a):
    """Throughput lines for the other workloads (one JSON line per measurement):
    7b_layer_decode (one 7B layer, cache pre-filled, B x context grid),
    13b_ragged (16 prompts of 64..1024 tokens, then 128 decode steps),
    70b_slice (16 GQA layers, 8 x 2048 prefill, then decode), tiny_f32,
    7b_batch1 (the full 7B shape, one 512-token prompt, then 256 decode steps)."""
    import decoder_only_transformer_llama_b200 as llb
    from workloads import make_lengths, make_normal
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm, tc_burst, _, peak_src = _peaks()
    name = a.workload
    wl = WORKLOADS[name]
    s = wl["shape"]
    if a.layers:
        s = s.replace(n_layers=a.layers)   # a shallower copy of the shape (profiling one kernel on a small case)
    if name == "7b_layer_decode":
        # the single-layer microbench has no vocabulary projection; a decode
        # step of the library always ends in one, so it gets the smallest head
        # a 16-bit model takes, 256 rows (2 MB of weights, counted in the
        # step's bytes)
        s = s.replace(vocab_size=256)
    stream = torch.cuda.current_stream()
    w = make_weights(s, weight_seed(wl["index"]), device=dev)
    model = llb.Model(llb.args_from_shape(s), device=dev)
    model.load(w)
    del w
    torch.cuda.empty_cache()
    out = []
    if name == "7b_layer_decode":
        kv, vv = model.kv_tensors(0)
        for L in wl["contexts"]:
            kv[:, :L].copy_(make_normal(kv[:, :L].shape, 11, device=dev))
            vv[:, :L].copy_(make_normal(vv[:, :L].shape, 12, device=dev))
            for B in wl["batches"]:
                tok = make_tokens(s.vocab_size, (B,), token_seed(wl["index"])).to(dev)
                pos = torch.full((B,), L, dtype=torch.int32, device=dev)
                lg = torch.empty(B, s.vocab_size, device=dev)
                step = lambda: model.decode_step(tok, pos, logits=lg)
                for _ in range(5):
                    step()
                # consecutive steps chained in one graph, as a decode loop runs
                # them (each step complete: embedding, the layer, the head); the
                # replay boundary is paid once per LAYER_CHAIN steps
                g = torch.cuda.CUDAGraph()
                sc = torch.cuda.Stream(device=dev)
                sc.wait_stream(stream)
                with torch.cuda.stream(sc):
                    with torch.cuda.graph(g, stream=sc):
                        for _ in range(LAYER_CHAIN):
                            step()
                stream.wait_stream(sc)
                torch.cuda.synchronize()
                once, _ = _timed(g.replay, 20, stream)
                ms, clk = _timed(g.replay, max(100, a.iters, _reps_for(once)), stream, clocks=True)
                ms /= LAYER_CHAIN
                byts = decode_step_bytes(s, B, L + 1)
                # the layer's own share of a step (the microbench has no
                # embedding and no head): exclusive device time of its five
                # launches in the second of two graph-replayed steps, from the
                # library's timeline, against the layer's bytes alone
                model.timeline_start()
                g_tl = capture_graph(lambda: (step(), step()), dev, stream)
                model.timeline_stop()
                for _ in range(8):
                    g_tl.replay()
                del g_tl
                recs = model.timeline_stop()
                n_step = len(recs) // 2
                ends = [r[0] for r in recs]
                second = range(n_step, 2 * n_step)
                head = max(i for i in second if recs[i][1] == "projection")
                layer_ns = sum(ends[i] - ends[i - 1] for i in second
                               if recs[i][1] in ("projection", "attention") and i != head)
                layer_bytes = (byts - 2 * s.vocab_size * s.dim - 4 * s.dim - 2 * B * s.dim
                               - 4 * B * s.vocab_size)
                out.append({"workload": name, "n_layers": s.n_layers, "head_rows": s.vocab_size, "batch": B,
                            "context": L + 1, "steps_per_graph": LAYER_CHAIN, "us_per_step": round(ms * 1e3, 2),
                            "tok_s": round(B / (ms / 1e3), 1), "GB_s": round(byts / ms / 1e6, 1),
                            "hbm_frac": round(byts / ms / 1e6 / hbm, 4), "peak_source": peak_src,
                            "layer_us": round(layer_ns / 1e3, 2),
                            "layer_tok_s": round(B / (layer_ns / 1e9), 1),
                            "layer_hbm_frac": round(layer_bytes / layer_ns / hbm, 4),
                            "layer_what": "the layer's five launches (wq/wk/wv, attention, wo, w1/w3, w2) of a "
                                          "graph-replayed step, exclusive %globaltimer time each, without the "
                                          "embedding and the 256-row stand-in head a library step also runs",
                            "clocks": clk})
                del g
    else:
        B = wl["batch"]
        if name == "13b_ragged":
            lens = make_lengths(B, wl["min_len"], wl["max_len"], token_seed(wl["index"]))
            T = max(lens)
            steps = wl["decode_steps"]
        elif name == "70b_slice":
            T = wl["prompt_len"]
            lens = [T] * B
            steps = a.decode_steps or (wl["decode_to"] - T)
        else:
            T = wl["prompt_len"]
            lens = [T] * B
            steps = wl["decode_steps"]
        prompt = make_tokens(s.vocab_size, (B, T), token_seed(wl["index"])).to(dev)
        logits = torch.empty(B, s.vocab_size, device=dev)
        tok = torch.empty(B, dtype=torch.int32, device=dev)
        pos0 = torch.tensor(lens, dtype=torch.int32, device=dev)
        pos = pos0.clone()
        for _ in range(2):
            model.prefill(prompt, lens=lens, logits=logits)
        torch.cuda.synchronize()
        prefill = lambda: model.prefill(prompt, lens=lens, logits=logits)  # noqa: E731
        once, _ = _timed(prefill, 1, stream)
        pre_ms, pre_clk = _timed(prefill, max(3, _reps_for(once)), stream, clocks=True)
        llb.sample(logits, 0.0, 0.9, None, tok)
        pos.copy_(pos0)
        for _ in range(3):
            model.decode_step(tok, pos, temperature=0.0, next_tokens=tok, advance=True)
        pos.copy_(pos0)
        torch.cuda.synchronize()
        g = None
        if s.dtype != "f32":
            g = torch.cuda.CUDAGraph()
            sc = torch.cuda.Stream(device=dev)
            sc.wait_stream(stream)
            with torch.cuda.stream(sc):
                with torch.cuda.graph(g, stream=sc):
                    model.decode_step(tok, pos, temperature=0.0, next_tokens=tok, advance=True)
            stream.wait_stream(sc)
            pos.copy_(pos0)
            torch.cuda.synchronize()
        step = g.replay if g is not None else (lambda: model.decode_step(tok, pos, temperature=0.0,
                                                                           next_tokens=tok, advance=True))
        # one decode sequence = `steps` steps from the prompts' ends (positions
        # reset on the device first); repeated so the region lasts >= 0.6 s
        def sequence():
            pos.copy_(pos0)
            for _ in range(steps):
                step()
        once, _ = _timed(sequence, 1, stream)
        seq_ms, dec_clk = _timed(sequence, _reps_for(once), stream, clocks=True)
        dec_ms = seq_ms / steps
        assert model.status() == 0
        n_tok = sum(lens)
        mean_ctx = sum(lens) / B + steps / 2
        byts = decode_step_bytes(s, B, int(mean_ctx), logits=False) if s.dtype != "f32" else None
        out.append({"workload": name, "n_layers": s.n_layers, "batch": B, "prompt_tokens": n_tok,
                    "prefill_ms": round(pre_ms, 3),
                    "prefill_tok_s": round(n_tok / (pre_ms / 1e3), 1), "decode_steps": steps,
                    "decode_ms_per_step": round(dec_ms, 4), "decode_tok_s": round(B / (dec_ms / 1e3), 1),
                    "decode_hbm_frac": round(byts / dec_ms / 1e6 / hbm, 4) if byts else None,
                    "peak_source": peak_src, "prefill_clocks": pre_clk, "decode_clocks": dec_clk})
        del g
    for line in out:
        print(json.dumps(line), flush=True)


def run_profile_steps(a):
    """A short, fixed launch sequence for ncu captures: the 7B shape (--layers
    to shorten it), one 4 x 512 prefill, then --profile-steps greedy decode
    steps launched directly (no graph).  With --profile-prefill-kernels the
    prefill projections are also timed one by one (events; the prefill runs
    no programmatic dependent launch) and printed as one JSON line."""
    import decoder_only_transformer_llama_b200 as llb
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = L7B.replace(n_layers=a.layers) if a.layers else L7B
    w = make_weights(s, weight_seed(WL["index"]), device=dev)
    model = llb.Model(llb.args_from_shape(s), device=dev)
    model.load(w)
    del w
    torch.cuda.empty_cache()
    B, T = WL["batch"], WL["prompt_len"]
    prompt = make_tokens(s.vocab_size, (B, T), token_seed(WL["index"])).to(dev)
    logits = torch.empty(B, s.vocab_size, device=dev)
    tok = torch.empty(B, dtype=torch.int32, device=dev)
    pos = torch.full((B,), T, dtype=torch.int32, device=dev)
    if a.profile_prefill_kernels:
        model.prefill(prompt, logits=logits)
        torch.cuda.synchronize()
        model.profile_start(8 * s.n_layers + 8)
    model.prefill(prompt, logits=logits)
    if a.profile_prefill_kernels:
        recs = model.profile_stop(8 * s.n_layers + 8)
        names = ["wq/wk/wv", "wo", "w1/w3", "w2"]
        per = {}
        for i, r in enumerate(recs):
            if r[3] <= 64:
                continue
            k = names[i % 4] if i < 4 * s.n_layers else "output"
            per.setdefault(k, [0.0, 0])
            per[k][0] += r[0]
            per[k][1] += r[2]
        print(json.dumps({"prefill_projection_ms": {k: round(v[0], 3) for k, v in per.items()},
                          "prefill_projection_tflops": {k: round(v[1] / (v[0] / 1e3) / 1e12, 1)
                                                        for k, v in per.items() if v[0] > 0}}), flush=True)
    llb.sample(logits, 0.0, 0.9, None, tok)
    for _ in range(a.profile_steps):
        model.decode_step(tok, pos, temperature=0.0, next_tokens=tok, advance=True)
    torch.cuda.synchronize()
    assert model.status() == 0
    print(json.dumps({"profile_steps": a.profile_steps, "n_layers": s.n_layers,
                      "launches": llb.launch_count()}), flush=True)


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op-linear", default=None, metavar="M,N,K",
                    help="time one bf16 projection instead of the model (kernel microbenchmark)")
    ap.add_argument("--op-sample", default=None, metavar="B,V",
                    help="time top-p sampling of B rows of V logits (llama_sample) and exit")
    ap.add_argument("--iters", type=int, default=50)
    ap.add_argument("--no-graph", action="store_true", help="launch decode steps directly instead of a CUDA graph")
    ap.add_argument("--workload", default="7b", choices=list(WORKLOADS),
                    help="7b is the headline line; the others print throughput lines of their own")
    ap.add_argument("--decode-steps", type=int, default=0, help="decode steps of the 70b_slice workload")
    ap.add_argument("--layers", type=int, default=0,
                    help="--workload / --profile-steps: run the shape with this many layers (small cases for kernel profiles)")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="ncu helper: 7B prefill 4x512 + this many directly launched decode steps, then exit")
    ap.add_argument("--profile-prefill-kernels", action="store_true",
                    help="with --profile-steps: time the prefill projections one by one and print them")
    a = ap.parse_args()
    if a.op_linear:
        run_op_linear(a)
        return
    if a.op_sample:
        run_op_sample(a)
        return
    if a.profile_steps or a.profile_prefill_kernels:
        a.profile_steps = max(a.profile_steps, 1)
        run_profile_steps(a)
        return
    if a.workload != "7b":
        run_workload(a)
        return
    if a.warmup < 3:
        a.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if a.impl == "reference":
        line = run_reference(a, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        line = run_ours(a, rank, world, local_rank)
        if rank == 0 and world == 1 and not a.no_cpu_baseline:
            v, sample, cores = oracle_sample()
            line["cpu_baseline"] = {"value": round(v, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
                                    "sample": sample}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
