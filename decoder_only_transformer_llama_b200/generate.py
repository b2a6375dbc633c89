"""Host driver of the reference's generation loop over the C ABI (Admin Guide
§8.5; User Guide §1 and the per-call parameters of §3.4; source tour, "The
decode loop in generate").

Every row advances through the same positions: the prompts are right-padded
into a (rows, total_len) table, the first forward (llama_prefill) runs the
first min(prompt lengths) tokens of every row, and each later position is one
llama_decode_step of all rows at that position.  The next token comes from
llama_sample (argmax at temperature 0, else nucleus sampling with the caller's
uniforms); where a row's prompt still covers the position, the prompt's token
is kept instead.  A row has finished once it produced EOS outside its prompt;
the loop ends early when every row has.  Log-probabilities come from
llama_token_logprobs on the logits of each forward.

Readings of what the pages leave open (the oracle's generate takes the same):
total_len = min(max_seq_len, max_gen_len + longest prompt), max_gen_len
defaulting to max_seq_len - 1; the draw for position p of row b uses
uniforms[p, b]; the log-probability of the token at position p is the
log-softmax (of the raw logits) at that token of the logits that predict p,
and 0 for position 0; a row's result runs from position 0 (echo) or from the
end of its prompt up to prompt length + max_gen_len, cut before the first EOS
at or after the end of its prompt.

The driver only moves data and makes the per-step decisions the loop makes on
the host (keep the prompt token, track EOS); every forward pass, every sampled
token and every log-probability is computed by the library's kernels.
"""
from typing import List, Optional, Sequence, Tuple

import numpy as np

from . import Model, sample, token_logprobs

PAD = -1


def generate(model: Model, prompts: Sequence[Sequence[int]], max_gen_len: Optional[int] = None,
             temperature: float = 0.6, top_p: float = 0.9, uniforms=None, logprobs: bool = False,
             echo: bool = False, eos_id: Optional[int] = None
             ) -> Tuple[List[List[int]], Optional[List[List[float]]]]:
    """Generate continuations of `prompts` (lists of token ids) with `model`.

    uniforms: device fp32 tensor [>= total_len, len(prompts)], needed when
    temperature > 0.  Returns (token lists, log-probability lists or None)."""
    import torch

    a = model.args
    S, V = a.max_seq_len, a.vocab_size
    dev = model.arena.device
    B = len(prompts)
    if B < 1 or B > a.max_batch_size:
        raise ValueError(f"{B} prompts for max_batch_size {a.max_batch_size}")
    lens = [len(p) for p in prompts]
    if min(lens) < 1 or max(lens) > S:
        raise ValueError("every prompt needs 1 .. max_seq_len tokens")
    if max_gen_len is None:
        max_gen_len = S - 1
    total = min(S, max_gen_len + max(lens))
    if temperature > 0 and (uniforms is None or uniforms.shape[0] < total or uniforms.shape[1] != B):
        raise ValueError(f"sampling needs uniforms of shape [>= {total}, {B}]")

    tok = np.full((B, total), PAD, dtype=np.int64)
    for b, p in enumerate(prompts):
        tok[b, :len(p)] = p
    in_prompt = tok != PAD
    lp = np.zeros((B, total))
    done = np.zeros(B, dtype=bool)
    start = min(lens)

    def logprobs_of(rows_logits, first, last):
        # log-probabilities of tok[:, first:last] under rows_logits [B * (last - first), V]
        n = last - first
        tgt = torch.from_numpy(tok[:, first:last].reshape(-1).astype(np.int32)).to(dev)
        out = torch.empty(B * n, dtype=torch.float32, device=dev)
        token_logprobs(rows_logits, tgt, out)
        lp[:, first:last] = out.cpu().numpy().astype(np.float64).reshape(B, n)

    last_lg = torch.empty(B, V, dtype=torch.float32, device=dev)
    nxt = torch.empty(B, dtype=torch.int32, device=dev)
    pos = torch.empty(B, dtype=torch.int32, device=dev)
    if start == total:
        if logprobs:   # nothing to generate: only the prompts' log-probabilities
            all_lg = torch.empty(B, total, V, dtype=torch.float32, device=dev)
            x = torch.from_numpy(tok[:, :total].astype(np.int32)).to(dev)
            model.prefill(x, logits=all_lg, all_logits=True)
            logprobs_of(all_lg[:, :-1].reshape(B * (total - 1), V).contiguous(), 1, total)
    prev = 0
    for cur in range(start, total):
        if cur == start:
            x = torch.from_numpy(tok[:, :start].astype(np.int32)).to(dev)
            if logprobs:
                all_lg = torch.empty(B, start, V, dtype=torch.float32, device=dev)
                model.prefill(x, logits=all_lg, all_logits=True)
                last_lg.copy_(all_lg[:, -1])
                rows = all_lg.reshape(B * start, V)
            else:
                model.prefill(x, logits=last_lg)
        else:
            x = torch.from_numpy(tok[:, prev].astype(np.int32)).to(dev)
            pos.fill_(prev)
            model.decode_step(x, pos, logits=last_lg)
            rows = last_lg
        if temperature > 0:
            sample(last_lg, temperature, top_p, uniforms[cur].contiguous(), nxt)
        else:
            sample(last_lg, 0.0, top_p, None, nxt)
        chosen = nxt.cpu().numpy().astype(np.int64)
        tok[:, cur] = np.where(in_prompt[:, cur], tok[:, cur], chosen)
        if logprobs:
            logprobs_of(rows, prev + 1, cur + 1)
        if eos_id is not None:
            done |= (~in_prompt[:, cur]) & (tok[:, cur] == eos_id)
        prev = cur
        if eos_id is not None and done.all():
            break
    status = model.status()
    if status != 0:
        raise RuntimeError(f"device status {status} during generation")

    out_tok, out_lp = [], []
    for b in range(B):
        first = 0 if echo else lens[b]
        last = min(total, lens[b] + max_gen_len)
        t = tok[b, first:last].tolist()
        l = lp[b, first:last].tolist()
        if eos_id is not None:
            for i in range(max(0, lens[b] - first), len(t)):
                if t[i] == eos_id:
                    t, l = t[:i], l[:i]
                    break
        out_tok.append(t)
        out_lp.append(l)
    return out_tok, (out_lp if logprobs else None)
