"""Seeded synthetic workloads for one chunk of a chunked prefill.

This module only *draws* tensors: it holds none of the selection or attention
arithmetic, so both the CUDA path (through the binding) and the fp64 oracle can be
fed from it without sharing any method code.

Six workloads are defined, matching the shapes of the QUOKA page's chunked-prefill
setting (page "Qualcomm QuoKA ...", Figure 1(a): a prompt split into chunks, each
chunk attending over a compacted KV cache) and its ~12 % KV budget (same page,
results section):

    tiny_mqa      H_q=4, H_kv=1, d=64, prompt 512 in 4 chunks of 128, Nq=16, B=128, fp32
    gqa_8k        H_q=32, H_kv=8, d=128, prefix 8192 + chunk 512, Nq=64, B=1024, bf16
    long_chunk    H_q=64, H_kv=8, d=128, prefix 32768 + chunk 2048, Nq=128, B=4096, bf16
    ctx_128k      H_q=32, H_kv=8, d=128, prefix 131072 + chunk 4096, Nq=128, B=16384, bf16
    ragged_8      8 sequences, prefix ~ U[4096, 65536], chunk 1024, H_q=64, H_kv=4,
                  d=128, Nq=64, B = 12 % of each prefix rounded to 64, bf16
    decode_32     one decode step of 32 sequences: prefix ~ U[2048, 16384], chunk 1 (the
                  new token), H_q=32, H_kv=8, d=128, Nq=1, B = 12 % of each prefix
                  rounded to 64, bf16, selection every step

and one whole prompt for the prefill call (chunk after chunk, cache appended inside):

    prompt_128k   the ctx_128k shapes from the first token: 33 chunks of 4096, chunk c
                  keeping c * 4096 / 8 prefix keys (its last chunk is the ctx_128k step)

Value recipes (all drawn in fp32 from ``torch.Generator('cpu').manual_seed(seed)``
and then rounded once to the workload dtype):

    gauss   Q, K, V ~ N(0, 1)
    rank4   Q, K ~ N(0, 1) + 2 * U_g z, with U_g an orthonormal d x 4 basis per KV
            head (QR of a Gaussian) and z ~ N(0, I_4) per token and head; V ~ N(0, 1)
    heavy   N(0, 1), then per (sequence, KV head) 2 % of the prefix rows (of a whole
            prompt: of all its rows) (without replacement) are replaced by 3 * sqrt(d) * q_hat, q_hat the direction of a
            uniformly drawn chunk query of a uniformly drawn head of that group

KV cache layout: ``k_cache``/``v_cache`` are [H_kv, kv_total, d]; sequence b owns rows
``[kv_off[b], kv_off[b+1])`` holding its prefix followed by its own chunk rows.
Queries are [batch, H_q, C, d].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    h_q: int
    h_kv: int
    head_dim: int
    chunk: int
    prefix: Tuple[int, ...]          # per sequence (for prompt workloads: chunk 0's)
    nq: int
    budget: Tuple[int, ...]          # per sequence, counts prefix keys only
    dtype: str                       # "f32" or "bf16"
    seed: int
    recipe: str                      # "gauss", "rank4" or "heavy"
    prompt_chunks: int = 1           # >1: whole prompt of prompt_chunks * chunk tokens
    chunk_budget: Tuple[int, ...] = ()   # whole prompts: budget of each chunk (else `budget`)

    @property
    def batch(self) -> int:
        return len(self.prefix)

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def seq_rows(self) -> Tuple[int, ...]:
        """Rows each sequence owns in the cache (prefix plus every chunk it will run)."""
        return tuple(p + self.chunk * self.prompt_chunks for p in self.prefix)

    def budgets_of_chunks(self) -> Tuple[int, ...]:
        """Budget of each chunk of a whole prompt (every sequence uses the same)."""
        if self.chunk_budget:
            return self.chunk_budget
        return (self.budget[0],) * self.prompt_chunks

    def chunk_steps(self):
        """(chunk index, per-sequence prefix lengths) for every chunk step of the workload."""
        for c in range(self.prompt_chunks):
            yield c, tuple(p + c * self.chunk for p in self.prefix)


def _budget_12pct(p: int) -> int:
    """12 % of a prefix, rounded to a multiple of 64 (halves up), at least 64."""
    return max(64, 64 * int(math.floor(0.12 * p / 64.0 + 0.5)))


def _ragged_prefixes(seed: int) -> Tuple[int, ...]:
    g = torch.Generator(device="cpu").manual_seed(seed)
    return tuple(int(x) for x in torch.randint(4096, 65537, (8,), generator=g))


_RAGGED = _ragged_prefixes(4)


def _decode_prefixes(seed: int) -> Tuple[int, ...]:
    g = torch.Generator(device="cpu").manual_seed(seed)
    return tuple(int(x) for x in torch.randint(2048, 16385, (32,), generator=g))


_DECODE = _decode_prefixes(5)

WORKLOADS: Dict[str, Workload] = {
    "tiny_mqa": Workload("tiny_mqa", 4, 1, 64, 128, (0,), 16, (128,), "f32", 0, "gauss",
                         prompt_chunks=4),
    "gqa_8k": Workload("gqa_8k", 32, 8, 128, 512, (8192,), 64, (1024,), "bf16", 1, "rank4"),
    "long_chunk": Workload("long_chunk", 64, 8, 128, 2048, (32768,), 128, (4096,), "bf16", 2,
                           "heavy"),
    "ctx_128k": Workload("ctx_128k", 32, 8, 128, 4096, (131072,), 128, (16384,), "bf16", 3,
                         "heavy"),
    "ragged_8": Workload("ragged_8", 64, 4, 128, 1024, _RAGGED, 64,
                         tuple(_budget_12pct(p) for p in _RAGGED), "bf16", 4, "rank4"),
    "decode_32": Workload("decode_32", 32, 8, 128, 1, _DECODE, 1,
                          tuple(_budget_12pct(p) for p in _DECODE), "bf16", 5, "heavy"),
}

# The headline single-GPU workload (128K context).
HEADLINE = "ctx_128k"

# Whole prompts run chunk by chunk through the prefill call (kept apart from WORKLOADS,
# whose entries are single chunk steps).  prompt_128k is the 128K-context workload's
# prompt from its first token: 33 chunks of 4096, chunk c keeping 1/8 of its c * 4096
# prefix keys, so its last chunk is the ctx_128k step (prefix 131072, B 16384).
PROMPTS: Dict[str, Workload] = {
    "prompt_128k": Workload("prompt_128k", 32, 8, 128, 4096, (0,), 128, (16384,), "bf16", 3,
                            "heavy", prompt_chunks=33,
                            chunk_budget=tuple(c * 4096 // 8 for c in range(33))),
}


def custom(name: str = "custom", *, h_q: int, h_kv: int, head_dim: int, chunk: int,
           prefix, nq: int, budget, dtype: str = "bf16", seed: int = 0,
           recipe: str = "gauss", prompt_chunks: int = 1, chunk_budget=()) -> Workload:
    """A small ad-hoc workload (tests use these for edge cases)."""
    prefix = tuple(int(p) for p in (prefix if hasattr(prefix, "__len__") else (prefix,)))
    if not hasattr(budget, "__len__"):
        budget = (int(budget),) * len(prefix)
    return Workload(name, h_q, h_kv, head_dim, chunk, prefix, nq, tuple(int(b) for b in budget),
                    dtype, seed, recipe, prompt_chunks, tuple(int(x) for x in chunk_budget))


@dataclasses.dataclass
class Tensors:
    """CPU tensors of one workload, already rounded to the workload dtype."""
    q: torch.Tensor          # [batch, H_q, prompt_chunks * C, d]
    k_cache: torch.Tensor    # [H_kv, kv_total, d]
    v_cache: torch.Tensor    # [H_kv, kv_total, d]
    kv_off: Tuple[int, ...]  # batch + 1 row offsets

    def q_chunk(self, c: int, chunk: int) -> torch.Tensor:
        return self.q[:, :, c * chunk:(c + 1) * chunk, :].contiguous()


def _orthonormal(g: torch.Generator, d: int, r: int) -> torch.Tensor:
    a = torch.randn(d, r, generator=g, dtype=torch.float64)
    qmat, _ = torch.linalg.qr(a)
    return qmat.to(torch.float32)


def generate(w: Workload) -> Tensors:
    """Draw the workload's Q and KV cache on the CPU from its seed."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    d = w.head_dim
    rows = w.seq_rows()
    kv_off = [0]
    for r in rows:
        kv_off.append(kv_off[-1] + r)
    total = kv_off[-1]
    qlen = w.chunk * w.prompt_chunks

    q = torch.randn(w.batch, w.h_q, qlen, d, generator=g)
    k = torch.randn(w.h_kv, total, d, generator=g)
    v = torch.randn(w.h_kv, total, d, generator=g)

    if w.recipe == "rank4":
        for kv in range(w.h_kv):
            basis = _orthonormal(g, d, 4)                               # [d, 4]
            zk = torch.randn(total, 4, generator=g)
            k[kv] += 2.0 * zk @ basis.T
            for h in range(kv * w.group, (kv + 1) * w.group):
                zq = torch.randn(w.batch, qlen, 4, generator=g)
                q[:, h] += 2.0 * zq @ basis.T
    elif w.recipe == "heavy":
        scale = 3.0 * math.sqrt(d)
        for b in range(w.batch):
            p = w.prefix[b] if w.prompt_chunks == 1 else rows[b]   # candidate rows
            n_heavy = int(round(0.02 * p))
            if n_heavy == 0:
                continue
            for kv in range(w.h_kv):
                pos = torch.randperm(p, generator=g)[:n_heavy]
                heads = torch.randint(kv * w.group, (kv + 1) * w.group, (n_heavy,), generator=g)
                toks = torch.randint(0, qlen, (n_heavy,), generator=g)
                src = q[b, heads, toks]                                  # [n_heavy, d]
                src = src / src.norm(dim=-1, keepdim=True).clamp_min(1e-30)
                k[kv, kv_off[b] + pos] = scale * src
    elif w.recipe != "gauss":
        raise ValueError(f"unknown recipe {w.recipe!r}")

    dt = w.torch_dtype
    return Tensors(q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous(),
                   tuple(kv_off))


def per_query_selection(seed: int, h_q: int, n_queries: int, n_keys: int, s: int,
                        group: int = 16, shared: float = 0.75) -> torch.Tensor:
    """Per-query key sets with locality, the input of shared-query execution (QUILT page:
    nearby queries select many of the same key-value entries).  Per query head, every run
    of `group` consecutive queries draws one base set of s keys; each query keeps
    round(shared * s) of them and draws the rest on its own, without repeats.  Returns
    int32 [h_q, n_queries, s], each row ascending."""
    if s > n_keys:
        raise ValueError("s must not exceed n_keys")
    g = torch.Generator(device="cpu").manual_seed(seed)
    keep = int(round(shared * s))
    out = torch.empty(h_q, n_queries, s, dtype=torch.int32)
    for h in range(h_q):
        for t0 in range(0, n_queries, group):
            base = torch.randperm(n_keys, generator=g)[:s]
            for t in range(t0, min(n_queries, t0 + group)):
                mine = base[torch.randperm(s, generator=g)[:keep]]
                taken = torch.zeros(n_keys, dtype=torch.bool)
                taken[mine] = True
                rest = torch.randperm(n_keys, generator=g)
                rest = rest[~taken[rest]][:s - keep]
                out[h, t] = torch.sort(torch.cat([mine, rest])).values.to(torch.int32)
    return out


def per_query_selection_large(seed: int, h_q: int, n_queries: int, n_keys: int, s: int,
                              group: int = 16, shared: float = 0.75,
                              causal_prefix=None) -> torch.Tensor:
    """per_query_selection for large sizes, vectorised per head: every run of `group`
    consecutive queries draws one base set; each entry of a query's set is the base
    set's entry at that slot with probability `shared`, else a draw of its own.  Draws
    are with replacement, so a set may hold a position twice (the attention counts it
    once).  With `causal_prefix` = P, query t draws only from rows 0 .. P + t (the
    prefix and the chunk rows up to its own), the base set of a run from the rows its
    first query may see; else from all n_keys rows.  Returns int32 [h_q, n_queries, s],
    rows ascending."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    ngroups = (n_queries + group - 1) // group
    gid = torch.arange(n_queries) // group
    if causal_prefix is None:
        lim_q = torch.full((n_queries, 1), n_keys, dtype=torch.float64)
        lim_g = torch.full((ngroups, 1), n_keys, dtype=torch.float64)
    else:
        lim_q = (causal_prefix + 1 + torch.arange(n_queries, dtype=torch.float64))[:, None]
        lim_g = (causal_prefix + 1 + group * torch.arange(ngroups, dtype=torch.float64))[:, None]
        if causal_prefix + n_queries > n_keys:
            raise ValueError("causal_prefix + n_queries exceeds n_keys")
    out = torch.empty(h_q, n_queries, s, dtype=torch.int32)
    for h in range(h_q):
        base = (torch.rand(ngroups, s, generator=g, dtype=torch.float64) * lim_g).long()
        own = (torch.rand(n_queries, s, generator=g, dtype=torch.float64) * lim_q).long()
        take = torch.rand(n_queries, s, generator=g) < shared
        rows = torch.where(take, base[gid], own)
        out[h] = torch.sort(rows, dim=1).values.to(torch.int32)
    return out


def drifting_queries(seed: int, q0: torch.Tensor, steps: int, sigma: float = 0.3) -> torch.Tensor:
    """Queries of consecutive decode steps that drift: step 0 is q0 [batch, h_q, d]; step
    s adds sigma * |q_{s-1}| / sqrt(d) * N(0, I) to step s-1's query (per row), so
    consecutive steps point in nearby directions and select overlapping key sets, as
    consecutive tokens of one text do.  Returns [steps, batch, h_q, 1, d] in q0's dtype."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    d = q0.shape[-1]
    cur = q0.float()
    out = [cur]
    for _ in range(1, steps):
        noise = torch.randn(cur.shape, generator=g)
        cur = cur + sigma * cur.norm(dim=-1, keepdim=True) / math.sqrt(d) * noise
        out.append(cur)
    return torch.stack(out, 0).unsqueeze(-2).to(q0.dtype).contiguous()
