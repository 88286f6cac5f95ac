"""fp64 CPU oracle for QUOKA-style KV selection followed by sparse chunk attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module; only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the CUDA
library and imports nothing from the product package.

What it computes, and where each step comes from
------------------------------------------------
Sources are the QUOKA page ("Qualcomm QuoKA: ... 5x", arXiv 2602.08722), its
method summary and the captions of Figure 1 and Figure 2, plus the multi-query
attention page ("Multi-Query Attention", technical insight section) for the
sharing of one K/V head by several query heads.

QUOKA is a heuristic selection followed by exact dense attention over the selected
set, so the oracle follows the method's steps in the pages' order:

1. mean query (method summary; Q&A 1): per query head, the mean of the chunk's
   unit-normalised queries, m = (1/C) sum_t q_t / |q_t|.
2. query subselection (Figure 1(b): "filter queries by cosine dissimilarity";
   Figure 2: queries with high S_q interact more strongly): c_t = cos(q_t, m);
   keep the Nq queries with the smallest c_t (largest S_q = -c_t); ties go to
   the lower chunk position.  Nq >= C keeps every query.
3. cosine scoring (Figure 1(b): "query-key cosine similarity filters keys"):
   cos(q_i, k_j) for every kept query i and every prefix key j < P.
4. group-aware aggregation (method summary: max pooling "to preserve important
   interactions", mean pooling "to adapt to GQA", respectively): per key, max over
   the kept queries of each query head, then mean over the G heads sharing the
   KV head.
5. top-B (Figure 1(a): the KV cache is sub-selected into a "compacted cache"):
   per KV head the B best-scoring prefix keys, ties to the lower cache index,
   returned in ascending index order; P <= B keeps every prefix key.
6. dense attention over the compacted cache (Figure 1(a)): query t of head h
   attends to the selected prefix keys of KV head h // G plus the chunk's own
   keys P .. P+t (causal), softmax(q k^T / sqrt(d)) v.

7. whole-prompt chunked prefill (Figure 1(a): a prompt cut into chunks, each chunk
   sub-selecting the cache that the chunks before it wrote): chunk c has prefix
   P = c * C, selects over rows 0 .. P-1 with that chunk's budget, and attends.
8. per-query sparse attention (QUILT page, summary: each query has its own selected
   key-value entries, and nearby queries share many of them): query t of head h
   attends to exactly its own set of key positions, softmax(q k^T / sqrt(d)) v over
   that set.  This is what shared-query execution must reproduce, whatever grouping
   and union loading it uses.
9. selected-value cache (SQD page, the sparse-attention paragraph: the top-k choice
   scans the whole cache, attention runs over the chosen values kept where it runs, and
   only the values not kept yet, the misses, are sent): the slot map after moving the
   kept rows to a new selection.  The page does not say where a fetched row goes; the
   reading here is that a row kept before and chosen again stays in its slot and the
   misses, in ascending row order, fill the freed slots in ascending order.

Readings where the pages are silent (each is listed with its reason in the design
notes of the repository): the budget B counts prefix keys only and the chunk's own
causal keys are always attended; the mean query is per query head and over
*normalised* queries; a zero vector has cosine 0 with everything; the softmax scale
is 1/sqrt(d); head h maps to KV head h // G.

All arithmetic is float64 on exact copies of the (fp32 or bf16) inputs.
Pins: tests/test_oracle.py checks every step against brute force, closed forms,
invariants and an independent library routine.  End-to-end agreement with the
authors' own implementation is "parity unpinned": the pages print no worked numbers.
"""
from __future__ import annotations

from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "unit_rows", "mean_query", "query_cosines", "subselect_queries", "pooled_key_scores",
    "top_budget", "select_chunk", "attend_chunk", "select_batch", "attend_batch",
    "prefill_prompt", "attend_per_query", "selected_value_slots",
]


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):                       # a torch tensor: exact widening
        x = x.detach().to("cpu")
        import torch  # local: only for the dtype conversion of torch inputs
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def unit_rows(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Row norms and unit rows of x [n, d]; a zero row stays zero (cosine 0)."""
    x = _f64(x)
    n = np.sqrt(np.einsum("nd,nd->n", x, x))
    u = np.zeros_like(x)
    nz = n > 0
    u[nz] = x[nz] / n[nz, None]
    return n, u


def mean_query(q: np.ndarray, raw: bool = False) -> np.ndarray:
    """Step 1: the chunk's mean query for one head, q [C, d] -> [d].

    ``raw=True`` averages the unnormalised queries instead; it exists only so the
    tests can show that this alternative reading breaks the per-query scale
    invariance that the cosine-based method has.
    """
    q = _f64(q)
    if raw:
        return q.mean(axis=0)
    _, u = unit_rows(q)
    return u.mean(axis=0)


def query_cosines(q: np.ndarray, raw_mean: bool = False) -> np.ndarray:
    """Step 2a: c_t = cos(q_t, m) for one head, q [C, d] -> [C]."""
    _, u = unit_rows(q)
    m = mean_query(q, raw=raw_mean)
    mn = np.sqrt(m @ m)
    if mn == 0.0:
        return np.zeros(u.shape[0])
    return u @ (m / mn)


def subselect_queries(q: np.ndarray, nq: int, raw_mean: bool = False) -> np.ndarray:
    """Step 2b: indices (ascending) of the min(nq, C) queries least similar to the mean.

    Ordering key: cosine ascending, then chunk position ascending.
    """
    c = query_cosines(q, raw_mean=raw_mean)
    C = c.shape[0]
    if nq >= C:
        return np.arange(C, dtype=np.int64)
    order = np.lexsort((np.arange(C), c))
    return np.sort(order[:nq]).astype(np.int64)


def pooled_key_scores(kept_units: Sequence[np.ndarray], k: np.ndarray,
                      block: int = 8192) -> np.ndarray:
    """Steps 3-4 for one KV head.

    kept_units: one array [Nk_h, d] of unit kept queries per query head of the group.
    k: prefix keys [P, d].  Returns score [P]:
        score_j = mean_h max_{i in K_h} (u_i . k_j) / |k_j|   (0 for a zero key).
    Keys are processed in blocks only to bound memory; no reordering of the
    arithmetic beyond that.
    """
    k = _f64(k)
    P = k.shape[0]
    out = np.zeros(P)
    if P == 0:
        return out
    G = len(kept_units)
    for s in range(0, P, block):
        kb = k[s:s + block]
        r, _ = unit_rows(kb)
        acc = np.zeros(kb.shape[0])
        for uh in kept_units:
            dots = _f64(uh) @ kb.T                      # [Nk_h, blk]
            acc += dots.max(axis=0)
        acc /= G
        nz = r > 0
        blk = np.zeros(kb.shape[0])
        blk[nz] = acc[nz] / r[nz]
        out[s:s + block] = blk
    return out


def top_budget(score: np.ndarray, budget: int) -> np.ndarray:
    """Step 5: the min(budget, P) best prefix keys, ties to the lower index, ascending."""
    score = _f64(score)
    P = score.shape[0]
    if budget >= P:
        return np.arange(P, dtype=np.int64)
    order = np.lexsort((np.arange(P), -score))
    return np.sort(order[:budget]).astype(np.int64)


def select_chunk(q_chunk, k_seq, prefix_len: int, nq: int, budget: int,
                 kept_override: Optional[Sequence[np.ndarray]] = None,
                 raw_mean: bool = False) -> Dict[str, object]:
    """Steps 1-5 for one sequence.

    q_chunk [H_q, C, d]; k_seq [H_kv, >= P, d] (rows of this sequence only).
    ``kept_override`` replaces step 2's kept sets (one index array per query head),
    used to re-score with another implementation's kept sets when those differ only
    by near-ties.
    Returns kept (list per query head), cos [H_q, C], score [H_kv, P], idx (list per
    KV head, ascending).
    """
    q = _f64(q_chunk)
    H_q, C, d = q.shape
    k = _f64(k_seq)
    H_kv = k.shape[0]
    G = H_q // H_kv
    P = int(prefix_len)
    cos = np.stack([query_cosines(q[h], raw_mean=raw_mean) for h in range(H_q)]) if C else \
        np.zeros((H_q, 0))
    if kept_override is not None:
        kept = [np.sort(np.asarray(x, dtype=np.int64)) for x in kept_override]
    else:
        kept = [subselect_queries(q[h], nq, raw_mean=raw_mean) for h in range(H_q)]
    score = np.zeros((H_kv, P))
    idx: List[np.ndarray] = []
    for g in range(H_kv):
        units = []
        for h in range(g * G, (g + 1) * G):
            _, u = unit_rows(q[h])
            units.append(u[kept[h]])
        score[g] = pooled_key_scores(units, k[g, :P])
        idx.append(top_budget(score[g], budget))
    return {"kept": kept, "cos": cos, "score": score, "idx": idx}


def attend_chunk(q_chunk, k_seq, v_seq, prefix_len: int, idx: Sequence[np.ndarray],
                 rows: Optional[Iterable[Tuple[int, int]]] = None) -> np.ndarray:
    """Step 6 for one sequence.

    q_chunk [H_q, C, d]; k_seq, v_seq [H_kv, >= P + C, d]; idx: per KV head the
    selected prefix indices.  Returns O [H_q, C, d], or, when ``rows`` is given, an
    array [len(rows), d] holding only those (head, position) rows.
    """
    q = _f64(q_chunk)
    H_q, C, d = q.shape
    k = _f64(k_seq)
    v = _f64(v_seq)
    H_kv = k.shape[0]
    G = H_q // H_kv
    P = int(prefix_len)
    scale = 1.0 / np.sqrt(d)
    want = None if rows is None else list(rows)
    heads = range(H_q) if want is None else sorted({h for h, _ in want})
    out = {}
    for h in heads:
        g = h // G
        sel = np.asarray(idx[g], dtype=np.int64)
        sel = sel[sel >= 0]
        ks = np.concatenate([k[g, sel], k[g, P:P + C]], axis=0)
        vs = np.concatenate([v[g, sel], v[g, P:P + C]], axis=0)
        ns = sel.shape[0]
        ts = range(C) if want is None else sorted({t for hh, t in want if hh == h})
        for t in ts:
            n_keys = ns + t + 1                        # selected prefix + chunk keys P..P+t
            logits = (ks[:n_keys] @ q[h, t]) * scale
            mx = logits.max()
            p = np.exp(logits - mx)
            out[(h, t)] = (p @ vs[:n_keys]) / p.sum()
    if want is None:
        o = np.zeros((H_q, C, d))
        for (h, t), val in out.items():
            o[h, t] = val
        return o
    return np.stack([out[r] for r in want]) if want else np.zeros((0, d))


def _seq_rows(x, kv_off, b):
    return x[:, kv_off[b]:kv_off[b + 1]]


def select_batch(q, k_cache, kv_off, prefix_len, nq, budget):
    """select_chunk over a batch: q [batch, H_q, C, d], k_cache [H_kv, total, d]."""
    return [select_chunk(q[b], _seq_rows(k_cache, kv_off, b), prefix_len[b], nq, budget[b])
            for b in range(len(prefix_len))]


def attend_batch(q, k_cache, v_cache, kv_off, prefix_len, idx_per_seq):
    """attend_chunk over a batch; idx_per_seq[b] is a list of per-KV-head index arrays."""
    return np.stack([attend_chunk(q[b], _seq_rows(k_cache, kv_off, b),
                                  _seq_rows(v_cache, kv_off, b), prefix_len[b], idx_per_seq[b])
                     for b in range(len(prefix_len))])


def prefill_prompt(q_prompt, k_prompt, v_prompt, chunk: int, nq: int,
                   budgets: Sequence[int]) -> Dict[str, object]:
    """Step 7 for one sequence: the chunk loop of Figure 1(a) over a whole prompt.

    q_prompt [H_q, n*C, d]; k_prompt, v_prompt [H_kv, n*C, d] (the prompt's own K/V,
    row t written by chunk t // C); budgets has one entry per chunk.  Chunk c runs
    steps 1-6 with P = c * C: it can only see rows the earlier chunks appended, plus
    its own rows causally.  Returns out [H_q, n*C, d] and, per chunk, the selection.
    """
    q = _f64(q_prompt)
    k = _f64(k_prompt)
    v = _f64(v_prompt)
    n_tok = q.shape[1]
    C = int(chunk)
    n = n_tok // C
    assert n * C == n_tok and len(budgets) == n
    out = np.zeros_like(q)
    idx = []
    for c in range(n):
        P = c * C
        qc = q[:, P:P + C]
        sel = select_chunk(qc, k[:, :P], P, nq, int(budgets[c]))
        out[:, P:P + C] = attend_chunk(qc, k[:, :P + C], v[:, :P + C], P, sel["idx"])
        idx.append(sel["idx"])
    return {"out": out, "idx": idx}


def attend_per_query(q, k, v, sel) -> np.ndarray:
    """Step 8: every query row over its own selected keys.

    q [H_q, T, d]; k, v [H_kv, N, d] (rows of one sequence); sel int [H_q, T, S]: the
    key positions query (h, t) attends to, padded with -1 (duplicates count once).
    Query head h reads KV head h // G.  Returns O [H_q, T, d].
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    sel = np.asarray(sel, dtype=np.int64)
    H_q, T, d = q.shape
    G = H_q // k.shape[0]
    scale = 1.0 / np.sqrt(d)
    out = np.zeros((H_q, T, d))
    for h in range(H_q):
        g = h // G
        for t in range(T):
            keys = np.unique(sel[h, t][sel[h, t] >= 0])
            assert keys.size > 0, "every query needs at least one key"
            logits = (k[g, keys] @ q[h, t]) * scale
            p = np.exp(logits - logits.max())
            out[h, t] = (p @ v[g, keys]) / p.sum()
    return out


def selected_value_slots(slots_prev, idx_new, n: int):
    """Step 9: the slot map of a selected-value cache after moving it to a new selection.

    slots_prev: the row each slot held (-1 for none); idx_new: the n rows now selected
    (distinct); n: the live slots.  A slot below n whose row is selected again keeps it
    (if two slots held the same row, the lower one); every other slot below n is free;
    the misses (selected rows no live slot kept) go, in ascending order, into the free
    slots in ascending order; slots from n on are emptied.
    Returns (new slot map as a list, the misses in ascending order).
    """
    prev = [int(x) for x in slots_prev]
    wanted = set(int(x) for x in list(idx_new)[:n])
    assert len(wanted) == n, "the selection must name n distinct rows"
    new = [-1] * len(prev)
    kept = set()
    free = []
    for s in range(n):
        r = prev[s] if s < len(prev) else -1
        if r in wanted and r not in kept:
            new[s] = r
            kept.add(r)
        else:
            free.append(s)
    misses = sorted(wanted - kept)
    assert len(misses) == len(free)
    for s, r in zip(free, misses):
        new[s] = r
    return new, misses
