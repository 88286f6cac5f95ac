"""Runs one chunk step through the C ABI and checks it against the oracle."""
from __future__ import annotations

import numpy as np
import torch

from oracle import quoka_oracle as O
from query_oriented_sparse_b200 import binding as Bd
from query_oriented_sparse_b200 import workloads as W

from parity_util import (ATTN_TOL, check_index_row, compare_kept_set, compare_top_set,
                         row_rel_err, stratified_rows)


def run_gpu(w: W.Workload, t: W.Tensors, chunk_index: int = 0, device="cuda"):
    """Selection + attention for one chunk step; returns host copies of every output."""
    prefix = tuple(p + chunk_index * w.chunk for p in w.prefix)
    q = t.q_chunk(chunk_index, w.chunk).to(device)
    k = t.k_cache.to(device)
    v = t.v_cache.to(device)
    shape = Bd.shape_of(q, k)
    b_max = max(max(w.budget), 1)
    kept = torch.full((w.batch, w.h_q, w.nq), -7, dtype=torch.int32, device=device)
    ws_bytes = Bd.select_workspace_size(shape, max(prefix), w.nq)
    ws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device=device)   # NaN-poisoned
    idx = torch.full((w.batch, w.h_kv, b_max), -7, dtype=torch.int32, device=device)
    Bd.quoka_select(q, k, t.kv_off, prefix, w.nq, w.budget, b_max, idx_out=idx, kept_out=kept,
                    workspace=ws)
    out = torch.full_like(q, float("nan"))
    Bd.sparse_chunk_attn(q, k, v, t.kv_off, prefix, w.budget, idx, out=out)
    torch.cuda.synchronize()
    err = Bd.device_error()
    pooled = Bd.pooled_view(ws, shape, max(prefix), w.nq)
    return {
        "prefix": prefix,
        "kept": kept.cpu().numpy(),
        "idx": idx.cpu().numpy(),
        "pooled": pooled.cpu().numpy(),
        "out": out.float().cpu().numpy(),
        "device_error": err,
    }


def check_step(w: W.Workload, t: W.Tensors, res, chunk_index: int = 0, attn_rows=None):
    """Asserts parity of one chunk step; returns a report dict.

    attn_rows: None for every output row, or "tiles" for one row of every query tile of
    every KV head of every sequence plus each head's first and last position of the
    last tile (parity_util.stratified_rows).
    """
    assert res["device_error"] == 0
    report = {"kept_near_ties": 0, "idx_near_ties": 0, "max_pooled_err": 0.0,
              "max_attn_rel_err": 0.0}
    q_all = t.q_chunk(chunk_index, w.chunk)
    nk = min(w.nq, w.chunk)
    tol = ATTN_TOL[w.dtype]
    rng = np.random.default_rng(1234 + chunk_index)
    for b in range(w.batch):
        P = res["prefix"][b]
        lo, hi = t.kv_off[b], t.kv_off[b + 1]
        q64 = q_all[b].to(torch.float64).numpy()
        kseq = t.k_cache[:, lo:hi].to(torch.float64).numpy()
        vseq = t.v_cache[:, lo:hi].to(torch.float64).numpy()
        cos = np.stack([O.query_cosines(q64[h]) for h in range(w.h_q)])
        gpu_kept = []
        for h in range(w.h_q):
            row = res["kept"][b, h]
            head = row[:nk].astype(np.int64)
            assert (row[nk:] == -1).all()
            assert ((head >= 0) & (head < w.chunk)).all() and (np.diff(head) > 0).all()
            n = compare_kept_set(head, cos[h], w.nq)
            report["kept_near_ties"] += n
            gpu_kept.append(head)
        ref = O.select_chunk(q64, kseq, P, w.nq, w.budget[b], kept_override=gpu_kept)
        n_sel = min(w.budget[b], P)
        gpu_idx = []
        for g in range(w.h_kv):
            sc = ref["score"][g]
            got = res["pooled"][b, g, :P].astype(np.float64)
            if P:
                err = np.abs(got - sc)
                assert (err <= 2e-6 + 1e-5 * np.abs(sc)).all(), \
                    f"pooled scores off: max err {err.max()} at {int(err.argmax())}"
                report["max_pooled_err"] = max(report["max_pooled_err"], float(err.max()))
            head = check_index_row(res["idx"][b, g], n_sel, P)
            n = compare_top_set(head, sc, w.budget[b])
            report["idx_near_ties"] += n
            gpu_idx.append(head)
        if attn_rows is None:
            o_ref = O.attend_chunk(q64, kseq, vseq, P, gpu_idx)
            e = row_rel_err(res["out"][b], o_ref)
        else:
            assert attn_rows == "tiles", attn_rows
            rows = stratified_rows(w.h_q, w.h_kv, w.chunk, rng)
            o_ref = O.attend_chunk(q64, kseq, vseq, P, gpu_idx, rows=rows)
            o_gpu = np.stack([res["out"][b, h, tt] for h, tt in rows])
            e = row_rel_err(o_gpu, o_ref)
        assert e <= tol, f"attention rel err {e} > {tol} (sequence {b})"
        report["max_attn_rel_err"] = max(report["max_attn_rel_err"], e)
    return report
