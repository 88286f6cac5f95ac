"""Per-query sparse attention with shared loading (QUILT page, summary): every query
attends to its own key set, tiles of up to 16 rows load the union of their sets once.
Checked row by row against the oracle's per-query attention, across both dtypes and head
sizes, group sizes 1 to 16 (3 and 12 leave padding rows in every tile), ragged tiles,
ragged batches, padding, duplicate entries and an empty set (zeros)."""
import numpy as np
import pytest
import torch

from oracle import quoka_oracle as O
from query_oriented_sparse_b200 import binding as Bd
from query_oriented_sparse_b200 import workloads as W

from parity_util import ATTN_TOL, row_rel_err

pytestmark = pytest.mark.gpu

C_ = W.custom
CASES = [
    # (workload: prefix + chunk give each sequence's rows, S entries per query)
    (C_("pq_bf16_d128_g4", h_q=8, h_kv=2, head_dim=128, chunk=64, prefix=2000, nq=1, budget=1,
        recipe="rank4", seed=61), 32),
    (C_("pq_f32_d64_g2_ragged", h_q=4, h_kv=2, head_dim=64, chunk=37, prefix=(500, 1300), nq=1,
        budget=1, dtype="f32", seed=62), 16),
    (C_("pq_bf16_d64_g16", h_q=16, h_kv=1, head_dim=64, chunk=10, prefix=3000, nq=1, budget=1,
        seed=63), 200),
    (C_("pq_bf16_d128_g1_long", h_q=2, h_kv=2, head_dim=128, chunk=50, prefix=40000, nq=1,
        budget=1, recipe="heavy", seed=64), 64),
    # group sizes that do not divide the 16-row tile: rows G * TQ .. 15 are padding
    (C_("pq_bf16_d128_g3_ragged", h_q=6, h_kv=2, head_dim=128, chunk=23, prefix=(700, 90),
        nq=1, budget=1, recipe="rank4", seed=65), 24),
    (C_("pq_f32_d128_g12", h_q=12, h_kv=1, head_dim=128, chunk=9, prefix=1500, nq=1, budget=1,
        dtype="f32", seed=66), 40),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_perq_parity(case, cuda_device):
    w, S = case
    t = W.generate(w)
    C = w.chunk
    sel = torch.empty(w.batch, w.h_q, C, S, dtype=torch.int32)
    for b in range(w.batch):
        n = t.kv_off[b + 1] - t.kv_off[b]
        sel[b] = W.per_query_selection(w.seed * 10 + b, w.h_q, C, n, S, group=8, shared=0.75)
    # padding, a duplicate entry, and (on the first case with S > 2) an empty set
    sel[0, 0, 1, S - 1] = -1
    sel[0, w.h_q - 1, C - 1, 0] = sel[0, w.h_q - 1, C - 1, 1]
    empty = (0, 1, C // 2)
    sel[empty] = -1
    dev = cuda_device
    out = Bd.sparse_perq_attn(t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev), t.kv_off,
                              sel.to(dev))
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    got = out.float().cpu().numpy()
    assert (got[empty] == 0).all()
    tol = ATTN_TOL[w.dtype]
    for b in range(w.batch):
        lo, hi = t.kv_off[b], t.kv_off[b + 1]
        sb = sel[b].numpy().copy()
        if b == 0:
            sb[empty[1:]] = 0                       # give the oracle a key; row not compared
        ref = O.attend_per_query(t.q[b], t.k_cache[:, lo:hi], t.v_cache[:, lo:hi], sb)
        keep = np.ones((w.h_q, C), dtype=bool)
        if b == 0:
            keep[empty[1:]] = False
        e = row_rel_err(got[b][keep], ref[keep])
        assert e <= tol, f"{w.name} sequence {b}: rel err {e} > {tol}"


def test_perq_rejects(cuda_device):
    w, S = CASES[0]
    t = W.generate(w)
    dev = cuda_device
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    sel = torch.zeros(1, w.h_q, w.chunk, S, dtype=torch.int32, device=dev)
    out = torch.full_like(q, 7.0)
    with pytest.raises(Bd.QuokaError) as ex:
        Bd.sparse_perq_attn(q, k, v, t.kv_off, sel, out=out,
                            workspace=torch.zeros(256, dtype=torch.uint8, device=dev))
    assert ex.value.status == Bd.QUOKA_ERR_WORKSPACE
    with pytest.raises(Bd.QuokaError) as ex:
        Bd.sparse_perq_attn(q, k, v, (0, 0), sel, out=out)
    assert ex.value.status == Bd.QUOKA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())


# ---- the tensor-core form over 256-row pair tiles ----------------------------------------

TC_CASES = [
    # (workload, S, locality group, shared fraction, heads share their token's set)
    (C_("pqtc_g4", h_q=8, h_kv=2, head_dim=128, chunk=100, prefix=3000, nq=1, budget=1,
        recipe="rank4", seed=81), 48, 64, 0.9, True),
    (C_("pqtc_g3_ragged", h_q=6, h_kv=2, head_dim=128, chunk=90, prefix=(1500, 700), nq=1,
        budget=1, recipe="heavy", seed=82), 40, 32, 0.75, False),
    (C_("pqtc_g1", h_q=2, h_kv=2, head_dim=128, chunk=300, prefix=5000, nq=1, budget=1,
        seed=83), 64, 128, 0.95, False),
    (C_("pqtc_g16", h_q=32, h_kv=2, head_dim=128, chunk=20, prefix=2500, nq=1, budget=1,
        seed=84), 32, 16, 0.9, True),
    # a set size that is not a multiple of 4: the union kernel's 4-byte entry loads
    (C_("pqtc_g2_s37", h_q=4, h_kv=2, head_dim=128, chunk=70, prefix=1800, nq=1, budget=1,
        seed=85), 37, 32, 0.8, False),
]


def _tc_sel(w, t, S, group, shared, share_heads):
    sel = torch.empty(w.batch, w.h_q, w.chunk, S, dtype=torch.int32)
    for b in range(w.batch):
        n = t.kv_off[b + 1] - t.kv_off[b]
        x = W.per_query_selection_large(w.seed * 10 + b, w.h_q, w.chunk, n, S, group=group,
                                        shared=shared)
        if share_heads:                       # every head of a KV group reads its token's set
            G = w.h_q // w.h_kv
            x = x.view(w.h_kv, G, w.chunk, S)[:, :1].expand(w.h_kv, G, w.chunk, S).reshape_as(x)
        sel[b] = x
    return sel


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: c[0].name)
def test_perq_tc_parity(case, cuda_device):
    w, S, group, shared, share_heads = case
    t = W.generate(w)
    C = w.chunk
    sel = _tc_sel(w, t, S, group, shared, share_heads)
    sel = sel[..., torch.randperm(S, generator=torch.Generator().manual_seed(5))].contiguous()  # any order
    sel[0, 0, 1, 0] = -1                                  # padding
    sel[0, w.h_q - 1, C - 1, 1] = sel[0, w.h_q - 1, C - 1, 2]   # a duplicate
    empty = (0, 1, C // 2)
    sel[empty] = -1
    dev = cuda_device
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    cap = 256 * S
    out = Bd.sparse_perq_attn_tc(q, k, v, t.kv_off, sel.to(dev), max_union=cap)
    ref_gpu = Bd.sparse_perq_attn(q, k, v, t.kv_off, sel.to(dev))
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    got = out.float().cpu().numpy()
    assert (got[empty] == 0).all()
    tol = ATTN_TOL[w.dtype]
    for b in range(w.batch):
        lo, hi = t.kv_off[b], t.kv_off[b + 1]
        sb = sel[b].numpy().copy()
        if b == 0:
            sb[empty[1:]] = 0
        ref = O.attend_per_query(t.q[b], t.k_cache[:, lo:hi], t.v_cache[:, lo:hi], sb)
        keep = np.ones((w.h_q, C), dtype=bool)
        if b == 0:
            keep[empty[1:]] = False
        e = row_rel_err(got[b][keep], ref[keep])
        assert e <= tol, f"{w.name} sequence {b}: rel err {e} > {tol}"
    # the two forms agree (up to the order of summation)
    e2 = row_rel_err(got.reshape(-1, w.head_dim), ref_gpu.float().cpu().numpy().reshape(-1, w.head_dim))
    assert e2 <= tol, e2


def test_perq_tc_union_bound_is_flagged(cuda_device):
    """A union larger than max_union sets bit 3 of the device error word and the call
    still finishes (the over-full tiles keep their first max_union keys)."""
    w, S, group, shared, share_heads = TC_CASES[0]
    t = W.generate(w)
    sel = _tc_sel(w, t, S, group, shared, share_heads)
    dev = cuda_device
    Bd.sparse_perq_attn_tc(t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev), t.kv_off,
                           sel.to(dev), max_union=S)
    torch.cuda.synchronize()
    assert Bd.device_error() & 8


def test_perq_tc_rejects(cuda_device):
    w, S = CASES[1][0], CASES[1][1]                     # fp32: not taken by the tensor-core form
    t = W.generate(w)
    dev = cuda_device
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    sel = torch.zeros(w.batch, w.h_q, w.chunk, S, dtype=torch.int32, device=dev)
    with pytest.raises(Bd.QuokaError) as ex:
        Bd.sparse_perq_attn_tc(q, k, v, t.kv_off, sel, max_union=64,
                               workspace=torch.zeros(256, dtype=torch.uint8, device=dev))
    assert ex.value.status == Bd.QUOKA_ERR_UNSUPPORTED
