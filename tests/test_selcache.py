"""Selected-value cache with miss-only fetch (SQD page, the sparse-attention paragraph:
the chosen values are kept where attention runs and only the misses are fetched).

Each case runs a sequence of selections through one cache: the selection quoka_select
makes (from an empty cache), the same again (no miss), one that keeps half of it, one
that shares nothing with it, and one with a smaller budget.  After every update:
  - the slot map equals the oracle's slot map, and the miss counts its misses;
  - every live slot holds its row's K/V bytes exactly, the chunk rows follow, then zero
    rows up to the next multiple of 128;
  - attention over the cache matches the oracle's attention over the rows the slots
    hold, and is bit-identical to sparse_chunk_attn whenever the slots hold the rows in
    ascending order (from an empty cache, with no miss, and when nothing was kept).
Tensor-core (bf16, d 128 and 64), decode-gather (bf16) and CUDA-core (fp32) paths.
"""
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
    C_("sc_bf16_d128", h_q=8, h_kv=2, head_dim=128, chunk=96, prefix=(1500, 700), nq=16,
       budget=(256, 128), recipe="rank4", seed=71),
    C_("sc_bf16_decode", h_q=8, h_kv=2, head_dim=128, chunk=1, prefix=(3000, 900, 2000), nq=1,
       budget=(384, 100, 200), recipe="heavy", seed=72),
    C_("sc_f32_d64", h_q=4, h_kv=1, head_dim=64, chunk=40, prefix=800, nq=8, budget=100,
       dtype="f32", seed=73),
    C_("sc_bf16_d64", h_q=4, h_kv=2, head_dim=64, chunk=64, prefix=1000, nq=8, budget=150,
       seed=74),
]


def _pack(rows_per_bg, batch, h_kv, b_max):
    idx = torch.full((batch, h_kv, b_max), -1, dtype=torch.int32)
    for (b, g), r in rows_per_bg.items():
        idx[b, g, :len(r)] = torch.as_tensor(np.sort(np.asarray(r, dtype=np.int64)), dtype=torch.int32)
    return idx


def _steps(w, idx0, rng):
    """(budget, idx) of each step after the first: the same selection, half kept, none
    kept, then half the budget drawn from the previous selection."""
    b_max = idx0.shape[-1]
    out = [(w.budget, idx0.clone())]
    sets = {}
    for b in range(w.batch):
        n = min(w.budget[b], w.prefix[b])
        for g in range(w.h_kv):
            sets[(b, g)] = idx0[b, g, :n].numpy().astype(np.int64)
    out.append((w.budget, idx0.clone()))
    half, none = {}, {}
    for (b, g), s in sets.items():
        P = w.prefix[b]
        keep = s[::2]
        rest = np.setdiff1d(np.arange(P), s)
        half[(b, g)] = np.concatenate([keep, rng.choice(rest, size=len(s) - len(keep), replace=False)])
        rest2 = np.setdiff1d(np.arange(P), half[(b, g)])
        none[(b, g)] = rng.choice(rest2, size=len(s), replace=False)
    out.append((w.budget, _pack(half, w.batch, w.h_kv, b_max)))
    out.append((w.budget, _pack(none, w.batch, w.h_kv, b_max)))
    small = tuple(max(1, x // 2) for x in w.budget)
    shrink = {}
    for (b, g), s in none.items():
        n = min(small[b], w.prefix[b])
        shrink[(b, g)] = rng.choice(s, size=n, replace=False)
    out.append((small, _pack(shrink, w.batch, w.h_kv, b_max)))
    return out


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_selcache_steps(w, cuda_device):
    dev = cuda_device
    t = W.generate(w)
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    b_max = max(w.budget)
    idx0 = Bd.quoka_select(q, k, t.kv_off, w.prefix, w.nq, w.budget, b_max).cpu()
    shape = Bd.shape_of(q, k)
    cache = Bd.SelCache(shape, b_max, dev)
    rng = np.random.default_rng(w.seed)
    slots_prev = np.full((w.batch, w.h_kv, b_max), -1, dtype=np.int64)
    q64 = t.q.to(torch.float64).numpy()
    C, d = w.chunk, w.head_dim
    kc_rows = (b_max + C + 127) // 128 * 128
    ascending_steps = {0, 1, 3}
    for step, (budget, idx) in enumerate(_steps(w, idx0, rng)):
        misses = cache.update(k, v, t.kv_off, w.prefix, budget, idx.to(dev)).cpu().numpy()
        out = cache.attend(q, w.prefix, budget)
        ref_gpu = Bd.sparse_chunk_attn(q, k, v, t.kv_off, w.prefix, budget, idx.to(dev))
        torch.cuda.synchronize()
        assert Bd.device_error() == 0
        slots = cache.slot_rows.cpu().numpy()
        kb, vb = (x.cpu() for x in cache.blocks(w.torch_dtype))
        for b in range(w.batch):
            P = w.prefix[b]
            n = min(budget[b], P)
            lo = t.kv_off[b]
            for g in range(w.h_kv):
                want, miss = O.selected_value_slots(slots_prev[b, g], idx[b, g, :n].numpy(), n)
                assert slots[b, g].tolist() == want, (step, b, g)
                assert misses[b, g] == len(miss), (step, b, g, misses[b, g], len(miss))
                rows = torch.as_tensor(slots[b, g, :n], dtype=torch.long)
                assert torch.equal(kb[b, g, :n], t.k_cache[g, lo + rows])
                assert torch.equal(vb[b, g, :n], t.v_cache[g, lo + rows])
                assert torch.equal(kb[b, g, n:n + C], t.k_cache[g, lo + P:lo + P + C])
                assert torch.equal(vb[b, g, n:n + C], t.v_cache[g, lo + P:lo + P + C])
                end = (n + C + 127) // 128 * 128
                assert end <= kc_rows
                assert not kb[b, g, n + C:end].any() and not vb[b, g, n + C:end].any()
            slots_prev[b] = slots[b]
            kseq = t.k_cache[:, lo:t.kv_off[b + 1]].to(torch.float64).numpy()
            vseq = t.v_cache[:, lo:t.kv_off[b + 1]].to(torch.float64).numpy()
            held = [slots[b, g, :n] for g in range(w.h_kv)]
            o_ref = O.attend_chunk(q64[b], kseq, vseq, P, held)
            e = row_rel_err(out[b].float().cpu().numpy(), o_ref)
            assert e <= ATTN_TOL[w.dtype], (step, b, e)
        if step in ascending_steps:
            assert torch.equal(out, ref_gpu), f"step {step}: not bit-identical to sparse_chunk_attn"


def test_selcache_rejects(cuda_device):
    w = CASES[0]
    t = W.generate(w)
    dev = cuda_device
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    shape = Bd.shape_of(q, k)
    b_max = max(w.budget)
    cache = Bd.SelCache(shape, b_max, dev)
    idx = torch.full((w.batch, w.h_kv, b_max), -1, dtype=torch.int32, device=dev)
    lib = Bd.lib()
    ctypes = Bd.ctypes
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def upd(budget=w.budget, ws_bytes=None, cache_ptr=None):
        return lib.quoka_selcache_update(
            ctypes.byref(shape), Bd._ptr(k), Bd._ptr(v), Bd._host_i64(t.kv_off),
            Bd._host_i32(w.prefix), Bd._host_i32(budget), Bd._ptr(idx), b_max,
            cache_ptr if cache_ptr is not None else Bd._ptr(cache.cache), Bd._ptr(cache.slot_rows),
            None, Bd._ptr(cache.workspace),
            cache.workspace.numel() if ws_bytes is None else ws_bytes, st)

    before = cache.slot_rows.clone()
    assert upd(budget=(b_max + 1, 1)) == Bd.QUOKA_ERR_INVALID_ARG
    assert upd(ws_bytes=256) == Bd.QUOKA_ERR_WORKSPACE
    assert upd(cache_ptr=ctypes.c_void_p(cache.cache.data_ptr() + 16)) == Bd.QUOKA_ERR_INVALID_ARG
    out = torch.full_like(q, 5.0)
    assert lib.sparse_chunk_attn_selcache(
        ctypes.byref(shape), Bd._ptr(q), Bd._host_i32(w.prefix), Bd._host_i32((b_max + 1, 1)),
        Bd._ptr(cache.cache), b_max, Bd._ptr(out), Bd._ptr(cache.workspace),
        cache.workspace.numel(), st) == Bd.QUOKA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.equal(cache.slot_rows, before) and bool((out == 5.0).all())
