"""GPU parity of every stage against the oracle on small seeded cases that span
several tiles and ragged tails, plus the method's degenerate cases."""
import numpy as np
import pytest
import torch

from query_oriented_sparse_b200 import binding as Bd
from query_oriented_sparse_b200 import workloads as W

from gpu_harness import check_step, run_gpu

pytestmark = pytest.mark.gpu

C = W.custom
CASES = [
    C("mqa_f32_d64", h_q=4, h_kv=1, head_dim=64, chunk=128, prefix=384, nq=16, budget=128,
      dtype="f32"),
    C("f32_d128_ragged", h_q=4, h_kv=2, head_dim=128, chunk=130, prefix=700, nq=20, budget=90,
      dtype="f32", seed=3),
    C("gqa_bf16_ragged", h_q=8, h_kv=2, head_dim=128, chunk=200, prefix=1000, nq=24,
      budget=100, recipe="rank4", seed=5),
    C("no_prefix", h_q=4, h_kv=2, head_dim=128, chunk=70, prefix=0, nq=8, budget=16, seed=6),
    C("budget_covers_prefix", h_q=4, h_kv=2, head_dim=128, chunk=64, prefix=50, nq=8,
      budget=64, seed=7),
    C("nq_covers_chunk", h_q=4, h_kv=1, head_dim=64, chunk=40, prefix=300, nq=64, budget=32,
      seed=8),
    C("batch3_ragged", h_q=8, h_kv=4, head_dim=128, chunk=96, prefix=(0, 77, 1500), nq=12,
      budget=(10, 64, 200), recipe="heavy", seed=9),
    C("d64_group8", h_q=16, h_kv=2, head_dim=64, chunk=256, prefix=4096, nq=32, budget=512,
      seed=10),
    C("chunk1", h_q=4, h_kv=2, head_dim=128, chunk=1, prefix=300, nq=4, budget=32, seed=11),
    C("budget0", h_q=4, h_kv=2, head_dim=128, chunk=32, prefix=100, nq=4, budget=0, seed=12),
    C("group16", h_q=32, h_kv=2, head_dim=128, chunk=64, prefix=2000, nq=8, budget=256,
      recipe="rank4", seed=13),
    C("long_tail_bf16", h_q=8, h_kv=1, head_dim=128, chunk=300, prefix=5000, nq=40, budget=613,
      recipe="heavy", seed=14),
    # 3 heads of 112 padded rows per column group: two uneven head-aligned slices
    C("uneven_slices", h_q=12, h_kv=2, head_dim=128, chunk=150, prefix=3000, nq=100, budget=300,
      recipe="rank4", seed=17),
    # three heads of 128 kept queries per KV head (accumulator slices of 256 and 128
    # columns), a prefix that ends inside a key tile
    C("g3_nq128", h_q=6, h_kv=2, head_dim=128, chunk=300, prefix=2100, nq=128,
      budget=300, recipe="heavy", seed=19),
    # three heads of 64 kept queries, head_dim 64
    C("g3_nq64_d64", h_q=3, h_kv=1, head_dim=64, chunk=100, prefix=700, nq=64,
      budget=96, seed=20),
    # one head of 16 kept queries per KV head: a 16-column accumulator slice
    C("g1_nq16", h_q=2, h_kv=2, head_dim=128, chunk=64, prefix=600, nq=16, budget=64, seed=21),
    # two column groups of 8 heads per KV head, two sequences
    C("two_colgroups", h_q=16, h_kv=1, head_dim=128, chunk=128, prefix=(1500, 260), nq=64,
      budget=(200, 64), recipe="rank4", seed=22),
    # kept queries wider than one accumulator slice per head: CUDA-core scoring
    C("wide_nq", h_q=4, h_kv=2, head_dim=64, chunk=400, prefix=900, nq=300, budget=200, seed=18),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_stage_parity(w, cuda_device):
    t = W.generate(w)
    res = run_gpu(w, t)
    rep = check_step(w, t, res)
    print(w.name, rep)


def _tie_workload():
    """Keys drawn from 5 distinct rows and queries from 6 distinct rows, so pooled
    scores and query cosines tie exactly on the GPU (identical rows take identical
    arithmetic) and the tie-break decides which members of a class are kept."""
    w = C("exact_ties", h_q=4, h_kv=2, head_dim=128, chunk=48, prefix=640, nq=10, budget=100,
          seed=15)
    t = W.generate(w)
    g = torch.Generator().manual_seed(99)
    krows = torch.randn(2, 5, 128, generator=g).to(torch.bfloat16)
    pick = torch.randint(0, 5, (640,), generator=g)
    k = t.k_cache.clone()
    k[:, :640] = krows[:, pick]
    qrows = torch.randn(4, 6, 128, generator=g).to(torch.bfloat16)
    qpick = torch.randint(0, 6, (48,), generator=g)
    q = qrows[:, qpick][None].contiguous()
    return w, W.Tensors(q, k.contiguous(), t.v_cache, t.kv_off), pick.numpy(), qpick.numpy()


def _lowest_members_kept(kept_idx, classes):
    """Within every class of identical rows, the kept members are its lowest indices."""
    kept = set(int(x) for x in kept_idx)
    for c in np.unique(classes):
        members = np.flatnonzero(classes == c)
        flags = [int(m) in kept for m in members]
        n = sum(flags)
        assert flags == [True] * n + [False] * (len(flags) - n), (c, members, flags)


def test_exact_ties_take_lowest_index(cuda_device):
    w, t, pick, qpick = _tie_workload()
    res = run_gpu(w, t)
    check_step(w, t, res)
    for h in range(w.h_q):
        _lowest_members_kept(res["kept"][0, h, :w.nq], qpick)
    for g in range(w.h_kv):
        sel = res["idx"][0, g, :100]
        _lowest_members_kept(sel, pick)
        # and the split between classes follows the GPU's own pooled scores
        s = res["pooled"][0, g, :640]
        thr = np.sort(s)[::-1][99]
        assert set(np.flatnonzero(s > thr)) <= set(sel.tolist())
        assert not (set(sel.tolist()) & set(np.flatnonzero(s < thr)))


def test_zero_vectors(cuda_device):
    """A zero query and zero keys have cosine 0 (no NaN anywhere)."""
    w = C("zeros", h_q=4, h_kv=2, head_dim=128, chunk=64, prefix=512, nq=8, budget=64, seed=16)
    t = W.generate(w)
    q = t.q.clone()
    q[0, 1, 5] = 0
    k = t.k_cache.clone()
    k[:, 10:20] = 0
    t2 = W.Tensors(q, k, t.v_cache, t.kv_off)
    res = run_gpu(w, t2)
    assert np.isfinite(res["pooled"][0, :, :512]).all()
    assert (res["pooled"][0, :, 10:20] == 0).all()
    check_step(w, t2, res)


def test_deterministic(cuda_device):
    w = CASES[2]
    t = W.generate(w)
    a, b = run_gpu(w, t), run_gpu(w, t)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["kept"], b["kept"])
    assert np.array_equal(a["out"], b["out"])


def test_rejections_launch_nothing(cuda_device):
    """Invalid calls with real buffers return the documented status and leave the
    outputs untouched."""
    w = CASES[2]
    t = W.generate(w)
    q = t.q.cuda()
    k = t.k_cache.cuda()
    v = t.v_cache.cuda()
    idx = torch.full((1, 2, 100), -5, dtype=torch.int32, device="cuda")
    with pytest.raises(Bd.QuokaError) as e:
        Bd.quoka_select(q, k, t.kv_off, (t.kv_off[1],), w.nq, w.budget, 100, idx_out=idx)
    assert e.value.status == Bd.QUOKA_ERR_INVALID_ARG
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(Bd.QuokaError) as e:
        Bd.quoka_select(q, k, t.kv_off, w.prefix, w.nq, w.budget, 100, idx_out=idx,
                        workspace=small)
    assert e.value.status == Bd.QUOKA_ERR_WORKSPACE
    out = torch.full_like(q, 3.0)
    with pytest.raises(Bd.QuokaError):
        Bd.sparse_chunk_attn(q, k, v, t.kv_off, w.prefix, (101,), idx, out=out)
    torch.cuda.synchronize()
    assert (idx == -5).all() and (out == 3.0).all()
