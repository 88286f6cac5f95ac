"""The decode shape: one new token per sequence (C = 1) or a short chunk, so that at
most 16 query rows share a KV head.  The selection then scores keys on CUDA cores
(every query kept), the top-k runs one CTA per row when there are many short rows, and
the attention runs the split-K gather kernel (selected rows read straight from the
cache, partials merged per KV head).  These cases check all of it against the oracle
on every row, across many splits, ragged batches, both dtypes and head sizes, exact
ties, zero vectors and the degenerate cases (no prefix, budget 0, a chunk longer than
one token)."""
import numpy as np
import pytest
import torch

from query_oriented_sparse_b200 import workloads as W

from gpu_harness import check_step, run_gpu

pytestmark = pytest.mark.gpu

C = W.custom
CASES = [
    # rows per KV head G*C: 4 (R 4)
    C("dec_bf16_d128_batch3", h_q=32, h_kv=8, head_dim=128, chunk=1, prefix=(5000, 300, 12000),
      nq=1, budget=(600, 64, 1500), recipe="heavy", seed=31),
    # one sequence, 16384 selected keys: 65 splits per KV head
    C("dec_bf16_128k", h_q=32, h_kv=8, head_dim=128, chunk=1, prefix=131072, nq=1,
      budget=16384, recipe="heavy", seed=32),
    # 70000 selected keys for one KV head: hundreds of splits
    C("dec_bf16_70k_splits", h_q=2, h_kv=1, head_dim=128, chunk=1, prefix=80000, nq=1,
      budget=70000, recipe="heavy", seed=44),
    # G*C = 16 (R 16), d 64, a two-token chunk
    C("dec_bf16_d64_g8_c2", h_q=16, h_kv=2, head_dim=64, chunk=2, prefix=3000, nq=2, budget=400,
      recipe="rank4", seed=33),
    # G*C = 6 (R 8), budget covering the prefix
    C("dec_bf16_c3_full", h_q=4, h_kv=2, head_dim=128, chunk=3, prefix=200, nq=3, budget=256,
      seed=34),
    C("dec_f32_d128", h_q=8, h_kv=2, head_dim=128, chunk=1, prefix=(2000, 777), nq=1,
      budget=(256, 100), dtype="f32", seed=35),
    C("dec_f32_d64_g16", h_q=16, h_kv=1, head_dim=64, chunk=1, prefix=4000, nq=1, budget=512,
      dtype="f32", recipe="rank4", seed=36),
    C("dec_no_prefix", h_q=8, h_kv=2, head_dim=128, chunk=1, prefix=0, nq=1, budget=64, seed=37),
    C("dec_budget0", h_q=8, h_kv=2, head_dim=128, chunk=2, prefix=500, nq=2, budget=0, seed=38),
    C("dec_mqa_g1", h_q=1, h_kv=1, head_dim=128, chunk=1, prefix=9000, nq=1, budget=1000,
      seed=39),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_decode_parity(w, cuda_device):
    t = W.generate(w)
    res = run_gpu(w, t)
    rep = check_step(w, t, res)
    print(w.name, rep)


def test_decode_zero_vectors(cuda_device):
    """Decode scoring: a zero query and zero keys have cosine 0 (no NaN anywhere)."""
    w = C("dec_zeros", h_q=8, h_kv=2, head_dim=128, chunk=1, prefix=700, nq=1, budget=64, seed=40)
    t = W.generate(w)
    q = t.q.clone()
    q[0, 3, 0] = 0
    k = t.k_cache.clone()
    k[:, 10:20] = 0
    t2 = W.Tensors(q, k, t.v_cache, t.kv_off)
    res = run_gpu(w, t2)
    assert np.isfinite(res["pooled"][0, :, :700]).all()
    assert (res["pooled"][0, :, 10:20] == 0).all()
    check_step(w, t2, res)


# 32 (sequence, KV head) rows with short prefixes: the one-CTA-per-row top-k
MANY_ROWS = [
    C("rows32_tc", h_q=16, h_kv=4, head_dim=128, chunk=64,
      prefix=(0, 50, 700, 3000, 5000, 100, 12000, 2047), nq=8,
      budget=(16, 64, 100, 600, 1, 50, 2000, 2047), recipe="rank4", seed=41),
    C("rows64_decode_f32", h_q=8, h_kv=8, head_dim=64, chunk=1,
      prefix=(900, 33, 4000, 128, 2500, 640, 7, 1000), nq=1,
      budget=(128, 64, 512, 100, 300, 64, 0, 999), dtype="f32", seed=42),
]


@pytest.mark.parametrize("w", MANY_ROWS, ids=lambda w: w.name)
def test_block_topk_rows(w, cuda_device):
    t = W.generate(w)
    res = run_gpu(w, t)
    rep = check_step(w, t, res)
    print(w.name, rep)


def test_block_topk_exact_ties(cuda_device):
    """Keys of every sequence drawn from 5 distinct rows, so pooled scores tie exactly and
    the one-CTA top-k must keep the lowest indices of each tied class."""
    n_seq, P, B = 16, 640, 100
    w = C("ties_rows32", h_q=4, h_kv=2, head_dim=128, chunk=1, prefix=(P,) * n_seq, nq=1,
          budget=B, seed=43)
    t = W.generate(w)
    g = torch.Generator().manual_seed(7)
    k = t.k_cache.clone()
    picks = []
    for b in range(n_seq):
        krows = torch.randn(2, 5, 128, generator=g).to(torch.bfloat16)
        pick = torch.randint(0, 5, (P,), generator=g)
        lo = t.kv_off[b]
        k[:, lo:lo + P] = krows[:, pick]
        picks.append(pick.numpy())
    t2 = W.Tensors(t.q, k.contiguous(), t.v_cache, t.kv_off)
    res = run_gpu(w, t2)
    check_step(w, t2, res)
    for b in range(n_seq):
        for gg in range(w.h_kv):
            sel = res["idx"][b, gg, :B]
            kept = set(int(x) for x in sel)
            for c in np.unique(picks[b]):
                members = np.flatnonzero(picks[b] == c)
                flags = [int(m) in kept for m in members]
                n = sum(flags)
                assert flags == [True] * n + [False] * (len(flags) - n), (b, gg, c)
