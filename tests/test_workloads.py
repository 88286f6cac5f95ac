"""The seeded input generators (no method arithmetic): determinism and structure."""
import torch

from query_oriented_sparse_b200 import workloads as W


def test_generate_is_deterministic_and_shaped():
    w = W.custom("gen", h_q=4, h_kv=2, head_dim=64, chunk=16, prefix=(40, 0), nq=4, budget=8,
                 recipe="heavy", seed=3)
    a, b = W.generate(w), W.generate(w)
    assert torch.equal(a.q, b.q) and torch.equal(a.k_cache, b.k_cache)
    assert a.q.shape == (2, 4, 16, 64) and a.k_cache.shape == (2, 40 + 16 + 16, 64)
    assert a.kv_off == (0, 56, 72)


def test_prompt_budgets():
    w = W.PROMPTS["prompt_128k"]
    bud = w.budgets_of_chunks()
    assert len(bud) == w.prompt_chunks == 33
    assert bud[0] == 0 and bud[-1] == 16384 == W.WORKLOADS["ctx_128k"].budget[0]
    assert w.seq_rows() == (33 * 4096,)


def test_per_query_selection_locality():
    x = W.per_query_selection(5, 2, 64, 1000, 32, group=16, shared=0.75)
    assert x.shape == (2, 64, 32) and x.dtype == torch.int32
    rows = x.reshape(-1, 32)
    assert all(len(set(r.tolist())) == 32 for r in rows)
    assert bool((rows[:, 1:] > rows[:, :-1]).all()) and int(x.min()) >= 0 and int(x.max()) < 1000
    assert torch.equal(x, W.per_query_selection(5, 2, 64, 1000, 32, group=16, shared=0.75))

    def overlap(a, b):
        return len(set(a.tolist()) & set(b.tolist()))
    near = sum(overlap(x[0, t], x[0, t + 1]) for t in range(0, 15))
    far = sum(overlap(x[0, t], x[0, t + 16]) for t in range(0, 15))
    assert near > 10 * 15 and far < 4 * 15


def test_per_query_selection_large_locality():
    x = W.per_query_selection_large(3, 2, 64, 5000, 64, group=16, shared=0.75)
    assert x.shape == (2, 64, 64) and x.dtype == torch.int32
    assert bool((x[..., 1:] >= x[..., :-1]).all()) and int(x.min()) >= 0 and int(x.max()) < 5000
    near = len(set(x[0, 0].tolist()) & set(x[0, 1].tolist()))
    far = len(set(x[0, 0].tolist()) & set(x[0, 40].tolist()))
    assert near > 30 and far < 8


def test_per_query_selection_large_causal():
    """With causal_prefix = P, query t only draws rows 0 .. P + t."""
    P, T = 300, 40
    x = W.per_query_selection_large(4, 3, T, P + T, 50, group=16, shared=0.75, causal_prefix=P)
    assert bool((x[..., 1:] >= x[..., :-1]).all()) and int(x.min()) >= 0
    lim = P + torch.arange(T, dtype=torch.int32)
    assert bool((x.max(dim=-1).values <= lim[None]).all())
    assert bool((x[:, T - 1] > P).any())          # late queries do reach chunk rows
