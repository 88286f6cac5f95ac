"""Whole-prompt chunked prefill (QUOKA page, Figure 1(a)) through quoka_prefill.

Three checks per case:
  1. composition: every chunk's output is bit-identical to quoka_select +
     sparse_chunk_attn called by hand after appending the chunk's rows, and the cache
     holds the prompt's K/V rows bit-exact afterwards, with every other row untouched;
  2. parity: each chunk's selection matches the oracle's (near-ties aside) and its
     output matches the oracle's attention over that selection;
  3. a budget covering every prefix key reproduces the oracle's whole-prompt loop
     (plain causal attention) directly.
"""
import numpy as np
import pytest
import torch

from oracle import quoka_oracle as O
from query_oriented_sparse_b200 import binding as Bd
from query_oriented_sparse_b200 import workloads as W

from parity_util import (ATTN_TOL, check_index_row, compare_kept_set, compare_top_set,
                         row_rel_err, stratified_rows)

pytestmark = pytest.mark.gpu

SLACK = (37, 5, 0, 64)     # extra cache rows after each sequence's prompt (never written)

CASES = [
    # (workload, per-chunk budgets)
    (W.custom("pf_bf16_d128", h_q=8, h_kv=2, head_dim=128, chunk=256, prefix=(0, 0), nq=32,
              budget=256, recipe="rank4", seed=21, prompt_chunks=4), (0, 64, 200, 256)),
    (W.custom("pf_bf16_d64_g8_ragged", h_q=8, h_kv=1, head_dim=64, chunk=200, prefix=0, nq=24,
              budget=400, recipe="heavy", seed=22, prompt_chunks=3), (50, 100, 400)),
    (W.custom("pf_f32_d64", h_q=4, h_kv=1, head_dim=64, chunk=128, prefix=0, nq=16,
              budget=128, dtype="f32", seed=23, prompt_chunks=4), (128, 128, 128, 128)),
    (W.custom("pf_f32_d128_b2", h_q=4, h_kv=2, head_dim=128, chunk=70, prefix=(0, 0), nq=12,
              budget=30, dtype="f32", seed=24, prompt_chunks=3), (0, 30, 0)),
]


def prompt_tensors(w, t):
    """Chunk-major prompt tensors: q [n, batch, h_q, C, d], k/v [n, batch, h_kv, C, d]."""
    n, C, d = w.prompt_chunks, w.chunk, w.head_dim
    q = t.q.view(w.batch, w.h_q, n, C, d).permute(2, 0, 1, 3, 4).contiguous()

    def rows(cache):
        per_seq = [cache[:, t.kv_off[b]:t.kv_off[b] + n * C].reshape(w.h_kv, n, C, d)
                   for b in range(w.batch)]
        return torch.stack(per_seq, dim=0).permute(2, 0, 1, 3, 4).contiguous()
    return q, rows(t.k_cache), rows(t.v_cache)


def bits(x):
    return x.view(torch.int16 if x.element_size() == 2 else torch.int32)


def slack_cache(w, seed):
    """A cache with slack rows after each prompt, filled with seeded junk."""
    n_rows = [w.prompt_chunks * w.chunk + SLACK[b % len(SLACK)] for b in range(w.batch)]
    kv_off = [0]
    for r in n_rows:
        kv_off.append(kv_off[-1] + r)
    g = torch.Generator(device="cpu").manual_seed(seed)
    k = torch.randn(w.h_kv, kv_off[-1], w.head_dim, generator=g).to(w.torch_dtype)
    v = torch.randn(w.h_kv, kv_off[-1], w.head_dim, generator=g).to(w.torch_dtype)
    return k, v, kv_off


def run_prefill(w, budgets, q, kn, vn, k0, v0, kv_off, dev):
    k = k0.to(dev)
    v = v0.to(dev)
    b_max = max(max(budgets), 1)
    idx = torch.full((w.batch, w.h_kv, b_max), -7, dtype=torch.int32, device=dev)
    out = torch.full_like(q, float("nan"), device=dev)
    shape = Bd.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.chunk, w.torch_dtype)
    n_ws = Bd.prefill_workspace_size(shape, w.prompt_chunks, w.nq, b_max)
    assert n_ws > 0
    ws = torch.full((n_ws,), 0xFF, dtype=torch.uint8, device=dev)
    Bd.quoka_prefill(q.to(dev), kn.to(dev), vn.to(dev), k, v, kv_off, w.nq, budgets, idx,
                     out=out, workspace=ws)
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    return out.cpu(), k.cpu(), v.cpu()


def run_by_hand(w, budgets, q, kn, vn, k0, v0, kv_off, dev):
    """The same prompt chunk by chunk through the two single-chunk calls."""
    k = k0.to(dev)
    v = v0.to(dev)
    b_max = max(max(budgets), 1)
    C = w.chunk
    outs, idxs, kepts = [], [], []
    for c in range(w.prompt_chunks):
        P = c * C
        for b in range(w.batch):
            k[:, kv_off[b] + P:kv_off[b] + P + C] = kn[c, b].to(dev)
            v[:, kv_off[b] + P:kv_off[b] + P + C] = vn[c, b].to(dev)
        qc = q[c].to(dev)
        prefix = [P] * w.batch
        budget = [budgets[c]] * w.batch
        idx = torch.full((w.batch, w.h_kv, b_max), -1, dtype=torch.int32, device=dev)
        kept = torch.full((w.batch, w.h_q, w.nq), -1, dtype=torch.int32, device=dev)
        if P > 0 and budgets[c] > 0:
            Bd.quoka_select(qc, k, kv_off, prefix, w.nq, budget, b_max, idx_out=idx,
                            kept_out=kept)
        outs.append(Bd.sparse_chunk_attn(qc, k, v, kv_off, prefix, budget, idx).cpu())
        idxs.append(idx.cpu().numpy())
        kepts.append(kept.cpu().numpy())
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    return torch.stack(outs), idxs, kepts


def check_chunk(w, c, budget, q, kn, vn, out_c, idx_c, kept_c, attn_rows=None):
    """Oracle parity of chunk c of the prompt: the GPU's kept queries and selected keys
    against the oracle's (near-ties counted and returned), then its output against the
    oracle's attention over the GPU's selection (every row, or with attn_rows="tiles"
    one row of every query tile of every KV head plus the last tile's first and last
    position of every head)."""
    C = w.chunk
    P = c * C
    nk = min(w.nq, C)
    tol = ATTN_TOL[w.dtype]
    near = 0
    rng = np.random.default_rng(77 + c)
    for b in range(w.batch):
        qc = q[c, b].to(torch.float64).numpy()
        kp = kn[:c + 1, b].permute(1, 0, 2, 3).reshape(w.h_kv, P + C, -1)
        vp = vn[:c + 1, b].permute(1, 0, 2, 3).reshape(w.h_kv, P + C, -1)
        kp, vp = kp.to(torch.float64).numpy(), vp.to(torch.float64).numpy()
        gpu_idx = [np.zeros(0, dtype=np.int64) for _ in range(w.h_kv)]
        if P > 0 and budget > 0:
            gpu_kept = []
            for h in range(w.h_q):
                head = kept_c[b, h][:nk].astype(np.int64)
                near += compare_kept_set(head, O.query_cosines(qc[h]), w.nq)
                gpu_kept.append(head)
            sel = O.select_chunk(qc, kp[:, :P], P, w.nq, budget, kept_override=gpu_kept)
            for g in range(w.h_kv):
                head = check_index_row(idx_c[b, g], min(budget, P), P)
                near += compare_top_set(head, sel["score"][g], budget)
                gpu_idx[g] = head
        if attn_rows is None:
            o_ref = O.attend_chunk(qc, kp, vp, P, gpu_idx)
            e = row_rel_err(out_c[b].float().numpy(), o_ref)
        else:
            assert attn_rows == "tiles", attn_rows
            rows = stratified_rows(w.h_q, w.h_kv, C, rng)
            o_ref = O.attend_chunk(qc, kp, vp, P, gpu_idx, rows=rows)
            e = row_rel_err(np.stack([out_c[b, h, t].float().numpy() for h, t in rows]), o_ref)
        assert e <= tol, f"chunk {c} sequence {b}: rel err {e} > {tol}"
    return near


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_prefill_composition_and_parity(case, cuda_device):
    w, budgets = case
    t = W.generate(w)
    q, kn, vn = prompt_tensors(w, t)
    k0, v0, kv_off = slack_cache(w, seed=w.seed + 1000)
    out, k_after, v_after = run_prefill(w, budgets, q, kn, vn, k0, v0, kv_off, cuda_device)
    ref_out, idxs, kepts = run_by_hand(w, budgets, q, kn, vn, k0, v0, kv_off, cuda_device)

    # 1. composition: bit-identical outputs, prompt rows appended, the rest untouched
    assert torch.equal(bits(out), bits(ref_out))
    n, C = w.prompt_chunks, w.chunk
    written = torch.zeros(k0.shape[1], dtype=torch.bool)
    for b in range(w.batch):
        lo = kv_off[b]
        written[lo:lo + n * C] = True
        expect_k = kn[:, b].permute(1, 0, 2, 3).reshape(w.h_kv, n * C, w.head_dim)
        expect_v = vn[:, b].permute(1, 0, 2, 3).reshape(w.h_kv, n * C, w.head_dim)
        assert torch.equal(k_after[:, lo:lo + n * C], expect_k)
        assert torch.equal(v_after[:, lo:lo + n * C], expect_v)
    assert torch.equal(k_after[:, ~written], k0[:, ~written])
    assert torch.equal(v_after[:, ~written], v0[:, ~written])

    # 2. parity of every chunk with the oracle
    near = sum(check_chunk(w, c, budgets[c], q, kn, vn, out[c], idxs[c], kepts[c])
               for c in range(n))
    print(w.name, "near-ties", near)


def test_prefill_full_budget_is_causal(cuda_device):
    """Budget >= every prefix: the prefill equals the oracle's whole-prompt loop."""
    w = W.custom("pf_full", h_q=8, h_kv=2, head_dim=128, chunk=128, prefix=0, nq=16,
                 budget=384, seed=25, prompt_chunks=4)
    budgets = (384,) * 4
    t = W.generate(w)
    q, kn, vn = prompt_tensors(w, t)
    k0, v0, kv_off = slack_cache(w, seed=26)
    out, _, _ = run_prefill(w, budgets, q, kn, vn, k0, v0, kv_off, cuda_device)
    n, C = w.prompt_chunks, w.chunk
    ref = O.prefill_prompt(t.q[0], t.k_cache[:, :n * C], t.v_cache[:, :n * C], C, w.nq, budgets)
    got = out[:, 0].permute(1, 0, 2, 3).reshape(w.h_q, n * C, -1).float().numpy()
    e = row_rel_err(got, ref["out"])
    assert e <= ATTN_TOL[w.dtype], e


def test_prefill_rejections_launch_nothing(cuda_device):
    w = W.custom("pf_rej", h_q=4, h_kv=2, head_dim=128, chunk=64, prefix=0, nq=8, budget=64,
                 seed=27, prompt_chunks=2)
    t = W.generate(w)
    q, kn, vn = prompt_tensors(w, t)
    dev = cuda_device
    k = t.k_cache.to(dev)
    v = t.v_cache.to(dev)
    idx = torch.zeros((1, 2, 64), dtype=torch.int32, device=dev)
    qd, knd, vnd = q.to(dev), kn.to(dev), vn.to(dev)
    out = torch.full_like(qd, 3.0)
    cases = [
        dict(kv_off=t.kv_off, budgets=(0, 65)),                       # budget > b_max
        dict(kv_off=(0, 100), budgets=(0, 64)),                       # cache rows < prompt
        dict(kv_off=t.kv_off, budgets=(0, -1)),                       # negative budget
    ]
    for cse in cases:
        with pytest.raises(Bd.QuokaError) as ex:
            Bd.quoka_prefill(qd, knd, vnd, k, v, cse["kv_off"], w.nq, cse["budgets"], idx,
                             out=out)
        assert ex.value.status == Bd.QUOKA_ERR_INVALID_ARG
    with pytest.raises(Bd.QuokaError):
        Bd.quoka_prefill(qd, knd, vnd, k, v, t.kv_off, w.nq, (0, 64), idx, out=qd)   # aliasing
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    with pytest.raises(Bd.QuokaError) as ex:
        Bd.quoka_prefill(qd, knd, vnd, k, v, t.kv_off, w.nq, (0, 64), idx, out=out, workspace=ws)
    assert ex.value.status == Bd.QUOKA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    assert torch.equal(k.cpu(), t.k_cache)


def test_prefill_full_size_prompt(cuda_device):
    """The 128K-context prompt (33 chunks of 4096) as the prefill benchmark runs it:
    every chunk bit-identical to the single-chunk calls, the cache filled with the
    prompt, and oracle parity of the second and the last chunk (one attention row of
    every query tile)."""
    w = W.PROMPTS["prompt_128k"]
    budgets = w.budgets_of_chunks()
    t = W.generate(w)
    dev = cuda_device
    n, C = w.prompt_chunks, w.chunk
    q, kn, vn = prompt_tensors(w, t)
    qd, knd, vnd = q.to(dev), kn.to(dev), vn.to(dev)
    b_max = max(budgets)
    k = torch.zeros_like(t.k_cache, device=dev)
    v = torch.zeros_like(t.v_cache, device=dev)
    idx = torch.empty((1, w.h_kv, b_max), dtype=torch.int32, device=dev)
    out = torch.empty_like(qd)
    Bd.quoka_prefill(qd, knd, vnd, k, v, t.kv_off, w.nq, budgets, idx, out=out)
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    assert torch.equal(k.cpu(), t.k_cache) and torch.equal(v.cpu(), t.v_cache)
    # by hand, over a second cache
    k2 = torch.zeros_like(k)
    v2 = torch.zeros_like(v)
    kept_of, idx_of = {}, {}
    for c in range(n):
        P = c * C
        k2[:, P:P + C] = knd[c, 0]
        v2[:, P:P + C] = vnd[c, 0]
        idx2 = torch.full_like(idx, -1)
        kept = torch.full((1, w.h_q, w.nq), -1, dtype=torch.int32, device=dev)
        if P > 0 and budgets[c] > 0:
            Bd.quoka_select(qd[c], k2, t.kv_off, [P], w.nq, [budgets[c]], b_max, idx_out=idx2,
                            kept_out=kept)
        o = Bd.sparse_chunk_attn(qd[c], k2, v2, t.kv_off, [P], [budgets[c]], idx2)
        assert torch.equal(bits(o), bits(out[c])), f"chunk {c} differs from the single-chunk calls"
        if c in (1, n - 1):
            kept_of[c] = kept.cpu().numpy()
            idx_of[c] = idx2.cpu().numpy()
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    out_h = {c: out[c].cpu() for c in kept_of}
    del qd, knd, vnd, k, v, k2, v2, out
    for c in kept_of:
        near = check_chunk(w, c, budgets[c], q, kn, vn, out_h[c], idx_of[c], kept_of[c],
                           attn_rows="tiles")
        print("prompt_128k chunk", c, "near-ties", near)
