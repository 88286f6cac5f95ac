"""Pins of the fp64 oracle against things other than itself.

Every check here is either a closed form (2-D vectors given by angles, where cosines
are cos of angle differences), an invariant the cosine-based method must have, a
brute-force enumeration on tiny inputs, an independent library routine
(torch scaled_dot_product_attention in fp64 with an explicit mask), or a figure the
QUOKA page prints (tests/golden).  The mutation tests at the end plant plausible
mistakes in the oracle and check that some pin catches each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import quoka_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def vecs(deg, norms=None):
    th = np.deg2rad(np.asarray(deg, dtype=np.float64))
    v = np.stack([np.cos(th), np.sin(th)], axis=1)
    if norms is not None:
        v = v * np.asarray(norms, dtype=np.float64)[:, None]
    return v


# ----------------------------------------------------------------------------------
# pin helpers (plain functions so the mutation tests can re-run them)
# ----------------------------------------------------------------------------------

def pin_query_cosine_closed_form(seed=0):
    """2-D queries rho_t (cos th_t, sin th_t): the mean of unit queries has angle
    phi = atan2(mean sin th, mean cos th), so cos(q_t, m) = cos(th_t - phi),
    whatever the (positive) norms rho_t are."""
    rng = np.random.default_rng(seed)
    for C in (3, 7, 16):
        th = rng.uniform(-np.pi, np.pi, C)
        rho = rng.uniform(0.05, 20.0, C)
        q = np.stack([rho * np.cos(th), rho * np.sin(th)], axis=1)
        phi = math.atan2(np.mean(np.sin(th)), np.mean(np.cos(th)))
        expect = np.cos(th - phi)
        np.testing.assert_allclose(O.query_cosines(q), expect, rtol=0, atol=1e-12)


def brute_force_keep_smallest(c, n):
    """Smallest-index tuple S (|S| = n) with max_{S} c <= min_{not S} c."""
    C = len(c)
    if n >= C:
        return tuple(range(C))
    for S in itertools.combinations(range(C), n):      # lexicographic order
        rest = [t for t in range(C) if t not in S]
        if max(c[t] for t in S) <= min(c[t] for t in rest):
            return S
    raise AssertionError("no valid subset")


def pin_subselect_brute_force(seed=1):
    """Kept sets equal brute-force enumeration, using closed-form cosines."""
    rng = np.random.default_rng(seed)
    for trial in range(60):
        C = int(rng.integers(2, 9))
        nq = int(rng.integers(1, 5))
        if trial % 3 == 0:
            # exact ties: repeated angles with power-of-two norms give bitwise-equal
            # unit vectors, hence exactly equal cosines
            base = rng.choice([0.0, 90.0, 180.0, 270.0, 45.0], size=C)
            rho = 2.0 ** rng.integers(-2, 3, C)
        else:
            base = rng.uniform(-180, 180, C)
            rho = rng.uniform(0.1, 5.0, C)
        q = vecs(base, rho)
        th = np.deg2rad(base)
        phi = math.atan2(np.mean(np.sin(th)), np.mean(np.cos(th)))
        c = O.query_cosines(q)
        # closed form agrees to rounding; ties in the closed form are ties in c too
        np.testing.assert_allclose(c, np.cos(th - phi), atol=1e-12)
        got = tuple(O.subselect_queries(q, nq).tolist())
        assert got == brute_force_keep_smallest(c, nq), (base, rho, nq, c)


def pin_query_scale_invariance(seed=2):
    """Scaling any single query by a positive constant leaves the kept set unchanged."""
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(32, 16))
    base = O.subselect_queries(q, 8)
    for _ in range(5):
        alpha = np.exp(rng.uniform(-3, 3, size=(32, 1)))
        assert np.array_equal(O.subselect_queries(q * alpha, 8), base)


def pin_scoring_closed_forms():
    """Pooled scores on 2-D angle examples: cos(q, k) = cos(th_q - th_k)."""
    kdeg = np.array([0.0, 30.0, 90.0, 135.0, 200.0, 300.0])
    k = vecs(kdeg, [2.0, 0.5, 1.0, 3.0, 1.5, 0.25])
    # G = 1, Nq = 1: score = cos(th_q - th_k)
    s = O.pooled_key_scores([vecs([60.0])], k)
    np.testing.assert_allclose(s, np.cos(np.deg2rad(60.0 - kdeg)), atol=1e-12)
    # G = 1, Nq = 3: max over the kept queries
    qd = np.array([10.0, 100.0, 250.0])
    s = O.pooled_key_scores([vecs(qd)], k)
    exp = np.max(np.cos(np.deg2rad(qd[:, None] - kdeg[None, :])), axis=0)
    np.testing.assert_allclose(s, exp, atol=1e-12)
    # G = 3, Nq = 1: mean over the heads
    s = O.pooled_key_scores([vecs([d]) for d in qd], k)
    exp = np.mean(np.cos(np.deg2rad(qd[:, None] - kdeg[None, :])), axis=0)
    np.testing.assert_allclose(s, exp, atol=1e-12)
    # zero key scores 0
    s = O.pooled_key_scores([vecs([0.0])], np.zeros((1, 2)))
    assert s[0] == 0.0


def pin_key_scale_and_permutation(seed=3):
    """Scaling a key by beta > 0 leaves its score unchanged; permuting keys permutes scores."""
    rng = np.random.default_rng(seed)
    units = [O.unit_rows(rng.normal(size=(5, 8)))[1] for _ in range(3)]
    k = rng.normal(size=(40, 8))
    s = O.pooled_key_scores(units, k)
    beta = np.exp(rng.uniform(-4, 4, size=(40, 1)))
    np.testing.assert_allclose(O.pooled_key_scores(units, k * beta), s, rtol=1e-13, atol=1e-15)
    perm = rng.permutation(40)
    np.testing.assert_allclose(O.pooled_key_scores(units, k[perm]), s[perm], rtol=0, atol=0)


def brute_force_top(score, B):
    P = len(score)
    if B >= P:
        return tuple(range(P))
    for S in itertools.combinations(range(P), B):
        rest = [j for j in range(P) if j not in S]
        if min(score[j] for j in S) >= max(score[j] for j in rest):
            return S
    raise AssertionError


def pin_top_budget_brute_force(seed=4):
    rng = np.random.default_rng(seed)
    for trial in range(80):
        P = int(rng.integers(1, 11))
        B = int(rng.integers(1, 7))
        if trial % 2:
            score = rng.integers(-2, 3, P).astype(np.float64)      # many ties
        else:
            score = rng.normal(size=P)
        got = tuple(O.top_budget(score, B).tolist())
        assert got == brute_force_top(score, B), (score, B)


def pin_worked_example():
    """Hand-derived 2-D example (H_q = 2, H_kv = 1, C = 4, Nq = 2, P = 3).

    head 0 queries (2,0),(0,1),(1,0),(0,-3): unit mean (0.5, 0) -> cosines 1,0,1,0;
      the two smallest tie at 0 -> kept {1, 3} (units (0,1), (0,-1)).
    head 1 queries (1,1),(-2,2),(4,4),(0.5,0.5): unit mean direction (0.5, 1)/|.|,
      cosines 3/sqrt(10) for the (1,1) rows and 1/sqrt(10) for (-1,1)
      -> kept {1} plus the lowest-index tie {0}: {0, 1} (units a=(1,1)/r2, b=(-1,1)/r2).
    keys k0=(2,0), k1=(0,1), k2=(0,-1):
      k0: head0 max(0, 0) = 0;    head1 max(1/r2, -1/r2) = 1/r2  -> (0 + 1/r2)/2
      k1: head0 max(1, -1) = 1;   head1 max(1/r2, 1/r2) = 1/r2   -> (1 + 1/r2)/2
      k2: head0 max(-1, 1) = 1;   head1 max(-1/r2, -1/r2) = -1/r2 -> (1 - 1/r2)/2
    budget 2 keeps {0, 1}; budget 1 keeps {1}.
    (A max over all kept queries of the group would give 1/r2, 1, 1 and keep {1, 2};
    mean-then-max would give 1/(2 r2), 1, 1/2 and keep {1, 2}.)
    """
    q = np.zeros((2, 4, 2))
    q[0] = [[2, 0], [0, 1], [1, 0], [0, -3]]
    q[1] = [[1, 1], [-2, 2], [4, 4], [0.5, 0.5]]
    k = np.zeros((1, 3 + 4, 2))
    k[0, :3] = [[2, 0], [0, 1], [0, -1]]
    r2 = math.sqrt(2.0)
    res = O.select_chunk(q, k, 3, 2, 2)
    assert [x.tolist() for x in res["kept"]] == [[1, 3], [0, 1]]
    np.testing.assert_allclose(res["cos"][0], [1, 0, 1, 0], atol=1e-15)
    np.testing.assert_allclose(res["cos"][1], [3 / math.sqrt(10), 1 / math.sqrt(10)] +
                               [3 / math.sqrt(10)] * 2, atol=1e-15)
    np.testing.assert_allclose(res["score"][0], [(0 + 1 / r2) / 2, (1 + 1 / r2) / 2,
                                                 (1 - 1 / r2) / 2], atol=1e-15)
    assert res["idx"][0].tolist() == [0, 1]
    assert O.select_chunk(q, k, 3, 2, 1)["idx"][0].tolist() == [1]


def sdpa_reference(q, k_seq, v_seq, P, sel):
    """Masked dense attention with torch's fp64 SDPA: query t of head h sees the
    selected prefix keys of its KV head and chunk keys P..P+t."""
    H_q, C, d = q.shape
    H_kv = k_seq.shape[0]
    G = H_q // H_kv
    n = P + C
    out = torch.zeros(H_q, C, d, dtype=torch.float64)
    for h in range(H_q):
        g = h // G
        mask = torch.zeros(C, n, dtype=torch.bool)
        mask[:, torch.as_tensor(sel[g], dtype=torch.long)] = True
        for t in range(C):
            mask[t, P:P + t + 1] = True
        qh = torch.as_tensor(q[h])[None, None]
        kh = torch.as_tensor(k_seq[g, :n])[None, None]
        vh = torch.as_tensor(v_seq[g, :n])[None, None]
        out[h] = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask[None, None])[0, 0]
    return out.numpy()


def pin_attention_vs_sdpa(seed=5):
    rng = np.random.default_rng(seed)
    for (H_q, H_kv, C, P, d, B) in [(4, 2, 5, 7, 8, 100), (4, 2, 5, 7, 8, 3),
                                    (3, 1, 6, 0, 4, 2), (6, 3, 4, 9, 16, 1),
                                    (2, 2, 1, 5, 8, 2)]:
        q = rng.normal(size=(H_q, C, d))
        k = rng.normal(size=(H_kv, P + C, d)) * 2.0
        v = rng.normal(size=(H_kv, P + C, d))
        sel = [np.sort(rng.choice(P, size=min(B, P), replace=False)) for _ in range(H_kv)]
        got = O.attend_chunk(q, k, v, P, sel)
        np.testing.assert_allclose(got, sdpa_reference(q, k, v, P, sel), rtol=1e-12, atol=1e-13)
        rows = [(H_q - 1, C - 1), (0, 0)]
        np.testing.assert_allclose(O.attend_chunk(q, k, v, P, sel, rows=rows),
                                   got[[r[0] for r in rows], [r[1] for r in rows]], atol=0)


def pin_full_budget_is_full_causal(seed=6):
    """B >= P: the whole pipeline equals full causal attention over prefix + chunk."""
    rng = np.random.default_rng(seed)
    H_q, H_kv, C, P, d = 4, 2, 6, 9, 8
    q = rng.normal(size=(H_q, C, d))
    k = rng.normal(size=(H_kv, P + C, d))
    v = rng.normal(size=(H_kv, P + C, d))
    res = O.select_chunk(q, k, P, 3, P + 5)
    assert all(x.tolist() == list(range(P)) for x in res["idx"])
    o = O.attend_chunk(q, k, v, P, res["idx"])
    full = np.zeros_like(o)
    for h in range(H_q):
        g = h // (H_q // H_kv)
        qh = torch.as_tensor(q[h])[None, None]
        kh = torch.as_tensor(k[g])[None, None]
        vh = torch.as_tensor(v[g])[None, None]
        mask = torch.ones(C, P + C, dtype=torch.bool).tril(diagonal=P)
        full[h] = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask)[0, 0].numpy()
    np.testing.assert_allclose(o, full, rtol=1e-12, atol=1e-13)


def pin_gqa_is_independent_mqa(seed=7):
    """GQA with H_kv groups equals H_kv independent MQA problems (G = H_q each)."""
    rng = np.random.default_rng(seed)
    H_q, H_kv, C, P, d, nq, B = 6, 3, 8, 20, 8, 3, 5
    q = rng.normal(size=(H_q, C, d))
    k = rng.normal(size=(H_kv, P + C, d))
    v = rng.normal(size=(H_kv, P + C, d))
    full = O.select_chunk(q, k, P, nq, B)
    o = O.attend_chunk(q, k, v, P, full["idx"])
    G = H_q // H_kv
    for g in range(H_kv):
        sub = O.select_chunk(q[g * G:(g + 1) * G], k[g:g + 1], P, nq, B)
        assert sub["idx"][0].tolist() == full["idx"][g].tolist()
        np.testing.assert_allclose(sub["score"][0], full["score"][g], atol=0)
        og = O.attend_chunk(q[g * G:(g + 1) * G], k[g:g + 1], v[g:g + 1], P, sub["idx"])
        np.testing.assert_allclose(og, o[g * G:(g + 1) * G], atol=0)


def pin_decode_is_mean_cosine(seed=14):
    """A decode step (C = 1): the subselect keeps the one query, so a key's score is the
    mean over the group's heads of its cosine with each head's query (torch's
    cosine_similarity), the top-B follows that, and a key scaled by any positive factor
    keeps its score."""
    rng = np.random.default_rng(seed)
    H_q, H_kv, P, d, B = 8, 2, 40, 16, 7
    G = H_q // H_kv
    q = rng.normal(size=(H_q, 1, d))
    k = rng.normal(size=(H_kv, P + 1, d))
    res = O.select_chunk(q, k, P, 1, B)
    for g in range(H_kv):
        qg = torch.as_tensor(q[g * G:(g + 1) * G, 0])                  # [G, d]
        kg = torch.as_tensor(k[g, :P])                                 # [P, d]
        cos = F.cosine_similarity(qg[:, None, :], kg[None, :, :], dim=-1)
        expect = cos.mean(0).numpy()
        np.testing.assert_allclose(res["score"][g], expect, rtol=1e-12, atol=1e-14)
        top = np.sort(np.argsort(-expect, kind="stable")[:B])
        assert res["idx"][g].tolist() == top.tolist()
    k2 = k.copy()
    k2[:, :P] *= rng.uniform(0.1, 10.0, size=(H_kv, P, 1))
    res2 = O.select_chunk(q, k2, P, 1, B)
    np.testing.assert_allclose(res2["score"], res["score"], rtol=1e-12, atol=1e-14)


def pin_per_query_vs_sdpa(seed=15):
    """Per-query selections (the QUILT setting): each query over exactly its own keys
    equals torch SDPA with a per-query boolean mask; a shared set reduces to the chunk
    attention of step 6 with that set and no chunk keys visible."""
    rng = np.random.default_rng(seed)
    H_q, H_kv, T, N, d, S = 4, 2, 6, 30, 8, 5
    G = H_q // H_kv
    q = rng.normal(size=(H_q, T, d))
    k = rng.normal(size=(H_kv, N, d))
    v = rng.normal(size=(H_kv, N, d))
    sel = rng.integers(0, N, size=(H_q, T, S))
    sel[0, 0, 2:] = -1                                  # padding
    sel[1, 3, 1] = sel[1, 3, 0]                         # a duplicate counts once
    o = O.attend_per_query(q, k, v, sel)
    for h in range(H_q):
        mask = torch.zeros(T, N, dtype=torch.bool)
        for t in range(T):
            for j in sel[h, t]:
                if j >= 0:
                    mask[t, j] = True
        ref = F.scaled_dot_product_attention(
            torch.as_tensor(q[h])[None, None], torch.as_tensor(k[h // G])[None, None],
            torch.as_tensor(v[h // G])[None, None], attn_mask=mask)[0, 0].numpy()
        np.testing.assert_allclose(o[h], ref, rtol=1e-12, atol=1e-13)
    shared = np.sort(rng.choice(N - T, size=S, replace=False))
    sel2 = np.broadcast_to(shared, (H_q, 1, S)).copy()
    o2 = O.attend_per_query(q[:, :1], k, v, sel2)
    # step 6 with the prefix ending at the largest shared key: chunk position 0 attends to
    # the other shared keys (selected) plus its own row P, i.e. exactly the shared set
    P = int(shared[-1])
    o6 = O.attend_chunk(q[:, :1], k, v, P, [shared[:-1]] * H_kv)
    np.testing.assert_allclose(o2, o6, rtol=1e-12, atol=1e-13)


def _sdpa_masked(q, k, v, mask_of_head):
    """Library attention (fp64 torch SDPA) per query head with an explicit bool mask."""
    H_q, H_kv = q.shape[0], k.shape[0]
    G = H_q // H_kv
    out = np.zeros(q.shape)
    for h in range(H_q):
        g = h // G
        out[h] = F.scaled_dot_product_attention(
            torch.as_tensor(q[h])[None, None], torch.as_tensor(k[g])[None, None],
            torch.as_tensor(v[g])[None, None], attn_mask=mask_of_head(g))[0, 0].numpy()
    return out


def _prompt(seed, H_q=4, H_kv=2, C=5, n=4, d=8):
    rng = np.random.default_rng(seed)
    T = C * n
    return (rng.normal(size=(H_q, T, d)), rng.normal(size=(H_kv, T, d)),
            rng.normal(size=(H_kv, T, d)), C, n)


def pin_prefill_full_budget_is_causal(seed=11):
    """Figure 1(a) with a budget covering every prefix key: the chunk loop over the
    whole prompt equals plain causal attention over the prompt."""
    q, k, v, C, n = _prompt(seed)
    T = C * n
    res = O.prefill_prompt(q, k, v, C, 2, [T] * n)
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    np.testing.assert_allclose(res["out"], _sdpa_masked(q, k, v, lambda g: causal),
                               rtol=1e-12, atol=1e-13)


def pin_prefill_zero_budget_is_block_causal(seed=12):
    """Budget 0: every chunk attends only to itself, causally (block-diagonal mask)."""
    q, k, v, C, n = _prompt(seed)
    T = C * n
    res = O.prefill_prompt(q, k, v, C, 2, [0] * n)
    blk = torch.arange(T) // C
    mask = (blk[:, None] == blk[None, :]) & torch.ones(T, T, dtype=torch.bool).tril()
    np.testing.assert_allclose(res["out"], _sdpa_masked(q, k, v, lambda g: mask),
                               rtol=1e-12, atol=1e-13)


def pin_prefill_is_causal_over_chunks(seed=13):
    """A partial budget: chunk c keeps min(B_c, c*C) keys of rows written before it,
    its output is attention over exactly those keys plus its own causal keys, and
    nothing in later chunks (their queries, keys or values) changes it."""
    q, k, v, C, n = _prompt(seed)
    T = C * n
    budgets = [3, 2, 4, 7]
    res = O.prefill_prompt(q, k, v, C, 2, budgets)
    for c in range(n):
        P = c * C
        for sel in res["idx"][c]:
            assert sel.size == min(budgets[c], P)
            assert ((sel >= 0) & (sel < P)).all()
        def mask_of(g, c=c, P=P):
            m = torch.zeros(T, T, dtype=torch.bool)
            m[:, torch.as_tensor(res["idx"][c][g], dtype=torch.long)] = True
            m[:, P:P + C] = torch.ones(T, C, dtype=torch.bool).tril(diagonal=-P)[:, :]
            return m[P:P + C]
        ref = _sdpa_masked(q[:, P:P + C], k, v, mask_of)
        np.testing.assert_allclose(res["out"][:, P:P + C], ref, rtol=1e-12, atol=1e-13)
    rng = np.random.default_rng(seed + 100)
    cut = 2 * C                              # chunks 2 and 3 get new content
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for x in (q2, k2, v2):
        x[:, cut:] = rng.normal(size=x[:, cut:].shape)
    res2 = O.prefill_prompt(q2, k2, v2, C, 2, budgets)
    np.testing.assert_array_equal(res2["out"][:, :cut], res["out"][:, :cut])
    for c in range(2):
        for a, b in zip(res2["idx"][c], res["idx"][c]):
            assert a.tolist() == b.tolist()


def pin_batch_is_per_sequence(seed=16):
    """A ragged batch in one shared cache: sequence b owns rows kv_off[b] .. kv_off[b+1]-1
    (its prefix, its chunk rows at kv_off[b] + P_b + t, then rows nobody reads), and rows
    before kv_off[0] belong to no sequence.  select_batch / attend_batch must give, per
    sequence, what select_chunk / attend_chunk give on that sequence's own arrays, built
    apart before the cache is assembled; rewriting the unread rows or another sequence's
    rows changes nothing."""
    rng = np.random.default_rng(seed)
    H_q, H_kv, C, d, nq = 4, 2, 3, 6, 2
    prefix = [7, 0, 11]
    budget = [3, 2, 11]
    junk = [2, 4, 1]
    lead = 5
    q = rng.normal(size=(len(prefix), H_q, C, d))
    seq_k = [rng.normal(size=(H_kv, P + C, d)) for P in prefix]
    seq_v = [rng.normal(size=(H_kv, P + C, d)) for P in prefix]

    def assemble(fill):
        ks, vs, off = [fill((H_kv, lead, d))], [fill((H_kv, lead, d))], [lead]
        for b, P in enumerate(prefix):
            ks += [seq_k[b], fill((H_kv, junk[b], d))]
            vs += [seq_v[b], fill((H_kv, junk[b], d))]
            off.append(off[-1] + P + C + junk[b])
        return np.concatenate(ks, axis=1), np.concatenate(vs, axis=1), off

    k, v, kv_off = assemble(lambda shp: rng.normal(size=shp))
    sel = O.select_batch(q, k, kv_off, prefix, nq, budget)
    out = O.attend_batch(q, k, v, kv_off, prefix, [r["idx"] for r in sel])
    for b, P in enumerate(prefix):
        ref = O.select_chunk(q[b], seq_k[b], P, nq, budget[b])
        for g in range(H_kv):
            assert sel[b]["idx"][g].tolist() == ref["idx"][g].tolist(), (b, g)
            assert sel[b]["idx"][g].size == min(budget[b], P)
        np.testing.assert_array_equal(sel[b]["score"], ref["score"])
        np.testing.assert_array_equal(out[b], O.attend_chunk(q[b], seq_k[b], seq_v[b], P, ref["idx"]))
    # unread rows rewritten: nothing moves
    k2, v2, _ = assemble(lambda shp: 100.0 * rng.normal(size=shp))
    sel2 = O.select_batch(q, k2, kv_off, prefix, nq, budget)
    np.testing.assert_array_equal(O.attend_batch(q, k2, v2, kv_off, prefix,
                                                 [r["idx"] for r in sel2]), out)
    # another sequence's rows rewritten: sequences 0 and 1 keep their results
    k3, v3 = k.copy(), v.copy()
    k3[:, kv_off[2]:kv_off[3]] = rng.normal(size=k3[:, kv_off[2]:kv_off[3]].shape)
    v3[:, kv_off[2]:kv_off[3]] = rng.normal(size=v3[:, kv_off[2]:kv_off[3]].shape)
    sel3 = O.select_batch(q, k3, kv_off, prefix, nq, budget)
    out3 = O.attend_batch(q, k3, v3, kv_off, prefix, [r["idx"] for r in sel3])
    np.testing.assert_array_equal(out3[:2], out[:2])
    assert not np.array_equal(out3[2], out[2])


def pin_selected_value_slots(seed=17):
    """The selected-value cache's slot map: a hand-worked case, then on random cases the
    held set equals the selection, kept rows never move, the misses are exactly the
    selected rows not kept before and fill the freed slots in order, and slots past the
    live range are empty.  Attention over the rows in slot order equals attention over
    the ascending selection (the set, not the order, decides it)."""
    new, miss = O.selected_value_slots([5, 9, 2, -1], [2, 3, 9], 3)
    assert new == [3, 9, 2, -1] and miss == [3]
    new, miss = O.selected_value_slots([4, 4, 7, 1], [1, 4], 2)       # row 4 held twice
    assert new == [4, 1, -1, -1] and miss == [1]
    rng = np.random.default_rng(seed)
    for _ in range(200):
        P = int(rng.integers(1, 40))
        bm = int(rng.integers(1, 12))
        prev = [-1] * bm
        n0 = int(rng.integers(0, min(bm, P) + 1))
        prev[:n0] = rng.choice(P, size=n0, replace=False).tolist()
        n = int(rng.integers(0, min(bm, P) + 1))
        idx = np.sort(rng.choice(P, size=n, replace=False))
        new, miss = O.selected_value_slots(prev, idx, n)
        assert sorted(new[:n]) == sorted(idx.tolist()) and all(x == -1 for x in new[n:])
        live_prev = set(prev[:min(n0, n)])
        for s_ in range(n):
            if prev[s_] in set(idx.tolist()) and prev.index(prev[s_]) == s_:
                assert new[s_] == prev[s_]
        assert miss == sorted(set(idx.tolist()) - live_prev)
        freed = [s_ for s_ in range(n) if new[s_] != prev[s_]]
        assert [new[s_] for s_ in freed] == miss
    # attention is a function of the selected set: slot order changes nothing
    H_q, H_kv, C, P, d = 4, 2, 3, 12, 8
    q = rng.normal(size=(H_q, C, d))
    k = rng.normal(size=(H_kv, P + C, d))
    v = rng.normal(size=(H_kv, P + C, d))
    sel = [np.sort(rng.choice(P, size=5, replace=False)) for _ in range(H_kv)]
    shuffled = [rng.permutation(x) for x in sel]
    np.testing.assert_allclose(O.attend_chunk(q, k, v, P, shuffled), O.attend_chunk(q, k, v, P, sel),
                               rtol=1e-12, atol=1e-13)


ALL_PINS = [pin_query_cosine_closed_form, pin_subselect_brute_force, pin_query_scale_invariance,
            pin_scoring_closed_forms, pin_key_scale_and_permutation, pin_top_budget_brute_force,
            pin_worked_example, pin_attention_vs_sdpa, pin_full_budget_is_full_causal,
            pin_gqa_is_independent_mqa, pin_prefill_full_budget_is_causal,
            pin_prefill_zero_budget_is_block_causal, pin_prefill_is_causal_over_chunks,
            pin_decode_is_mean_cosine, pin_per_query_vs_sdpa, pin_batch_is_per_sequence,
            pin_selected_value_slots]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# ----------------------------------------------------------------------------------
# readings the pins depend on, and the page figures
# ----------------------------------------------------------------------------------

def test_raw_mean_reading_breaks_scale_invariance():
    """The unnormalised-mean reading is not scale-invariant per query: a query scaled
    up drags the raw mean toward itself and changes the kept set."""
    # unit queries at 0, 100 and 250 degrees: the unit mean points near 5 degrees, so
    # the 250-degree query is the least similar.  Scaling that query by 50 turns the
    # raw mean toward 250 degrees, and the 100-degree query becomes least similar.
    q = vecs([0.0, 100.0, 250.0])
    assert O.subselect_queries(q, 1, raw_mean=True).tolist() == [2]
    q2 = q.copy()
    q2[2] *= 50.0
    assert O.subselect_queries(q2, 1, raw_mean=True).tolist() == [1]
    assert O.subselect_queries(q2, 1).tolist() == O.subselect_queries(q, 1).tolist() == [2]


def test_nq_at_least_chunk_keeps_all():
    q = np.random.default_rng(8).normal(size=(5, 4))
    assert O.subselect_queries(q, 5).tolist() == [0, 1, 2, 3, 4]
    assert O.subselect_queries(q, 99).tolist() == [0, 1, 2, 3, 4]


def test_zero_query_and_zero_prefix():
    q = np.zeros((3, 4))
    assert O.query_cosines(q).tolist() == [0.0, 0.0, 0.0]
    assert O.subselect_queries(q, 2).tolist() == [0, 1]
    res = O.select_chunk(np.ones((2, 3, 4)), np.ones((1, 3, 4)), 0, 2, 4)
    assert res["idx"][0].size == 0 and res["score"].shape == (1, 0)


def test_figure1a_schedule():
    """Figure 1(a): 6 tokens in 3 chunks of 2.  Running the chunk loop with a budget
    covering every prefix key reproduces full causal attention over the prompt; with
    budget 1 chunk c attends to exactly 1 prefix key plus its causal chunk keys."""
    fx = json.load(open(os.path.join(GOLDEN, "figure1a_chunked_prefill.json")))
    n, c = fx["prompt_tokens"], fx["chunk_tokens"]
    assert fx["chunks"] * c == n
    prefixes = [i * c for i in range(fx["chunks"])]
    assert prefixes == fx["prefix_len_per_chunk"]
    rng = np.random.default_rng(9)
    H_q, H_kv, d = 2, 1, 4
    q = rng.normal(size=(H_q, n, d))
    k = rng.normal(size=(H_kv, n, d))
    v = rng.normal(size=(H_kv, n, d))
    mask = torch.ones(n, n, dtype=torch.bool).tril()
    full = np.stack([F.scaled_dot_product_attention(
        torch.as_tensor(q[h])[None, None], torch.as_tensor(k[0])[None, None],
        torch.as_tensor(v[0])[None, None], attn_mask=mask)[0, 0].numpy() for h in range(H_q)])
    out = np.zeros_like(full)
    for P in prefixes:
        qc = q[:, P:P + c]
        res = O.select_chunk(qc, k, P, 1, n)
        out[:, P:P + c] = O.attend_chunk(qc, k, v, P, res["idx"])
        res1 = O.select_chunk(qc, k, P, 1, 1)
        assert res1["idx"][0].size == min(1, P)
    np.testing.assert_allclose(out, full, rtol=1e-12, atol=1e-13)


def test_workload_budgets_match_kept_fraction():
    from query_oriented_sparse_b200 import workloads as W
    fx = json.load(open(os.path.join(GOLDEN, "kept_fraction.json")))
    for name in ("gqa_8k", "long_chunk", "ctx_128k", "ragged_8"):
        w = W.WORKLOADS[name]
        for p, b in zip(w.prefix, w.budget):
            assert abs(b / p - fx["kept_fraction"]) < 0.011, (name, p, b)


def test_small_workload_select_runs():
    """The oracle finishes the tiny MQA workload's four chunks in seconds."""
    from query_oriented_sparse_b200 import workloads as W
    w = W.WORKLOADS["tiny_mqa"]
    t = W.generate(w)
    for c, prefix in w.chunk_steps():
        qc = t.q_chunk(c, w.chunk)
        res = O.select_batch(qc, t.k_cache, t.kv_off, prefix, w.nq, w.budget)
        assert res[0]["idx"][0].size == min(w.budget[0], prefix[0])
        o = O.attend_batch(qc, t.k_cache, t.v_cache, t.kv_off, prefix, [r["idx"] for r in res])
        assert np.isfinite(o).all()


# ----------------------------------------------------------------------------------
# mutation tests: plant a plausible mistake in the oracle, expect a pin to fail
# ----------------------------------------------------------------------------------

def _mut_most_similar(mp):
    orig = O.query_cosines
    mp.setattr(O, "query_cosines", lambda q, raw_mean=False: -orig(q, raw_mean))


def _mut_raw_mean(mp):
    orig = O.mean_query
    mp.setattr(O, "mean_query", lambda q, raw=False: orig(q, raw=True))


def _mut_max_over_group(mp):
    orig = O.pooled_key_scores
    mp.setattr(O, "pooled_key_scores",
               lambda units, k, block=8192: orig([np.concatenate(units)], k, block))


def _mut_mean_then_max(mp):
    def bad(units, k, block=8192):
        k = np.asarray(k, dtype=np.float64)
        r = np.sqrt((k * k).sum(1))
        per_head = np.stack([(u @ k.T).mean(0) for u in units])
        return np.where(r > 0, per_head.max(0) / np.where(r > 0, r, 1), 0.0)
    mp.setattr(O, "pooled_key_scores", bad)


def _mut_no_key_norm(mp):
    orig = O.pooled_key_scores
    def bad(units, k, block=8192):
        k = np.asarray(k, dtype=np.float64)
        return orig(units, k, block) * np.sqrt((k * k).sum(1))
    mp.setattr(O, "pooled_key_scores", bad)


def _mut_ties_high_index(mp):
    def bad(score, budget):
        score = np.asarray(score, dtype=np.float64)
        P = score.shape[0]
        if budget >= P:
            return np.arange(P)
        order = np.lexsort((-np.arange(P), -score))
        return np.sort(order[:budget])
    mp.setattr(O, "top_budget", bad)


def _mut_no_softmax_scale(mp):
    orig = O.attend_chunk
    def bad(q, k, v, P, idx, rows=None):
        q = np.asarray(q, dtype=np.float64)
        return orig(q * math.sqrt(q.shape[-1]), k, v, P, idx, rows)
    mp.setattr(O, "attend_chunk", bad)


def _mut_causal_excludes_self(mp):
    orig = O.attend_chunk
    def bad(q, k, v, P, idx, rows=None):
        # shift the chunk keys by one row: query t then sees chunk keys P-1 .. P+t-1
        k = np.asarray(k, dtype=np.float64).copy()
        v = np.asarray(v, dtype=np.float64).copy()
        k[:, P:] = np.roll(k[:, P:], 1, axis=1)
        v[:, P:] = np.roll(v[:, P:], 1, axis=1)
        return orig(q, k, v, P, idx, rows)
    mp.setattr(O, "attend_chunk", bad)


def _mut_prefill_own_chunk_candidates(mp):
    """Chunk c's own rows also offered to the selection as prefix candidates."""
    def bad(q, k, v, chunk, nq, budgets):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        out = np.zeros_like(q)
        idx = []
        for c in range(q.shape[1] // chunk):
            P = c * chunk
            sel = O.select_chunk(q[:, P:P + chunk], k[:, :P + chunk], P + chunk, nq, budgets[c])
            out[:, P:P + chunk] = O.attend_chunk(q[:, P:P + chunk], k, v, P, sel["idx"])
            idx.append(sel["idx"])
        return {"out": out, "idx": idx}
    mp.setattr(O, "prefill_prompt", bad)


def _mut_prefill_budget_shift(mp):
    """Each chunk run with the previous chunk's budget."""
    orig = O.prefill_prompt
    mp.setattr(O, "prefill_prompt", lambda q, k, v, chunk, nq, budgets:
               orig(q, k, v, chunk, nq, [budgets[0]] + list(budgets[:-1])))


def _per_query_variant(dedupe: bool, drop_padding: bool):
    def bad(q, k, v, sel):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        sel = np.asarray(sel, dtype=np.int64)
        H_q, T, d = q.shape
        G = H_q // k.shape[0]
        out = np.zeros((H_q, T, d))
        for h in range(H_q):
            for t in range(T):
                keys = sel[h, t][sel[h, t] >= 0] if drop_padding else sel[h, t]
                keys = np.unique(keys) if dedupe else keys
                logits = (k[h // G, keys] @ q[h, t]) / np.sqrt(d)
                p = np.exp(logits - logits.max())
                out[h, t] = (p @ v[h // G, keys]) / p.sum()
        return out
    return bad


def _mut_per_query_counts_duplicates(mp):
    """A key listed twice in a query's set weighs twice."""
    mp.setattr(O, "attend_per_query", _per_query_variant(dedupe=False, drop_padding=True))


def _mut_per_query_reads_padding(mp):
    """Padding (-1) read as the last key row."""
    mp.setattr(O, "attend_per_query", _per_query_variant(dedupe=True, drop_padding=False))


def _mut_seq_rows_off_by_one(mp):
    """A sequence's rows taken one row late."""
    mp.setattr(O, "_seq_rows", lambda x, kv_off, b: x[:, kv_off[b] + 1:kv_off[b + 1] + 1])


def _mut_batch_budget_of_next_sequence(mp):
    """Each sequence selected with the next sequence's budget."""
    orig = O.select_batch
    mp.setattr(O, "select_batch", lambda q, k, kv_off, prefix, nq, budget:
               orig(q, k, kv_off, prefix, nq, list(budget[1:]) + list(budget[:1])))


def _mut_slots_misses_descending(mp):
    """Misses placed into the freed slots in descending row order."""
    orig = O.selected_value_slots
    def bad(prev, idx, n):
        new, miss = orig(prev, idx, n)
        freed = [s for s in range(n) if new[s] in miss]
        for s, r in zip(freed, sorted(miss, reverse=True)):
            new[s] = r
        return new, miss
    mp.setattr(O, "selected_value_slots", bad)


def _mut_slots_refetch_hits(mp):
    """Every selected row fetched again into ascending slots (hits not kept)."""
    def bad(prev, idx, n):
        rows = sorted(int(x) for x in list(idx)[:n])
        return rows + [-1] * (len(prev) - n), rows
    mp.setattr(O, "selected_value_slots", bad)


MUTANTS = [_mut_most_similar, _mut_raw_mean, _mut_max_over_group, _mut_mean_then_max,
           _mut_no_key_norm, _mut_ties_high_index, _mut_no_softmax_scale,
           _mut_causal_excludes_self, _mut_prefill_own_chunk_candidates,
           _mut_prefill_budget_shift, _mut_per_query_counts_duplicates,
           _mut_per_query_reads_padding, _mut_seq_rows_off_by_one,
           _mut_batch_budget_of_next_sequence, _mut_slots_misses_descending,
           _mut_slots_refetch_hits]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_pins_catch_mutant(mutant, monkeypatch):
    caught = []
    with monkeypatch.context() as mp:
        mutant(mp)
        for pin in ALL_PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
    assert caught, f"{mutant.__name__} passed every pin"
