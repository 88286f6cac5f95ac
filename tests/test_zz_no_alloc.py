"""quoka_select_noalloc: the selection call for callers that cannot allocate device
memory when they run it (a plugin inside a serving engine that reserved the GPU's
memory up front and offers no allocator, or a path that cannot afford the device
synchronisation of cudaMalloc/cudaFree).  It must give the same kept sets and
selected indices as quoka_select with a caller workspace, call after call, even
though every call reuses the library's one built-in scratch array.

This file is named so pytest collects it last."""
import numpy as np
import pytest
import torch

from query_oriented_sparse_b200 import binding as Bd
from query_oriented_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu

CALLS = [
    W.custom("noalloc_bf16", h_q=8, h_kv=2, head_dim=128, chunk=200, prefix=(1000, 333),
             nq=24, budget=(100, 64), recipe="rank4", seed=31),
    W.custom("noalloc_f32", h_q=4, h_kv=1, head_dim=64, chunk=96, prefix=700, nq=16,
             budget=128, dtype="f32", seed=32),
]


def _both(w):
    t = W.generate(w)
    q, k, v = t.q.cuda(), t.k_cache.cuda(), t.v_cache.cuda()
    b_max = max(w.budget)
    res = {}
    for name in ("workspace", "noalloc"):
        idx = torch.full((w.batch, w.h_kv, b_max), -9, dtype=torch.int32, device="cuda")
        kept = torch.full((w.batch, w.h_q, w.nq), -9, dtype=torch.int32, device="cuda")
        if name == "workspace":
            Bd.quoka_select(q, k, t.kv_off, w.prefix, w.nq, w.budget, b_max, idx_out=idx,
                            kept_out=kept)
        else:
            Bd.quoka_select_noalloc(q, k, t.kv_off, w.prefix, w.nq, w.budget, b_max,
                                    idx_out=idx, kept_out=kept)
        out = Bd.sparse_chunk_attn(q, k, v, t.kv_off, w.prefix, w.budget, idx)
        torch.cuda.synchronize()
        res[name] = (idx.cpu().numpy(), kept.cpu().numpy(), out.float().cpu().numpy())
    assert Bd.device_error() == 0
    return res


def test_noalloc_matches_workspace_call_twice(cuda_device):
    for w in CALLS:                      # two calls in a row, different shapes and dtypes
        r = _both(w)
        (i0, k0, o0), (i1, k1, o1) = r["workspace"], r["noalloc"]
        assert np.array_equal(i0, i1), f"{w.name}: selected indices differ"
        assert np.array_equal(k0, k1), f"{w.name}: kept queries differ"
        assert np.array_equal(o0, o1), f"{w.name}: attention over the selections differs"
        assert (i1[..., :1] >= 0).all()
