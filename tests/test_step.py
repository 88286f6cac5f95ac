"""quoka_step: one chunk (or decode) step with the cache append inside the call.

Each case runs the step on a cache whose chunk rows hold junk, and checks that the
output and the selection are bit-identical to appending the rows by hand and calling
quoka_select and sparse_chunk_attn, that the chunk rows land in the cache bit-exact,
and that no other row changes.  Both paths are held to the oracle elsewhere; this pins
the composition on the tensor-core, CUDA-core and decode paths.
"""
import pytest
import torch

from query_oriented_sparse_b200 import binding as Bd
from query_oriented_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.custom
CASES = [
    C("step_bf16_d128_ragged", h_q=8, h_kv=2, head_dim=128, chunk=96, prefix=(0, 77, 1500),
      nq=12, budget=(10, 64, 200), recipe="heavy", seed=51),
    C("step_bf16_d64", h_q=16, h_kv=2, head_dim=64, chunk=256, prefix=4096, nq=32, budget=512,
      seed=52),
    C("step_f32_d64", h_q=4, h_kv=1, head_dim=64, chunk=128, prefix=384, nq=16, budget=128,
      dtype="f32", seed=53),
    C("step_decode_bf16", h_q=32, h_kv=8, head_dim=128, chunk=1, prefix=(5000, 300, 12000),
      nq=1, budget=(600, 64, 1500), recipe="heavy", seed=54),
    C("step_decode_f32_budget0", h_q=8, h_kv=2, head_dim=128, chunk=2, prefix=(700, 0), nq=2,
      budget=(0, 16), dtype="f32", seed=55),
]


def bits(x):
    return x.view(torch.int16 if x.element_size() == 2 else torch.int32)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_step_equals_append_then_calls(w, cuda_device):
    dev = cuda_device
    t = W.generate(w)
    q = t.q.to(dev)
    rows = [(t.kv_off[b] + w.prefix[b], t.kv_off[b] + w.prefix[b] + w.chunk)
            for b in range(w.batch)]
    kn = torch.stack([t.k_cache[:, a:e] for a, e in rows]).contiguous().to(dev)
    vn = torch.stack([t.v_cache[:, a:e] for a, e in rows]).contiguous().to(dev)
    g = torch.Generator().manual_seed(w.seed + 7)
    k0, v0 = t.k_cache.clone(), t.v_cache.clone()
    for a, e in rows:                                   # junk where the chunk goes
        k0[:, a:e] = torch.randn(k0[:, a:e].shape, generator=g).to(k0.dtype)
        v0[:, a:e] = torch.randn(v0[:, a:e].shape, generator=g).to(v0.dtype)
    b_max = max(max(w.budget), 1)

    k, v = k0.to(dev), v0.to(dev)
    idx = torch.full((w.batch, w.h_kv, b_max), -7, dtype=torch.int32, device=dev)
    out = Bd.quoka_step(q, kn, vn, k, v, t.kv_off, w.prefix, w.nq, w.budget, idx)
    torch.cuda.synchronize()
    assert Bd.device_error() == 0

    k2, v2 = k0.to(dev), v0.to(dev)
    for b, (a, e) in enumerate(rows):
        k2[:, a:e] = kn[b]
        v2[:, a:e] = vn[b]
    idx2 = torch.full_like(idx, -7)
    if any(min(bb, p) > 0 for bb, p in zip(w.budget, w.prefix)):
        Bd.quoka_select(q, k2, t.kv_off, w.prefix, w.nq, w.budget, b_max, idx_out=idx2)
    out2 = Bd.sparse_chunk_attn(q, k2, v2, t.kv_off, w.prefix, w.budget, idx2)
    torch.cuda.synchronize()
    assert Bd.device_error() == 0

    assert torch.equal(bits(out), bits(out2))
    assert torch.equal(idx, idx2)
    assert torch.equal(k.cpu(), t.k_cache) and torch.equal(v.cpu(), t.v_cache)


def test_step_rejections_launch_nothing(cuda_device):
    w = CASES[0]
    t = W.generate(w)
    dev = cuda_device
    q = t.q.to(dev)
    k, v = t.k_cache.to(dev), t.v_cache.to(dev)
    kn = torch.zeros(w.batch, w.h_kv, w.chunk, w.head_dim, dtype=q.dtype, device=dev)
    idx = torch.zeros(w.batch, w.h_kv, 200, dtype=torch.int32, device=dev)
    out = torch.full_like(q, 5.0)
    with pytest.raises(Bd.QuokaError) as ex:                         # budget > b_max
        Bd.quoka_step(q, kn, kn, k, v, t.kv_off, w.prefix, w.nq, (10, 64, 201), idx, out=out)
    assert ex.value.status == Bd.QUOKA_ERR_INVALID_ARG
    with pytest.raises(Bd.QuokaError) as ex:                         # rows past the sequence
        Bd.quoka_step(q, kn, kn, k, v, t.kv_off, (0, 77, 1600), w.nq, w.budget, idx, out=out)
    assert ex.value.status == Bd.QUOKA_ERR_INVALID_ARG
    with pytest.raises(Bd.QuokaError) as ex:                         # too small a workspace
        Bd.quoka_step(q, kn, kn, k, v, t.kv_off, w.prefix, w.nq, w.budget, idx, out=out,
                      workspace=torch.zeros(256, dtype=torch.uint8, device=dev))
    assert ex.value.status == Bd.QUOKA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 5.0).all())
    assert torch.equal(k.cpu(), t.k_cache)
