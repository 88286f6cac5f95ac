"""The per-kernel timing hook (quoka_profile_events) through the binding's KernelTimer:
every kernel of a chunk step is named in launch order, its times are real device
times, and timing changes no output."""
import pytest
import torch

from query_oriented_sparse_b200 import binding as Bd
from query_oriented_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["chunk", "decode", "f32"])
def test_kernel_timer_names_every_launch(kind, cuda_device):
    if kind == "chunk":
        w = W.custom("prof_chunk", h_q=8, h_kv=2, head_dim=128, chunk=256, prefix=9000, nq=32,
                     budget=1024, recipe="rank4", seed=91)
        expect = ["qsub_kernel", "score_tc_kernel", "topk_kernel", "compact_kv_kernel",
                  "attn_tc2_kernel"]
    elif kind == "decode":
        w = W.custom("prof_decode", h_q=8, h_kv=2, head_dim=128, chunk=1, prefix=[3000] * 20,
                     nq=1, budget=384, recipe="heavy", seed=92)
        expect = ["score_decode_tc_kernel", "topk_block_kernel", "attn_decode_kernel",
                  "attn_decode_combine_kernel"]
    else:
        w = W.custom("prof_f32", h_q=4, h_kv=1, head_dim=64, chunk=64, prefix=500, nq=8,
                     budget=64, dtype="f32", seed=93)
        expect = ["qsub_kernel", "score_simt_kernel", "topk_block_kernel", "attn_simt_kernel"]
    t = W.generate(w)
    dev = cuda_device
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    idx0 = Bd.quoka_select(q, k, t.kv_off, w.prefix, w.nq, w.budget)
    out0 = Bd.sparse_chunk_attn(q, k, v, t.kv_off, w.prefix, w.budget, idx0)
    with Bd.KernelTimer() as kt:
        idx = Bd.quoka_select(q, k, t.kv_off, w.prefix, w.nq, w.budget)
        out = Bd.sparse_chunk_attn(q, k, v, t.kv_off, w.prefix, w.budget, idx)
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    assert [n for n, _ in kt.times] == expect
    assert all(ms > 0 for _, ms in kt.times)
    assert torch.equal(idx, idx0) and torch.equal(out, out0)
    # the hook is off again: a further call records nothing
    Bd.quoka_select(q, k, t.kv_off, w.prefix, w.nq, w.budget)
    assert Bd.lib().quoka_profile_marks(None, 0) == 0
