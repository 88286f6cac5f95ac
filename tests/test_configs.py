"""GPU parity on the six full-size workloads, through the same calls bench.py times.

Selection is checked completely (every kept set, pooled score and index set, with
near-ties counted); attention is checked on every row for the two small workloads
and the decode step, and on the large ones on one row of every 128-row query tile of
every KV head (so every CTA of every SM pair), plus the first and last position of
every head in the last tile.
"""
import pytest

from query_oriented_sparse_b200 import workloads as W

from gpu_harness import check_step, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_workload_parity(name, cuda_device):
    w = W.WORKLOADS[name]
    t = W.generate(w)
    full_rows = name in ("tiny_mqa", "gqa_8k", "decode_32")
    for c, _ in w.chunk_steps():
        res = run_gpu(w, t, chunk_index=c)
        rep = check_step(w, t, res, chunk_index=c, attn_rows=None if full_rows else "tiles")
        print(name, "chunk", c, rep)
