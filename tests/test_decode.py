"""The decode shape: one new token per sequence (C = 1) or a short chunk, so that at
most 16 query rows share a KV head.  The attention then runs the split-K gather kernel
(selected rows read straight from the cache, partials merged per KV head) instead of the
compacted tensor-core path; these cases check it against the oracle on every row,
across many splits, ragged batches, both dtypes and head sizes, and the degenerate
cases (no prefix, budget 0, a chunk longer than one token)."""
import pytest

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
