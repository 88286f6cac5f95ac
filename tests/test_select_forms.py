"""GPU parity of every launch form the selection picks per call: the query subselect's
cluster of 1, 2, 4 or 8 CTAs per query head (the fewest covering the chunk, doubled while
every head's cluster fits the SMs at once) and the top-k's one-CTA-per-row kernel or its
cluster of 16, 8 or 4 CTAs per row (halved while the rows' clusters overflow the SMs).
The shapes below land on each form on a 148-SM part; each step is checked whole against
the oracle (kept sets, pooled scores, index sets, every attention row)."""
import pytest

from query_oriented_sparse_b200 import workloads as W

from gpu_harness import check_step, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # top-k: 2 rows of 9000 keys -> 16-CTA clusters
    W.custom("topk_cs16", h_q=8, h_kv=2, head_dim=128, chunk=64, prefix=(9000,), nq=16,
             budget=(1100,), seed=801, recipe="rank4"),
    # 12 rows of up to 9000 keys -> 8-CTA clusters
    W.custom("topk_cs8", h_q=8, h_kv=4, head_dim=128, chunk=32, prefix=(9000, 8500, 8300), nq=8,
             budget=(1000, 900, 1100), seed=802, recipe="gauss"),
    # 20 rows of 9000 keys (a decode-shaped call, G * C = 16) -> 4-CTA clusters
    W.custom("topk_cs4", h_q=4, h_kv=4, head_dim=128, chunk=16, prefix=(9000,) * 5, nq=16,
             budget=(1000, 1200, 800, 1000, 1100), seed=803, recipe="heavy"),
    # 2 rows of 4000 keys -> one CTA per row
    W.custom("topk_block_few", h_q=8, h_kv=2, head_dim=64, chunk=64, prefix=(4000,), nq=16,
             budget=(600,), seed=804, recipe="rank4"),
    # one CTA per row with the kept queries in two column groups (16 heads x 64), one
    # sequence keeping every prefix key and one keeping none: the groups' partial scores
    # are summed before either early exit
    W.custom("topk_block_groups_edges", h_q=16, h_kv=1, head_dim=128, chunk=96, prefix=(600, 300),
             nq=64, budget=(700, 0), seed=809, recipe="rank4"),
    # subselect: 192 heads of 256 queries -> 1 CTA per head
    W.custom("qsub_cs1", h_q=64, h_kv=8, head_dim=128, chunk=256, prefix=(300, 200, 250), nq=32,
             budget=(64, 64, 64), seed=805, recipe="gauss"),
    # 96 heads of 1100 queries -> 2 CTAs per head
    W.custom("qsub_cs2", h_q=48, h_kv=8, head_dim=128, chunk=1100, prefix=(200, 150), nq=64,
             budget=(64, 64), seed=806, recipe="rank4"),
    # 40 heads of 3000 queries -> 4 CTAs per head
    W.custom("qsub_cs4", h_q=40, h_kv=8, head_dim=128, chunk=3000, prefix=(100,), nq=128,
             budget=(64,), seed=807, recipe="heavy"),
    # 8 heads of 512 queries -> 8 CTAs per head
    W.custom("qsub_cs8", h_q=8, h_kv=2, head_dim=64, chunk=512, prefix=(700,), nq=48,
             budget=(128,), seed=808, dtype="f32", recipe="gauss"),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_select_form_parity(w, cuda_device):
    t = W.generate(w)
    res = run_gpu(w, t)
    rep = check_step(w, t, res)
    print(w.name, rep)
