"""GPU parity of both grid forms of the SM-pair attention (head_dim 128, bf16): one cluster
per (sequence, KV head, pair) tile, or, when there are more tiles than resident clusters
and they are short, the persistent form where each cluster walks the tile list with its
pipeline, barriers and TMEM kept across tiles.  The persistent cases below carry the
tile shapes its bookkeeping has to survive: one-block tiles (the odd-block softmax group
has nothing to do), odd block counts (the two S buffers' use counts drift apart across
tiles), sequences without prefix keys or with a zero budget, and consecutive tiles of
different sequences.  Every attention row is compared with the oracle."""
import pytest

from query_oriented_sparse_b200 import workloads as W

from gpu_harness import check_step, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # persistent: 8 sequences x 8 KV heads x 4 pairs = 256 tiles of 1-4 key blocks
    W.custom("attn_persist_short", h_q=32, h_kv=8, head_dim=128, chunk=256,
             prefix=(0, 130, 300, 57, 0, 260, 90, 400), nq=32,
             budget=(0, 64, 128, 0, 0, 200, 90, 256), seed=901, recipe="rank4"),
    # persistent: odd block counts and one-block tiles (G = 8: 16 positions per tile)
    W.custom("attn_persist_odd", h_q=32, h_kv=4, head_dim=128, chunk=200,
             prefix=(500, 1, 700, 333, 2000, 0), nq=16,
             budget=(129, 1, 255, 300, 383, 0), seed=902, recipe="heavy"),
    # one cluster per tile: few long tiles
    W.custom("attn_onecluster_long", h_q=8, h_kv=2, head_dim=128, chunk=128,
             prefix=(20000,), nq=32, budget=(16000,), seed=903, recipe="gauss"),
    # one cluster per tile: more tiles than clusters, but long ones
    W.custom("attn_onecluster_many", h_q=16, h_kv=8, head_dim=128, chunk=1024,
             prefix=(14000, 14500), nq=32, budget=(13000, 13500), seed=904, recipe="rank4"),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attention_form_parity(w, cuda_device):
    t = W.generate(w)
    res = run_gpu(w, t)
    rep = check_step(w, t, res)
    print(w.name, rep)
