"""Host-side logic of bench.py that needs no GPU: the max-over-ranks timing reduction
on a world_size-2 gloo group, the reference arm's behaviour on ranks other than 0,
and the algorithmic bytes/FLOPs of the 128K-context step behind the roofline."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from query_oriented_sparse_b200 import workloads as W  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank times a different step; every rank must see the slowest one
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank], torch.device("cpu"))
        out_q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0]


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks([3, 4.5], torch.device("cpu")) == [3.0, 4.5]


def test_reference_arm_other_ranks_exit_quietly(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"gpus": 2, "steps": 1, "warmup": 0})()
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(args, W.WORKLOADS["gqa_8k"])
    assert rc == 0 and buf.getvalue() == ""


def test_stage_model_ctx_128k():
    """Algorithmic work of one 128K-context step: scoring 2*H_q*Nq*P*d flops over the
    whole prefix, attention 4*d*H_q*(C*B + C(C+1)/2) flops over selected + causal keys."""
    w = W.WORKLOADS["ctx_128k"]
    st = bench.stage_model(w)
    P, C, B, d = 131072, 4096, 16384, 128
    assert st["score"]["flops"] == 2.0 * 32 * 128 * P * d
    assert st["attn"]["flops"] == 4.0 * d * 32 * (C * B + C * (C + 1) / 2)
    assert st["score"]["bytes"] == 8 * P * d * 2 + 32 * 128 * d * 2
    assert st["attn"]["bytes"] == 2 * 32 * C * d * 2 + 2 * 8 * (B + C) * d * 2 + 8 * B * 4
    rl = bench.roofline_us(st, {"hbm_gbs": 6440.7, "bf16_tflops": 1687.0, "bf16_tflops_sustained": 1436.0})
    assert abs(rl["attn"] - 733.2) < 0.1 and abs(rl["score"] - 81.5) < 0.1
    assert abs(sum(rl.values()) - 820.2) < 0.1


def test_attn_traffic_is_pinned_to_workload():
    assert bench.attn_traffic(W.WORKLOADS["gqa_8k"]) is None
    t = bench.attn_traffic(W.WORKLOADS["ctx_128k"])
    # one ncu capture of the kernel on this workload: dram read 117.63 MB + write 19.44 MB
    assert t is None or abs(t - 137.07e6) < 1e5


def test_oracle_prompt_sample_extrapolates():
    """The prefill line's CPU baseline: a bounded oracle sample scaled to the prompt,
    within a small factor of running the whole oracle loop on a small prompt."""
    import time
    from oracle import quoka_oracle as O
    w = W.custom("pp", h_q=8, h_kv=2, head_dim=64, chunk=64, prefix=0, nq=8, budget=64, seed=1,
                 prompt_chunks=5, chunk_budget=(0, 8, 16, 24, 32))
    t = W.generate(w)
    r = bench.oracle_prompt_sample(w, t, rows=32)
    t0 = time.perf_counter()
    O.prefill_prompt(t.q[0], t.k_cache, t.v_cache, 64, 8, w.budgets_of_chunks())
    full = time.perf_counter() - t0
    assert 0.2 * full < r["ttft_s"] < 5.0 * full
    assert "chunk 4" in r["sample"]


def test_perq_union_rows_counts_distinct_per_tile():
    sel = W.per_query_selection_large(1, 8, 64, 3000, 32, group=16)
    u, flat = bench.perq_union_rows(sel, 2, 4)
    ref = sum(len(set(sel[4 * g:4 * g + 4, t0:t0 + 4].flatten().tolist()))
              for g in range(2) for t0 in range(0, 64, 4))
    assert u == ref and flat == 2 * 16 * 16 * 32


def test_kernel_table_per_launch_rooflines():
    """Per-kernel rows: mean time per launch, the stage's algorithmic work, its bound."""
    w = W.WORKLOADS["ctx_128k"]
    peaks = {"hbm_gbs": 6440.7, "bf16_tflops": 1687.0, "bf16_tflops_sustained": 1436.0}
    steps = [[("qsub_kernel", 0.026), ("score_tc_kernel", 0.150), ("topk_kernel", 0.020),
              ("compact_kv_kernel", 0.024), ("attn_tc2_kernel", 1.090)]] * 3
    tab = bench.kernel_table(w, steps, peaks)
    assert list(tab) == ["qsub_kernel", "score_tc_kernel", "topk_kernel", "compact_kv_kernel",
                         "attn_tc2_kernel"]
    a = tab["attn_tc2_kernel"]
    assert a["bound"] == "tensor" and abs(a["us"] - 1090.0) < 1e-6
    assert abs(a["roofline_us"] - 733.24) < 0.1 and abs(a["frac"] - 733.24 / 1090.0) < 1e-3
    sc = tab["score_tc_kernel"]
    assert sc["bound"] == "tensor" and abs(sc["roofline_us"] - 81.47) < 0.1
    tk = tab["topk_kernel"]
    assert tk["bound"] == "hbm"
    assert abs(tk["achieved"] - (8 * (131072 + 16384) * 4) / 20e-6 / 1e9) < 1e-6
    cp = tab["compact_kv_kernel"]
    assert abs(cp["achieved"] - 2 * 2 * 8 * (16384 + 4096) * 256 / 24e-6 / 1e9) < 1e-6
    # a kernel launched twice per step is reported per launch
    tab2 = bench.kernel_table(w, [[("qsub_kernel", 0.01), ("qsub_kernel", 0.03)]], peaks)
    assert abs(tab2["qsub_kernel"]["us"] - 20.0) < 1e-9 and tab2["qsub_kernel"]["launches_per_step"] == 2


def test_perq_tc_unions_counts_distinct_per_pair_tile():
    sel = W.per_query_selection_large(2, 2, 64, 4000, 24, group=16, causal_prefix=3900)
    u = bench.perq_tc_unions(sel, 8)
    ref = [len(set(sel[g, t0:t0 + 16].flatten().tolist())) for g in range(2) for t0 in range(0, 64, 16)]
    assert u == ref and len(u) == 8
