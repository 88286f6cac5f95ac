"""Throughput of one chunked-prefill step (QUOKA selection + sparse chunk attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --prefill [prompt_128k] [--steps K] [--warmup W]

A step is one pass of the whole hot path over one batch of synthetic input: the
select call (query subselect, cosine scoring + pooling, top-B) and the attention
call, through the C ABI.  Default workload: the 128K-context chunk (prefix 131072 +
chunk 4096, H_q 32, H_kv 8, d 128, Nq 128, B 16384, bf16).  Each timed step is
bracketed by CUDA events on the launching stream, with a 256 MB L2 flush before it
(outside the events).  Under torchrun every rank runs its own independent chunk step
(weak scaling, no collective on the data path) and the slowest rank's time is used.

`--prefill` instead times a whole prompt (33 chunks of the 128K-context shapes) through
the prefill call, which appends each chunk's K/V to the cache, selects and attends: the
attention path's time to first token, with a dense causal SDPA over the same prompt
beside it for context.

Rank 0 prints one JSON line.  `--impl reference` times the fp64 CPU oracle instead
(test infrastructure, run on the host cores on a bounded sample of the workload).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from query_oriented_sparse_b200 import workloads as W  # noqa: E402

METRIC = "chunked-prefill sparse-attn tokens/s (select+attend) and % of roofline, 1 B200"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024                       # B200 L2
def launches_per_step(w):
    """Kernels one step launches.  Selection: query subselect, scoring and top-k, or only
    scoring and top-k when every query is kept and G * C <= 16 (the decode shape).
    Attention: the gather kernel and its combine when G * C <= 16, else compaction and
    the tensor-core kernel (bf16) or the CUDA-core kernel alone (fp32)."""
    small = w.group * w.chunk <= 16
    sel = 2 if small and w.nq >= w.chunk else 3
    att = 2 if small or w.dtype == "bf16" else 1
    return sel + att
# DRAM traffic of one attention-kernel launch on the 128K-context workload
# (dram__bytes_read.sum + dram__bytes_write.sum from one ncu capture of that kernel alone,
# one launch, on this workload), valid only for the kernel sources it was taken on: the
# digest below covers them, and a changed kernel reports null.
ATTN_TRAFFIC = {"workload": "ctx_128k", "bytes": 117.633280e6 + 19.436032e6,
                "sources": ['query_oriented_sparse_b200/csrc/attn_tc2.cuh', 'query_oriented_sparse_b200/csrc/tc_ptx.cuh'], "sha256_16": "ab69040dc3da8c8a"}


def attn_traffic(w):
    import hashlib
    if w.name != ATTN_TRAFFIC["workload"]:
        return None
    h = hashlib.sha256()
    for f in ATTN_TRAFFIC["sources"]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return ATTN_TRAFFIC["bytes"] if h.hexdigest()[:16] == ATTN_TRAFFIC["sha256_16"] else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def stage_model(w: W.Workload):
    """Algorithmic bytes and FLOPs per stage for one chunk step (compulsory traffic:
    the selection reads every prefix key once; attention reads only the selected and
    causal keys; tile padding and the 4-byte pooled intermediate are not counted)."""
    s, d, C, nq = w.elem_bytes, w.head_dim, w.chunk, min(w.nq, w.chunk)
    st = {k: {"bytes": 0.0, "flops": 0.0} for k in ("qsub", "score", "topk", "attn")}
    for P, B in zip(w.prefix, w.budget):
        n = min(B, P)
        st["qsub"]["bytes"] += w.h_q * C * d * s + w.h_q * nq * d * s
        st["score"]["bytes"] += w.h_kv * P * d * s + w.h_q * nq * d * s
        st["score"]["flops"] += 2.0 * w.h_q * nq * P * d
        st["topk"]["bytes"] += w.h_kv * n * 4
        st["attn"]["bytes"] += (2 * w.h_q * C * d * s + 2 * w.h_kv * (n + C) * d * s +
                                w.h_kv * n * 4)
        st["attn"]["flops"] += 4.0 * d * w.h_q * (C * n + C * (C + 1) / 2)
    return st


KERNEL_STAGE = {"qsub_kernel": "qsub", "score_tc_kernel": "score", "score_simt_kernel": "score",
                "score_decode_kernel": "score", "score_decode_tc_kernel": "score",
                "topk_kernel": "topk", "topk_block_kernel": "topk",
                "attn_tc2_kernel": "attn", "attn_tc_kernel": "attn", "attn_simt_kernel": "attn",
                "attn_decode_kernel": "attn"}


def kernel_work(w, name):
    """Algorithmic (flops, bytes) of one launch of a kernel of the chunk step.

    The method's stages take their compulsory work (stage_model).  Two kernels move
    bytes the method itself does not need, and are held to the bytes they must move:
    top-k reads the pooled scores (4 B per key and column group) and writes idx, and
    the compaction reads and writes every selected and chunk K/V row once."""
    s, d, C = w.elem_bytes, w.head_dim, w.chunk
    st = stage_model(w)
    if name in ("topk_kernel", "topk_block_kernel"):
        return 0.0, sum(w.h_kv * (P * 4 + min(B, P) * 4) for P, B in zip(w.prefix, w.budget))
    if name == "compact_kv_kernel":
        return 0.0, sum(2 * 2 * w.h_kv * (min(B, P) + C) * d * s
                        for P, B in zip(w.prefix, w.budget))
    stage = KERNEL_STAGE.get(name)
    if stage is None:
        return 0.0, 0.0
    return st[stage]["flops"], st[stage]["bytes"]


def kernel_table(w, times, peaks):
    """Mean device time of each kernel over the profiled steps, with its roofline."""
    acc = {}
    for step in times:
        for name, ms in step:
            acc.setdefault(name, []).append(ms)
    out = {}
    for name, ms in acc.items():
        n_per_step = len(ms) / len(times)
        t = sum(ms) / len(times) / 1e3 / n_per_step        # per launch
        fl, by = kernel_work(w, name)
        t_fl = fl / (peaks["bf16_tflops"] * 1e12)
        t_by = by / (peaks["hbm_gbs"] * 1e9)
        row = {"us": t * 1e6, "launches_per_step": n_per_step}
        if fl or by:
            if t_fl >= t_by:
                row.update(bound="tensor", achieved=fl / t / 1e12, unit="TFLOP/s",
                           roofline_us=t_fl * 1e6, frac=t_fl / t)
            else:
                row.update(bound="hbm", achieved=by / t / 1e9, unit="GB/s",
                           roofline_us=t_by * 1e6, frac=t_by / t)
        out[name] = row
    return out


def attn_kernel_name(w):
    if w.group * w.chunk <= 16:
        return ("attn_decode_kernel (split-K gather from the cache) + its combine kernel, timed "
                "as the sparse_chunk_attn call")
    if w.dtype == "f32":
        return "attn_simt_kernel, timed as the sparse_chunk_attn call"
    if w.head_dim == 128:
        return ("attn_tc2_kernel (SM pairs), timed as the sparse_chunk_attn call (compaction + "
                "attention)")
    return "attn_tc_kernel, timed as the sparse_chunk_attn call (compaction + attention)"


def dominant_roofline(w, st, peaks, peak_src, sel_s, att_s):
    """The roofline object of the call that takes longer (attention on the prefill
    workloads, the selection on the decode step), each against the bound its own
    algorithmic bytes and FLOPs set."""
    if att_s >= sel_s:
        fl, by, t = st["attn"]["flops"], st["attn"]["bytes"], att_s
        kernel, traffic = attn_kernel_name(w), attn_traffic(w)
    else:
        fl = sum(st[k]["flops"] for k in ("qsub", "score", "topk"))
        by = sum(st[k]["bytes"] for k in ("qsub", "score", "topk"))
        t = sel_s
        kernel = ("score kernel with query subselect and top-k, timed as the quoka_select call "
                  "(three kernels)")
        traffic = None
    if fl / (peaks["bf16_tflops"] * 1e12) >= by / (peaks["hbm_gbs"] * 1e9):
        a = fl / t / 1e12
        return {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": a / peaks["bf16_tflops"], "traffic": traffic, "kernel": kernel,
                "peak_source": f"{peak_src} bf16 dense (burst)"}
    a = by / t / 1e9
    return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": a / peaks["hbm_gbs"], "traffic": traffic, "kernel": kernel,
            "peak_source": f"{peak_src} HBM copy"}


def roofline_us(st, peaks):
    out = {}
    for k, v in st.items():
        out[k] = max(v["flops"] / (peaks["bf16_tflops"] * 1e12),
                     v["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e6
    return out


class ClockSampler:
    """Samples the SM clock and the active clock-event (throttle) reasons while the timed
    region runs: NVML reads from a thread every millisecond (read-only queries), so even
    a region of a few milliseconds gets samples; nvidia-smi at 200 ms if NVML is absent."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.sm, self.reasons, self.max_mhz, self.source = [], set(), None, None
        self.stop = threading.Event()
        self.thread = self.proc = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def _poll(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                mask = int(get_reasons(h))
                for name, bit in self.REASONS:
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.source = "nvml 1 ms"
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.device_index), "-lms", "200"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi 200 ms"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for ln in self.proc.stdout:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                self.sm.append(float(parts[0]))
                self.max_mhz = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    self.reasons.add(n)

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.sm:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.sm), "source": self.source}


# --------------------------------------------------------------------------------------
# CPU oracle arm
# --------------------------------------------------------------------------------------

def oracle_sample(w: W.Workload, t: W.Tensors, rows: int = 64):
    """Times the fp64 oracle on a bounded sample of one chunk step: the complete
    selection of KV head 0 of sequence 0 plus attention for `rows` query rows of its
    group; extrapolates to the whole step (all KV heads and query rows, all sequences)."""
    from oracle import quoka_oracle as O
    b, g = 0, 0
    P, B = w.prefix[b], w.budget[b]
    lo, hi = t.kv_off[b], t.kv_off[b + 1]
    G = w.group
    q = t.q_chunk(0, w.chunk)[b, g * G:(g + 1) * G].double().numpy()
    k = t.k_cache[g:g + 1, lo:hi].double().numpy()
    v = t.v_cache[g:g + 1, lo:hi].double().numpy()
    t0 = time.perf_counter()
    res = O.select_chunk(q, k, P, w.nq, B)
    t_sel = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    rr = [(int(rng.integers(G)), int(rng.integers(w.chunk))) for _ in range(rows)]
    t0 = time.perf_counter()
    O.attend_chunk(q, k, v, P, res["idx"], rows=rr)
    t_att = time.perf_counter() - t0
    # the sampled sequence stands for the others in proportion to their prefix
    scale_sel = sum(w.prefix) / max(P, 1) if P else w.batch
    est = t_sel * w.h_kv * scale_sel + t_att / rows * (w.h_q * w.chunk * w.batch)
    return {"t_select_s": t_sel, "t_attn_s": t_att, "est_step_s": est,
            "tokens_per_s": w.batch * w.chunk / est,
            "sample": f"selection of KV head 0 of sequence 0 (P={P}) + attention for {rows} "
                      f"sampled query rows of its group; extrapolated to {w.h_kv} KV heads x "
                      f"{w.h_q * w.chunk * w.batch} query rows"}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    t = W.generate(w)
    samples = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(w, t)
        if i >= args.warmup:
            samples.append(r)
    v = statistics.median(s["tokens_per_s"] for s in samples)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.batch * w.chunk / v, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "chunk": w.chunk,
                   "prefix": list(w.prefix), "h_q": w.h_q, "h_kv": w.h_kv, "head_dim": w.head_dim,
                   "nq": w.nq, "budget": list(w.budget), "input_dtype": w.dtype},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": samples[0]["sample"]},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------------------

def max_over_ranks(vals, device):
    """Element-wise maximum of per-rank timings over the process group (the slowest
    rank sets the job's time); the values themselves on a single process."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in vals]
    m = torch.tensor([float(x) for x in vals], dtype=torch.float64, device=device)
    dist.all_reduce(m, op=dist.ReduceOp.MAX)
    return m.tolist()


def run_ours(args, w):
    from query_oriented_sparse_b200 import binding as Bd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    peaks, peak_src = load_peaks()

    t = W.generate(w)
    q = t.q.to(dev)
    k = t.k_cache.to(dev)
    v = t.v_cache.to(dev)
    shape = Bd.shape_of(q, k)
    b_max = max(w.budget)
    ws = torch.empty(Bd.select_workspace_size(shape, max(w.prefix), w.nq), dtype=torch.uint8,
                     device=dev)
    idx = torch.empty(w.batch, w.h_kv, b_max, dtype=torch.int32, device=dev)
    aws = torch.empty(max(Bd.attn_workspace_size(shape, b_max), 256), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def select():
        Bd.quoka_select(q, k, t.kv_off, w.prefix, w.nq, w.budget, b_max, idx_out=idx,
                        workspace=ws)

    def attend():
        Bd.sparse_chunk_attn(q, k, v, t.kv_off, w.prefix, w.budget, idx, out=out, workspace=aws)

    for _ in range(args.warmup):
        flush.zero_()
        select()
        attend()
    torch.cuda.synchronize()
    select_eager, attend_eager = select, attend
    # Each call is captured once into a CUDA graph and replayed every step, as a serving
    # loop runs a fixed-shape step: the kernels are the same, the host's per-call work
    # (argument checks, tensor maps, ctypes marshalling) leaves the step.
    launch_mode = "eager"
    if not args.eager:
        g_sel, g_att = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_sel, capture_error_mode="thread_local"):
            select()
        with torch.cuda.graph(g_att, capture_error_mode="thread_local"):
            attend()
        select, attend = g_sel.replay, g_att.replay
        launch_mode = "CUDA graph per call, captured once and replayed every step"
        for _ in range(2):
            flush.zero_()
            select()
            attend()
        torch.cuda.synchronize()
    assert Bd.device_error() == 0

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            e0, e1, e2 = ev[i]
            e0.record(stream)
            select()
            e1.record(stream)
            attend()
            e2.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sel_ms = [a.elapsed_time(b) for a, b, _ in ev]
    att_ms = [b.elapsed_time(c) for _, b, c in ev]
    step_ms = [a + b for a, b in zip(sel_ms, att_ms)]
    total_s = sum(step_ms) / 1e3
    assert Bd.device_error() == 0

    # per-kernel device times: the same two calls launched eagerly, an event recorded
    # after every kernel (outside the timed region above; same L2 flush before each step)
    ktimes = []
    for i in range(args.steps):
        flush.zero_()
        with Bd.KernelTimer(stream=stream) as kt:
            select_eager()
            attend_eager()
        ktimes.append(kt.times)
    assert Bd.device_error() == 0
    kernels = kernel_table(w, ktimes, peaks)

    # end to end through host buffers and the serving call (quoka_step): every step's new
    # inputs (Q and the chunk's own K/V rows, packed [batch, h_kv, C, d]) go host->device
    # from pinned memory, the call appends the K/V rows to the cache, selects and attends,
    # and the output comes back device->host.  Steps are pipelined as a server runs them:
    # step i+1's inputs are uploaded on one copy stream and step i's output is read back
    # on another while step i computes, with inputs and outputs double-buffered (the
    # cache is written only by the steps themselves, in stream order).  The timed region
    # runs from the first upload to the last read-back, so every step's copies are in it.
    C = w.chunk
    q_h = t.q.pin_memory()
    kv_rows = [(t.kv_off[b] + w.prefix[b], t.kv_off[b] + w.prefix[b] + C) for b in range(w.batch)]
    kn_h = torch.stack([t.k_cache[:, a:b_] for a, b_ in kv_rows]).contiguous().pin_memory()
    vn_h = torch.stack([t.v_cache[:, a:b_] for a, b_ in kv_rows]).contiguous().pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in (q_h, kn_h, vn_h))
    d2h = out_h[0].numel() * out_h[0].element_size()
    qb, ob = [q, q.clone()], [torch.empty_like(out), torch.empty_like(out)]
    knb = [torch.empty(kn_h.shape, dtype=kn_h.dtype, device=dev) for _ in range(2)]
    vnb = [torch.empty(vn_h.shape, dtype=vn_h.dtype, device=dev) for _ in range(2)]
    sws = torch.empty(Bd.step_workspace_size(shape, max(w.prefix), w.nq, b_max), dtype=torch.uint8,
                      device=dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of buffer b landed
    ev_cmp = [torch.cuda.Event() for _ in range(2)]     # the step on buffer b has finished
    ev_out = [torch.cuda.Event() for _ in range(2)]     # output of buffer b read back

    def make_step(b):
        def run():
            Bd.quoka_step(qb[b], knb[b], vnb[b], k, v, t.kv_off, w.prefix, w.nq, w.budget, idx,
                          out=ob[b], workspace=sws)
        return run

    step_on = [make_step(0), make_step(1)]
    # Between end-to-end steps the L2 is flushed inside the timed region unless the K/V
    # cache the steps read is larger than twice the L2 by itself (then no step finds the
    # previous one's keys in L2, and a flush would only add its own time).
    kv_bytes = 2 * k.numel() * k.element_size()
    e2e_flush = kv_bytes <= 2 * L2_BYTES
    for b in range(2):                     # fill both input buffers once, warm each call
        knb[b].copy_(kn_h)
        vnb[b].copy_(vn_h)
        step_on[b]()
    torch.cuda.synchronize()
    if not args.eager:
        g_step = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
        for b in range(2):
            with torch.cuda.graph(g_step[b], capture_error_mode="thread_local"):
                step_on[b]()
        step_on = [g.replay for g in g_step]

    def e2e_run(nsteps, timed):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(nsteps):
            b = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[b])
                if i == 0 and timed:
                    t0.record(s_in)
                qb[b].copy_(q_h, non_blocking=True)
                knb[b].copy_(kn_h, non_blocking=True)
                vnb[b].copy_(vn_h, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])
            if e2e_flush:
                flush.zero_()
            step_on[b]()
            ev_cmp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b])
                out_h[b].copy_(ob[b], non_blocking=True)
                ev_out[b].record(s_out)
        if timed:
            t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) if timed else 0.0

    e2e_run(max(2, args.warmup), False)
    e2e_total_ms = e2e_run(args.steps, True)
    last = (args.steps - 1) & 1
    # the serving call's output equals the two single calls' (timed above)
    assert torch.equal(out_h[last].to(dev), ob[last]) and torch.equal(ob[last], out)

    tokens = w.batch * C
    total_s, e2e_total_s = max_over_ranks([total_s, e2e_total_ms / 1e3], dev)
    value = world * args.steps * tokens / total_s
    e2e_value = world * args.steps * tokens / e2e_total_s

    st = stage_model(w)
    rl = roofline_us(st, peaks)
    path_roof_us = sum(rl.values())
    roof = dominant_roofline(w, st, peaks, peak_src, statistics.mean(sel_ms) / 1e3,
                             statistics.mean(att_ms) / 1e3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_s * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "chunk": C, "prefix": list(w.prefix),
                   "h_q": w.h_q, "h_kv": w.h_kv, "head_dim": w.head_dim, "nq": w.nq,
                   "budget": list(w.budget), "l2": "256 MB flush before every timed step",
                   "launch": launch_mode,
                   "parallelism": f"independent chunk step per GPU x{world}"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "l2": ("256 MB flush inside every end-to-end step" if e2e_flush else
                       f"no flush: the K/V cache ({kv_bytes / 1e6:.0f} MB) is over twice the L2")},
        "gpu_launches": launches_per_step(w) * args.steps,
        "stage_us": {"select": statistics.mean(sel_ms) * 1e3,
                     "attn": statistics.mean(att_ms) * 1e3},
        "kernel_us": {k: v["us"] for k, v in kernels.items()},
        "kernels": kernels,
        "roofline": roof,
        "path_roofline": {"roofline_us": path_roof_us, "stage_roofline_us": rl,
                          "measured_us": total_s * 1e6 / args.steps,
                          "frac": path_roof_us / (total_s * 1e6 / args.steps)},
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample(w, t)
        line["cpu_baseline"] = {"value": r["tokens_per_s"], "unit": UNIT, "cores": blas_threads(),
                                "kind": "oracle", "sample": r["sample"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


# --------------------------------------------------------------------------------------
# whole-prompt prefill (time to first token of the attention path)
# --------------------------------------------------------------------------------------

PREFILL_METRIC = "whole-prompt chunked prefill, attention-path time to first token, 1 B200"


def prompt_inputs(w, t, dev):
    """Chunk-major prompt tensors on the device: q [n, batch, h_q, C, d] and the
    prompt's own K/V rows k_new, v_new [n, batch, h_kv, C, d]."""
    n, C, d = w.prompt_chunks, w.chunk, w.head_dim
    q = t.q.view(w.batch, w.h_q, n, C, d).permute(2, 0, 1, 3, 4).contiguous().to(dev)

    def rows(cache):
        per_seq = [cache[:, t.kv_off[b]:t.kv_off[b] + n * C].reshape(w.h_kv, n, C, d)
                   for b in range(w.batch)]
        return torch.stack(per_seq, 0).permute(2, 0, 1, 3, 4).contiguous().to(dev)
    return q, rows(t.k_cache), rows(t.v_cache)


def prompt_stage_model(w):
    """stage_model summed over the prompt's chunk steps."""
    tot = None
    for c, budget in enumerate(w.budgets_of_chunks()):
        step = W.custom(h_q=w.h_q, h_kv=w.h_kv, head_dim=w.head_dim, chunk=w.chunk,
                        prefix=tuple(p + c * w.chunk for p in w.prefix), nq=w.nq,
                        budget=budget, dtype=w.dtype)
        st = stage_model(step)
        if c == 0 or budget == 0:                  # no selection runs on this chunk
            for k in ("qsub", "score", "topk"):
                st[k] = {"bytes": 0.0, "flops": 0.0}
        if tot is None:
            tot = st
        else:
            for k in tot:
                for m in tot[k]:
                    tot[k][m] += st[k][m]
    return tot


def dense_reference_ms(q, k_new, v_new, steps, flush):
    """Dense causal attention over the same prompt with torch's fused SDPA (library
    flash / memory-efficient / cuDNN kernels, never the materialising math path), for
    context next to the sparse prefill; None if no fused kernel takes the shape."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    import torch.nn.functional as F
    n, batch, h_q, C, d = q.shape
    qd = q.permute(1, 2, 0, 3, 4).reshape(batch, h_q, n * C, d)
    kd = k_new.permute(1, 2, 0, 3, 4).reshape(batch, k_new.shape[2], n * C, d)
    vd = v_new.permute(1, 2, 0, 3, 4).reshape(batch, v_new.shape[2], n * C, d)
    try:
        with sdpa_kernel([SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION,
                          SDPBackend.CUDNN_ATTENTION]):
            F.scaled_dot_product_attention(qd, kd, vd, is_causal=True, enable_gqa=True)
            torch.cuda.synchronize()
            ms = []
            for _ in range(steps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                F.scaled_dot_product_attention(qd, kd, vd, is_causal=True, enable_gqa=True)
                b.record()
                torch.cuda.synchronize()
                ms.append(a.elapsed_time(b))
        return statistics.median(ms)
    except RuntimeError as e:
        print(f"dense reference unavailable: {str(e).splitlines()[0]}", file=sys.stderr)
        return None


def oracle_prompt_sample(w, t, rows: int = 64):
    """Times the fp64 oracle on a bounded sample of the whole-prompt prefill: the last
    chunk's selection for KV head 0 plus attention for `rows` sampled query rows of that
    chunk; extrapolates selection by prefix length over the chunks that select (times the
    KV heads) and attention by keys per query row over every row of the prompt."""
    from oracle import quoka_oracle as O
    C, n, G = w.chunk, w.prompt_chunks, w.group
    budgets = w.budgets_of_chunks()
    c = n - 1
    P = c * C
    q = t.q[0, 0:G, P:P + C].double().numpy()
    k = t.k_cache[0:1, :P + C].double().numpy()
    v = t.v_cache[0:1, :P + C].double().numpy()
    t0 = time.perf_counter()
    res = O.select_chunk(q, k[:, :P], P, w.nq, budgets[c])
    t_sel = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    rr = [(int(rng.integers(G)), int(rng.integers(C))) for _ in range(rows)]
    t0 = time.perf_counter()
    O.attend_chunk(q, k, v, P, res["idx"], rows=rr)
    t_att = time.perf_counter() - t0
    sel_prefix = sum(cc * C for cc in range(1, n) if budgets[cc] > 0)
    keys_sample = sum(min(budgets[c], P) + tt + 1 for _, tt in rr) / rows
    keys_total = w.h_q * sum(C * min(budgets[cc], cc * C) + C * (C + 1) / 2 for cc in range(n))
    est = t_sel * w.h_kv * sel_prefix / P + t_att / rows / keys_sample * keys_total
    return {"ttft_s": est, "sample": f"chunk {c}'s selection for KV head 0 (P={P}) + attention "
                                     f"for {rows} sampled query rows of that chunk; extrapolated "
                                     f"to {n} chunks x {w.h_kv} KV heads x {w.h_q * C * n} query rows"}


def run_prefill(args, w):
    from query_oriented_sparse_b200 import binding as Bd

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--prefill times one prompt on one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks, peak_src = load_peaks()
    t = W.generate(w)
    q, kn, vn = prompt_inputs(w, t, dev)
    k = torch.zeros_like(t.k_cache, device=dev)
    v = torch.zeros_like(t.v_cache, device=dev)
    budgets = w.budgets_of_chunks()
    b_max = max(max(budgets), 1)
    shape = Bd.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.chunk, w.torch_dtype)
    ws = torch.empty(Bd.prefill_workspace_size(shape, w.prompt_chunks, w.nq, b_max),
                     dtype=torch.uint8, device=dev)
    idx = torch.empty(w.batch, w.h_kv, b_max, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def prompt():
        Bd.quoka_prefill(q, kn, vn, k, v, t.kv_off, w.nq, budgets, idx, out=out, workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        prompt()
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    ms = []
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            prompt()
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
    assert Bd.device_error() == 0
    ttft = statistics.median(ms)
    tokens = w.batch * w.chunk * w.prompt_chunks
    st = prompt_stage_model(w)
    rl = roofline_us(st, peaks)
    roof_ms = sum(rl.values()) / 1e3
    dense_ms = dense_reference_ms(q, kn, vn, max(1, min(args.steps, 3)), flush)
    n_sel = sum(1 for c, bgt in enumerate(budgets) if c > 0 and bgt > 0)
    att_tflops = st["attn"]["flops"] / (ttft / 1e3) / 1e12

    # End to end: the prompt lives in pinned host memory and goes through quoka_step chunk
    # by chunk, as a server streams it: chunk c+1's inputs are uploaded on one copy stream
    # and chunk c's output read back on another while chunk c computes (inputs and outputs
    # double-buffered).  Timed from the first upload to the last read-back.
    n, C = w.prompt_chunks, w.chunk
    q_h, kn_h, vn_h = q.cpu().pin_memory(), kn.cpu().pin_memory(), vn.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    qd = [torch.empty_like(q[0]) for _ in range(2)]
    knd = [torch.empty_like(kn[0]) for _ in range(2)]
    vnd = [torch.empty_like(vn[0]) for _ in range(2)]
    od = [torch.empty_like(out[0]) for _ in range(2)]
    sws = torch.empty(Bd.step_workspace_size(shape, (n - 1) * C, w.nq, b_max), dtype=torch.uint8,
                      device=dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_prompt():
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for c in range(n):
            bb = c & 1
            with torch.cuda.stream(s_in):
                if c >= 2:
                    s_in.wait_event(ev_cmp[bb])
                if c == 0:
                    t0.record(s_in)
                qd[bb].copy_(q_h[c], non_blocking=True)
                knd[bb].copy_(kn_h[c], non_blocking=True)
                vnd[bb].copy_(vn_h[c], non_blocking=True)
                ev_in[bb].record(s_in)
            stream.wait_event(ev_in[bb])
            if c >= 2:
                stream.wait_event(ev_out[bb])
            Bd.quoka_step(qd[bb], knd[bb], vnd[bb], k, v, t.kv_off, [c * C] * w.batch, w.nq,
                          [budgets[c]] * w.batch, idx, out=od[bb], workspace=sws)
            ev_cmp[bb].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[bb])
                out_h[c].copy_(od[bb], non_blocking=True)
                ev_out[bb].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_ms = []
    for i in range(1 + args.steps):
        flush.zero_()
        torch.cuda.synchronize()
        e = e2e_prompt()
        if i > 0:
            e2e_ms.append(e)
    assert Bd.device_error() == 0
    assert torch.equal(out_h, out.cpu()), "the streamed prompt differs from the prefill call"
    e2e_value = statistics.median(e2e_ms)
    cpu = oracle_prompt_sample(w, t) if not args.no_cpu_baseline else None
    line = {
        "metric": PREFILL_METRIC, "value": ttft, "unit": "ms", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ttft,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "chunk": w.chunk,
                   "chunks": w.prompt_chunks, "prompt_tokens": w.chunk * w.prompt_chunks,
                   "h_q": w.h_q, "h_kv": w.h_kv, "head_dim": w.head_dim, "nq": w.nq,
                   "budget_per_chunk": "c * chunk / 8",
                   "l2": "256 MB flush before every timed prompt"},
        "tokens_per_s": tokens / (ttft / 1e3),
        "e2e": {"value": e2e_value, "unit": "ms",
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in (q_h, kn_h, vn_h)),
                "d2h_bytes_per_step": out_h.numel() * out_h.element_size()},
        "gpu_launches": (2 * w.prompt_chunks + 3 * n_sel) * args.steps,
        "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": att_tflops / peaks["bf16_tflops"],
                     "traffic": None,
                     "kernel": "attn_tc2_kernel over the prompt's chunks, timed as the whole "
                               "prefill call (selection included, so this understates the "
                               "kernel's own rate)",
                     "peak_source": f"{peak_src} bf16 dense (burst)"},
        "path_roofline": {"roofline_ms": roof_ms, "frac": roof_ms / ttft,
                          "peak_source": f"{peak_src} bf16 dense (burst) and HBM copy"},
        "dense_sdpa_ms": dense_ms,
        "ttft_reduction_vs_dense": (dense_ms / ttft) if dense_ms else None,
        "clocks": clk.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = {"value": cpu["ttft_s"] * 1e3, "unit": "ms", "cores": blas_threads(),
                                "kind": "oracle", "sample": cpu["sample"]}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------
# per-query selections with shared loading
# --------------------------------------------------------------------------------------

PERQ_METRIC = "per-query sparse attention tokens/s (each query its own key set), 1 B200"
PERQ_S = 512               # keys per query
PERQ_GROUP = 16            # consecutive queries drawing from one base set


def perq_union_rows(sel, h_kv, tq):
    """Union size of every tile (G heads x tq positions of a KV head) and the rows the
    tiles would load without sharing; sel int32 [h_q, C, S] on the CPU."""
    h_q, C, S = sel.shape
    G = h_q // h_kv
    nt = C // tq
    x = sel[:, :nt * tq].reshape(h_kv, G, nt, tq, S).permute(0, 2, 1, 3, 4).reshape(h_kv * nt, -1)
    x = torch.sort(x.long(), dim=1).values
    distinct = 1 + (x[:, 1:] != x[:, :-1]).sum(dim=1)
    return int(distinct.sum()), int(x.shape[0] * x.shape[1])


def run_perq(args):
    from query_oriented_sparse_b200 import binding as Bd

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--perq runs on one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks, peak_src = load_peaks()
    w = W.WORKLOADS["ctx_128k"]
    t = W.generate(w)
    n_rows = t.kv_off[1]
    # causal sets: query t draws from the prefix and the chunk rows up to its own
    sel_h = W.per_query_selection_large(7, w.h_q, w.chunk, n_rows, PERQ_S, group=PERQ_GROUP,
                                        causal_prefix=w.prefix[0])
    tq = max(1, 16 // w.group)
    union_rows, flat_rows = perq_union_rows(sel_h, w.h_kv, tq)
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    sel = sel_h[None].contiguous().to(dev)
    shape = Bd.shape_of(q, k)
    ws = torch.empty(Bd.perq_workspace_size(shape, PERQ_S), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def call():
        Bd.sparse_perq_attn(q, k, v, t.kv_off, sel, out=out, workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    assert Bd.device_error() == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        call()
    stream = torch.cuda.current_stream()
    ms = []
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
    assert Bd.device_error() == 0
    t_ms = statistics.median(ms)
    tokens = w.chunk
    row = w.head_dim * 2
    # compulsory bytes: the index sets, Q and O, and each tile's union of K and V rows once
    by = sel.numel() * 4 + 2 * q.numel() * 2 + 2 * union_rows * row
    fl = 4.0 * w.head_dim * w.h_q * w.chunk * PERQ_S
    gbs = by / (t_ms / 1e3) / 1e9
    line = {
        "metric": PERQ_METRIC, "value": tokens / (t_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "perq_128k", "chunk": w.chunk, "cache_rows": n_rows,
                   "h_q": w.h_q, "h_kv": w.h_kv, "head_dim": w.head_dim, "keys_per_query": PERQ_S,
                   "causal": True,
                   "locality_group": PERQ_GROUP, "tile_rows": w.group * tq,
                   "l2": "256 MB flush before every timed call",
                   "launch": "CUDA graph, captured once and replayed every step"},
        "gpu_launches": 3 * args.steps,
        "union_rows": union_rows, "rows_without_sharing": flat_rows,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "perq_union_kernel + perq_attn_kernel + combine, timed as the call",
                     "peak_source": f"{peak_src} HBM copy", "flops": fl},
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------
# selected-value cache with miss-only fetch (decode steps with drifting queries)
# --------------------------------------------------------------------------------------

SELCACHE_METRIC = "decode steps over a selected-value cache with miss-only fetch, tokens/s, 1 B200"
SELCACHE_SIGMA = 0.3       # per-step query drift (workloads.drifting_queries)


def run_selcache(args):
    from query_oriented_sparse_b200 import binding as Bd

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--selcache runs on one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    base = W.WORKLOADS["decode_32"]
    n_steps = args.warmup + args.steps + 1
    w = W.custom("decode_32_drift", h_q=base.h_q, h_kv=base.h_kv, head_dim=base.head_dim, chunk=1,
                 prefix=base.prefix, nq=1, budget=base.budget, recipe=base.recipe, seed=base.seed,
                 prompt_chunks=n_steps)
    t = W.generate(w)
    qs = W.drifting_queries(base.seed + 100, t.q[:, :, 0], n_steps, SELCACHE_SIGMA).to(dev)
    k, v = t.k_cache.to(dev), t.v_cache.to(dev)
    b_max = max(w.budget)
    shape = Bd.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, 1, w.torch_dtype)
    ws = torch.empty(Bd.select_workspace_size(shape, max(w.prefix) + n_steps, w.nq),
                     dtype=torch.uint8, device=dev)
    aws = torch.empty(max(Bd.attn_workspace_size(shape, b_max), 256), dtype=torch.uint8, device=dev)
    idx = torch.empty(w.batch, w.h_kv, b_max, dtype=torch.int32, device=dev)
    out_p = torch.empty(w.batch, w.h_q, 1, w.head_dim, dtype=w.torch_dtype, device=dev)
    out_c = torch.empty_like(out_p)
    cache = Bd.SelCache(shape, b_max, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    row_bytes = w.head_dim * w.elem_bytes
    rec = {"plain_ms": [], "cache_ms": [], "misses": [], "selected": []}
    for s in range(n_steps):
        prefix = tuple(p + s for p in w.prefix)
        q = qs[s]
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        # plain: select, then the decode gather straight from the KV cache
        flush.zero_()
        ev[0].record(stream)
        Bd.quoka_select(q, k, t.kv_off, prefix, w.nq, w.budget, b_max, idx_out=idx, workspace=ws)
        Bd.sparse_chunk_attn(q, k, v, t.kv_off, prefix, w.budget, idx, out=out_p, workspace=aws)
        ev[1].record(stream)
        # cached: the same selection, the misses fetched into the cache, attention over it
        flush.zero_()
        ev[2].record(stream)
        Bd.quoka_select(q, k, t.kv_off, prefix, w.nq, w.budget, b_max, idx_out=idx, workspace=ws)
        misses = cache.update(k, v, t.kv_off, prefix, w.budget, idx)
        cache.attend(q, prefix, w.budget, out=out_c)
        ev[3].record(stream)
        torch.cuda.synchronize()
        if s > args.warmup:                   # step 0 fills the empty cache
            rec["plain_ms"].append(ev[0].elapsed_time(ev[1]))
            rec["cache_ms"].append(ev[2].elapsed_time(ev[3]))
            rec["misses"].append(int(misses.sum()))
            rec["selected"].append(sum(w.h_kv * min(bb, p) for bb, p in zip(w.budget, prefix)))
    assert Bd.device_error() == 0
    o_p, o_c = out_p.float(), out_c.float()
    err = float(((o_p - o_c).abs().amax(-1) / o_p.abs().amax(-1).clamp_min(1e-30)).max())
    assert err <= 2e-2, f"cached attention differs from the plain path: {err}"
    cache_ms = statistics.median(rec["cache_ms"])
    plain_ms = statistics.median(rec["plain_ms"])
    miss = sum(rec["misses"]) / max(sum(rec["selected"]), 1)
    fetched = statistics.mean(rec["misses"]) * 2 * row_bytes + w.batch * w.h_kv * 2 * row_bytes
    gathered = statistics.mean(rec["selected"]) * 2 * row_bytes
    line = {
        "metric": SELCACHE_METRIC, "value": w.batch / (cache_ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": cache_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": "decode_32_drift", "batch": w.batch, "h_q": w.h_q, "h_kv": w.h_kv,
                   "head_dim": w.head_dim, "prefix": "decode_32's, growing one row per step",
                   "budget": list(w.budget), "query_drift_sigma": SELCACHE_SIGMA,
                   "l2": "256 MB flush before every timed step of each arm",
                   "launch": "eager (the prefix grows every step)"},
        "gpu_launches": 11 * args.steps,    # 4 plain + 7 cached (select 2, update 2, attend 3)
        "plain_tokens_per_s": w.batch / (plain_ms / 1e3), "plain_ms_per_step": plain_ms,
        "miss_fraction": miss,
        "fetched_bytes_per_step": fetched,
        "plain_gathered_bytes_per_step": gathered,
        "max_rel_diff_vs_plain": err,
    }
    print(json.dumps(line), flush=True)
    return 0


PERQ_TC_S = 2048           # keys per query token
PERQ_TC_GROUP = 64         # consecutive tokens drawing from one base set
PERQ_TC_SHARED = 0.9       # fraction of a token's set taken from its run's base set


def perq_tc_unions(sel_kv, tp):
    """Union size of every pair tile (2 * tp consecutive tokens of a KV head) for token
    sets sel_kv int32 [h_kv, C, S] that every head of the group shares."""
    h_kv, C, S = sel_kv.shape
    out = []
    for g in range(h_kv):
        for t0 in range(0, C, 2 * tp):
            out.append(int(torch.unique(sel_kv[g, t0:t0 + 2 * tp]).numel()))
    return out


def run_perq_tc(args):
    from query_oriented_sparse_b200 import binding as Bd

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--perq-tc runs on one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks, peak_src = load_peaks()
    w = W.WORKLOADS["ctx_128k"]
    t = W.generate(w)
    n_rows = t.kv_off[1]
    G = w.group
    # one set per token and KV head, read by every query head of the group (causal)
    sel_kv = W.per_query_selection_large(11, w.h_kv, w.chunk, n_rows, PERQ_TC_S, group=PERQ_TC_GROUP,
                                         shared=PERQ_TC_SHARED, causal_prefix=w.prefix[0])
    tp = 128 // G
    unions = perq_tc_unions(sel_kv, tp)
    cap = (max(unions) + 127) // 128 * 128
    sel = sel_kv[:, None].expand(w.h_kv, G, w.chunk, PERQ_TC_S).reshape(1, w.h_q, w.chunk, PERQ_TC_S)
    sel = sel.contiguous().to(dev)
    q, k, v = t.q.to(dev), t.k_cache.to(dev), t.v_cache.to(dev)
    shape = Bd.shape_of(q, k)
    ws_tc = torch.empty(Bd.perq_tc_workspace_size(shape, PERQ_TC_S, cap), dtype=torch.uint8, device=dev)
    ws_cc = torch.empty(Bd.perq_workspace_size(shape, PERQ_TC_S), dtype=torch.uint8, device=dev)
    out_tc, out_cc = torch.empty_like(q), torch.empty_like(q)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call_tc():
        Bd.sparse_perq_attn_tc(q, k, v, t.kv_off, sel, cap, out=out_tc, workspace=ws_tc)

    def call_cc():
        Bd.sparse_perq_attn(q, k, v, t.kv_off, sel, out=out_cc, workspace=ws_cc)

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return statistics.median(ms)

    with ClockSampler(0) as clk:
        tc_ms = timed(call_tc)
    cc_ms = timed(call_cc)
    assert Bd.device_error() == 0
    o1, o2 = out_tc.float(), out_cc.float()
    diff = float(((o1 - o2).abs().amax(-1) / o2.abs().amax(-1).clamp_min(1e-30)).max())
    assert diff <= 2e-2, f"the two per-query forms differ: {diff}"
    with Bd.KernelTimer(stream=stream) as kt:
        call_tc()
    kernels = {name: ms * 1e3 for name, ms in kt.times}
    flops_union = 4.0 * w.head_dim * 256 * sum(unions)         # dense MMAs over each tile's union
    flops_useful = 4.0 * w.head_dim * w.h_q * w.chunk * PERQ_TC_S
    attn_us = kernels.get("attn_tc2_kernel", tc_ms * 1e3)
    a = flops_union / (attn_us / 1e6) / 1e12
    line = {
        "metric": "per-query sparse attention on tensor cores, tokens/s, 1 B200", "value": w.chunk / (tc_ms / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": tc_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "perq_tc_128k", "chunk": w.chunk, "cache_rows": n_rows, "h_q": w.h_q,
                   "h_kv": w.h_kv, "head_dim": w.head_dim, "keys_per_token": PERQ_TC_S,
                   "sets": "one per token and KV head, shared by the group's query heads",
                   "locality_group": PERQ_TC_GROUP, "shared_fraction": PERQ_TC_SHARED, "causal": True,
                   "pair_tile_rows": 256, "max_union": cap,
                   "l2": "256 MB flush before every timed call", "launch": "eager"},
        "gpu_launches": 3 * args.steps,
        "union_keys_per_tile": {"mean": statistics.mean(unions), "max": max(unions)},
        "cuda_core_form_ms": cc_ms, "speedup_vs_cuda_core_form": cc_ms / tc_ms,
        "kernel_us": kernels,
        "roofline": {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": a / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "attn_tc2_kernel (membership masks) over each pair tile's union",
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "flops_over_unions": flops_union, "flops_of_the_sets": flops_useful},
        "max_rel_diff_vs_cuda_core_form": diff,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=W.HEADLINE, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch every call from the host each step instead of replaying graphs")
    ap.add_argument("--prefill", nargs="?", const="prompt_128k", choices=sorted(W.PROMPTS),
                    help="time a whole prompt through the prefill call (time to first token)")
    ap.add_argument("--perq", action="store_true",
                    help="time per-query sparse attention with shared loading")
    ap.add_argument("--selcache", action="store_true",
                    help="time decode steps over a selected-value cache with miss-only fetch")
    ap.add_argument("--perq-tc", action="store_true",
                    help="time per-query attention on tensor cores over 256-row pair tiles")
    args = ap.parse_args()
    if args.perq_tc:
        if args.impl != "ours":
            raise SystemExit("--perq-tc has no reference arm")
        return run_perq_tc(args)
    if args.selcache:
        if args.impl != "ours":
            raise SystemExit("--selcache has no reference arm")
        return run_selcache(args)
    if args.perq:
        if args.impl != "ours":
            raise SystemExit("--perq has no reference arm")
        return run_perq(args)
    if args.prefill:
        if args.impl != "ours":
            raise SystemExit("--prefill has no reference arm")
        return run_prefill(args, W.PROMPTS[args.prefill])
    w = W.WORKLOADS[args.workload]
    if w.prompt_chunks != 1:
        raise SystemExit("bench.py times single-chunk workloads")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
