"""ctypes binding over libquoka.so (argument marshalling only).

Every step of the selection and attention runs in the library's CUDA kernels; this
module turns torch tensors into pointers, host arrays and the current torch stream,
and turns non-OK statuses into exceptions.  torch provides device memory and streams.
If the library is missing the first call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libquoka.so")

QUOKA_OK, QUOKA_ERR_INVALID_ARG, QUOKA_ERR_UNSUPPORTED, QUOKA_ERR_WORKSPACE, QUOKA_ERR_CUDA = range(5)
QUOKA_F32, QUOKA_BF16 = 0, 1
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA"}

# (name, restype, argtypes) of every symbol include/quoka.h declares
_P = ctypes.c_void_p
_I64P = ctypes.POINTER(ctypes.c_int64)
_I32P = ctypes.POINTER(ctypes.c_int32)


class QuokaShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("chunk", ctypes.c_int), ("dtype", ctypes.c_int)]


_SHAPE_P = ctypes.POINTER(QuokaShape)

SIGNATURES = {
    "quoka_version": (ctypes.c_int, []),
    "quoka_last_error": (ctypes.c_char_p, []),
    "quoka_select_workspace_size": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int, ctypes.c_int]),
    "quoka_workspace_pooled_view": (ctypes.c_int, [_SHAPE_P, ctypes.c_int, ctypes.c_int,
                                                   ctypes.POINTER(ctypes.c_size_t),
                                                   ctypes.POINTER(ctypes.c_size_t)]),
    "quoka_select": (ctypes.c_int, [_SHAPE_P, _P, _P, _I64P, _I32P, ctypes.c_int, _I32P,
                                    ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "sparse_chunk_attn": (ctypes.c_int, [_SHAPE_P, _P, _P, _P, _I64P, _I32P, _I32P, _P,
                                         ctypes.c_int, _P, _P, ctypes.c_size_t, _P]),
    "sparse_chunk_attn_workspace_size": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int]),
    "quoka_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _P]),
    "quoka_select_noalloc": (ctypes.c_int, [_SHAPE_P, _P, _P, _I64P, _I32P, ctypes.c_int, _I32P,
                                            ctypes.c_int, _P, _P, _P]),
    "sparse_perq_attn": (ctypes.c_int, [_SHAPE_P, _P, _P, _P, _I64P, _P, ctypes.c_int, _P, _P,
                                        ctypes.c_size_t, _P]),
    "sparse_perq_attn_workspace_size": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int]),
    "sparse_perq_attn_tc": (ctypes.c_int, [_SHAPE_P, _P, _P, _P, _I64P, _P, ctypes.c_int, ctypes.c_int,
                                           _P, _P, ctypes.c_size_t, _P]),
    "sparse_perq_attn_tc_workspace_size": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int, ctypes.c_int]),
    "quoka_step": (ctypes.c_int, [_SHAPE_P, _P, _P, _P, _P, _P, _I64P, _I32P, ctypes.c_int,
                                  _I32P, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "quoka_step_workspace_size": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int]),
    "quoka_prefill": (ctypes.c_int, [_SHAPE_P, ctypes.c_int, _P, _P, _P, _P, _P, _I64P,
                                     ctypes.c_int, _I32P, ctypes.c_int, _P, _P, _P,
                                     ctypes.c_size_t, _P]),
    "quoka_prefill_workspace_size": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int, ctypes.c_int,
                                                       ctypes.c_int]),
    "quoka_selcache_bytes": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int]),
    "quoka_selcache_workspace_size": (ctypes.c_size_t, [_SHAPE_P, ctypes.c_int]),
    "quoka_selcache_update": (ctypes.c_int, [_SHAPE_P, _P, _P, _I64P, _I32P, _I32P, _P, ctypes.c_int,
                                             _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "sparse_chunk_attn_selcache": (ctypes.c_int, [_SHAPE_P, _P, _I32P, _I32P, _P, ctypes.c_int, _P,
                                                  _P, ctypes.c_size_t, _P]),
    "quoka_profile_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]),
    "quoka_profile_marks": (ctypes.c_int, [ctypes.POINTER(ctypes.c_char_p), ctypes.c_int]),
}

_lib = None


class QuokaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Loads libquoka.so from the package directory (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m query_oriented_sparse_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(status: int) -> None:
    if status != QUOKA_OK:
        raise QuokaError(status, lib().quoka_last_error().decode())


def make_shape(batch: int, h_q: int, h_kv: int, head_dim: int, chunk: int,
               dtype: torch.dtype) -> QuokaShape:
    if dtype == torch.float32:
        dt = QUOKA_F32
    elif dtype == torch.bfloat16:
        dt = QUOKA_BF16
    else:
        raise QuokaError(QUOKA_ERR_UNSUPPORTED, f"dtype {dtype}")
    return QuokaShape(batch, h_q, h_kv, head_dim, chunk, dt)


def shape_of(q_chunk: torch.Tensor, k_cache: torch.Tensor) -> QuokaShape:
    batch, h_q, chunk, d = q_chunk.shape
    return make_shape(batch, h_q, k_cache.shape[0], d, chunk, q_chunk.dtype)


def _host_i64(xs: Sequence[int]):
    arr = (ctypes.c_int64 * len(xs))(*[int(x) for x in xs])
    return arr


def _host_i32(xs: Sequence[int]):
    return (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def version() -> int:
    return lib().quoka_version()


def select_workspace_size(shape: QuokaShape, max_prefix: int, nq: int) -> int:
    return int(lib().quoka_select_workspace_size(ctypes.byref(shape), max_prefix, nq))


def pooled_view(workspace: torch.Tensor, shape: QuokaShape, max_prefix: int, nq: int) -> torch.Tensor:
    """The pooled key scores inside a quoka_select workspace, [batch, h_kv, stride] fp32."""
    off, stride = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().quoka_workspace_pooled_view(ctypes.byref(shape), max_prefix, nq,
                                             ctypes.byref(off), ctypes.byref(stride)))
    n = shape.batch * shape.h_kv * stride.value
    return workspace[off.value:off.value + 4 * n].view(torch.float32).view(
        shape.batch, shape.h_kv, stride.value)


def quoka_select(q_chunk: torch.Tensor, k_cache: torch.Tensor, kv_off: Sequence[int],
                 prefix_len: Sequence[int], nq: int, budget: Sequence[int],
                 b_max: Optional[int] = None, idx_out: Optional[torch.Tensor] = None,
                 kept_out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """QUOKA selection for one chunk step; returns idx [batch, h_kv, b_max] int32."""
    shape = shape_of(q_chunk, k_cache)
    if b_max is None:
        b_max = max(max(int(b) for b in budget), 1)
    dev = q_chunk.device
    if idx_out is None:
        idx_out = torch.empty(shape.batch, shape.h_kv, b_max, dtype=torch.int32, device=dev)
    if workspace is None:
        ws = select_workspace_size(shape, max(int(p) for p in prefix_len), nq)
        workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    _check(lib().quoka_select(
        ctypes.byref(shape), _ptr(q_chunk), _ptr(k_cache), _host_i64(kv_off),
        _host_i32(prefix_len), int(nq), _host_i32(budget), int(b_max), _ptr(idx_out),
        _ptr(kept_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        ctypes.c_void_p(_stream(stream))))
    return idx_out


def quoka_select_noalloc(q_chunk: torch.Tensor, k_cache: torch.Tensor, kv_off: Sequence[int],
                         prefix_len: Sequence[int], nq: int, budget: Sequence[int],
                         b_max: Optional[int] = None, idx_out: Optional[torch.Tensor] = None,
                         kept_out: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """quoka_select using the library's built-in scratch instead of a workspace (for
    callers that cannot allocate device memory); the outputs are still the caller's."""
    shape = shape_of(q_chunk, k_cache)
    if b_max is None:
        b_max = max(max(int(b) for b in budget), 1)
    if idx_out is None:
        idx_out = torch.empty(shape.batch, shape.h_kv, b_max, dtype=torch.int32,
                              device=q_chunk.device)
    _check(lib().quoka_select_noalloc(
        ctypes.byref(shape), _ptr(q_chunk), _ptr(k_cache), _host_i64(kv_off),
        _host_i32(prefix_len), int(nq), _host_i32(budget), int(b_max), _ptr(idx_out),
        _ptr(kept_out), ctypes.c_void_p(_stream(stream))))
    return idx_out


def attn_workspace_size(shape: QuokaShape, b_max: int) -> int:
    return int(lib().sparse_chunk_attn_workspace_size(ctypes.byref(shape), int(b_max)))


def sparse_chunk_attn(q_chunk: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      kv_off: Sequence[int], prefix_len: Sequence[int], budget: Sequence[int],
                      idx: torch.Tensor, out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Attention of the chunk over its compacted cache; returns out [batch, h_q, C, d]."""
    shape = shape_of(q_chunk, k_cache)
    if out is None:
        out = torch.empty_like(q_chunk)
    b_max = int(idx.shape[-1])
    if workspace is None:
        n = attn_workspace_size(shape, b_max)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q_chunk.device) if n else None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sparse_chunk_attn(
        ctypes.byref(shape), _ptr(q_chunk), _ptr(k_cache), _ptr(v_cache), _host_i64(kv_off),
        _host_i32(prefix_len), _host_i32(budget), _ptr(idx), b_max, _ptr(out), _ptr(workspace),
        ws_bytes, ctypes.c_void_p(_stream(stream))))
    return out


def perq_workspace_size(shape: QuokaShape, S: int) -> int:
    return int(lib().sparse_perq_attn_workspace_size(ctypes.byref(shape), int(S)))


def sparse_perq_attn(q_chunk: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     kv_off: Sequence[int], sel: torch.Tensor, out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Every query over its own key set, sel int32 [batch, h_q, C, S] (-1 = none);
    returns out [batch, h_q, C, d]."""
    shape = shape_of(q_chunk, k_cache)
    if out is None:
        out = torch.empty_like(q_chunk)
    S = int(sel.shape[-1])
    if workspace is None:
        n = perq_workspace_size(shape, S)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q_chunk.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().sparse_perq_attn(
        ctypes.byref(shape), _ptr(q_chunk), _ptr(k_cache), _ptr(v_cache), _host_i64(kv_off),
        _ptr(sel), S, _ptr(out), _ptr(workspace), ws_bytes, ctypes.c_void_p(_stream(stream))))
    return out


def perq_tc_workspace_size(shape: QuokaShape, S: int, max_union: int) -> int:
    return int(lib().sparse_perq_attn_tc_workspace_size(ctypes.byref(shape), int(S), int(max_union)))


def sparse_perq_attn_tc(q_chunk: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                        kv_off: Sequence[int], sel: torch.Tensor, max_union: int,
                        out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """sparse_perq_attn on tensor cores over 256-row pair tiles whose key unions hold at
    most max_union keys; returns out [batch, h_q, C, d]."""
    shape = shape_of(q_chunk, k_cache)
    if out is None:
        out = torch.empty_like(q_chunk)
    S = int(sel.shape[-1])
    if workspace is None:
        n = perq_tc_workspace_size(shape, S, max_union)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q_chunk.device)
    _check(lib().sparse_perq_attn_tc(
        ctypes.byref(shape), _ptr(q_chunk), _ptr(k_cache), _ptr(v_cache), _host_i64(kv_off),
        _ptr(sel), S, int(max_union), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.c_void_p(_stream(stream))))
    return out


def step_workspace_size(shape: QuokaShape, max_prefix: int, nq: int, b_max: int) -> int:
    return int(lib().quoka_step_workspace_size(ctypes.byref(shape), int(max_prefix), int(nq),
                                               int(b_max)))


def quoka_step(q_chunk: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
               k_cache: torch.Tensor, v_cache: torch.Tensor, kv_off: Sequence[int],
               prefix_len: Sequence[int], nq: int, budget: Sequence[int], idx: torch.Tensor,
               out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One chunk (or decode) step with the cache append: q_chunk [batch, h_q, C, d],
    k_new / v_new [batch, h_kv, C, d]; returns out [batch, h_q, C, d]."""
    shape = shape_of(q_chunk, k_cache)
    if out is None:
        out = torch.empty_like(q_chunk)
    b_max = int(idx.shape[-1])
    if workspace is None:
        n = step_workspace_size(shape, max(prefix_len), nq, b_max)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q_chunk.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().quoka_step(
        ctypes.byref(shape), _ptr(q_chunk), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
        _ptr(v_cache), _host_i64(kv_off), _host_i32(prefix_len), int(nq), _host_i32(budget),
        b_max, _ptr(idx), _ptr(out), _ptr(workspace), ws_bytes, ctypes.c_void_p(_stream(stream))))
    return out


def prefill_workspace_size(shape: QuokaShape, n_chunks: int, nq: int, b_max: int) -> int:
    return int(lib().quoka_prefill_workspace_size(ctypes.byref(shape), int(n_chunks), int(nq),
                                                  int(b_max)))


def quoka_prefill(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                  k_cache: torch.Tensor, v_cache: torch.Tensor, kv_off: Sequence[int], nq: int,
                  budgets: Sequence[int], idx: torch.Tensor, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """A whole prompt through chunked prefill, appending its K/V rows to the cache.

    q [n_chunks, batch, h_q, C, d]; k_new, v_new [n_chunks, batch, h_kv, C, d];
    budgets has one entry per chunk; returns out [n_chunks, batch, h_q, C, d].
    """
    n_chunks, batch, h_q, chunk, d = q.shape
    shape = make_shape(batch, h_q, k_cache.shape[0], d, chunk, q.dtype)
    if out is None:
        out = torch.empty_like(q)
    b_max = int(idx.shape[-1])
    if workspace is None:
        n = prefill_workspace_size(shape, n_chunks, nq, b_max)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().quoka_prefill(
        ctypes.byref(shape), int(n_chunks), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
        _ptr(v_cache), _host_i64(kv_off), int(nq), _host_i32(budgets), b_max, _ptr(idx),
        _ptr(out), _ptr(workspace), ws_bytes, ctypes.c_void_p(_stream(stream))))
    return out


def device_error(stream: Optional[torch.cuda.Stream] = None) -> int:
    code = ctypes.c_uint32(0)
    _check(lib().quoka_device_error(ctypes.byref(code), ctypes.c_void_p(_stream(stream))))
    return code.value


class SelCache:
    """A selected-value cache (quoka_selcache_update / sparse_chunk_attn_selcache) for one
    shape and b_max: the K/V blocks, the slot map (all -1 at first) and a workspace, all
    torch device memory owned by this object."""

    def __init__(self, shape: QuokaShape, b_max: int, device):
        self.shape, self.b_max = shape, int(b_max)
        n = int(lib().quoka_selcache_bytes(ctypes.byref(shape), self.b_max))
        w = int(lib().quoka_selcache_workspace_size(ctypes.byref(shape), self.b_max))
        if n == 0 or w == 0:
            raise QuokaError(QUOKA_ERR_INVALID_ARG, "bad shape or b_max for a selected-value cache")
        self.cache = torch.zeros(n, dtype=torch.uint8, device=device)
        self.slot_rows = torch.full((shape.batch, shape.h_kv, self.b_max), -1, dtype=torch.int32,
                                    device=device)
        self.misses = torch.zeros(shape.batch, shape.h_kv, dtype=torch.int32, device=device)
        self.workspace = torch.empty(w, dtype=torch.uint8, device=device)

    def blocks(self, dtype: torch.dtype):
        """(K, V) views [batch, h_kv, kc_rows, head_dim] of the cache."""
        s = self.shape
        half = self.cache.numel() // 2
        esz = torch.empty((), dtype=dtype).element_size()
        rows = (self.b_max + s.chunk + 127) // 128 * 128
        n = s.batch * s.h_kv * rows * s.head_dim * esz
        k = self.cache[:n].view(dtype).view(s.batch, s.h_kv, rows, s.head_dim)
        v = self.cache[half:half + n].view(dtype).view(s.batch, s.h_kv, rows, s.head_dim)
        return k, v

    def update(self, k_cache: torch.Tensor, v_cache: torch.Tensor, kv_off: Sequence[int],
               prefix_len: Sequence[int], budget: Sequence[int], idx: torch.Tensor,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """Brings the cache to the selection idx; returns the misses per (sequence, KV head)."""
        if int(idx.shape[-1]) != self.b_max:
            raise QuokaError(QUOKA_ERR_INVALID_ARG, "idx's last dimension must be the cache's b_max")
        _check(lib().quoka_selcache_update(
            ctypes.byref(self.shape), _ptr(k_cache), _ptr(v_cache), _host_i64(kv_off),
            _host_i32(prefix_len), _host_i32(budget), _ptr(idx), self.b_max, _ptr(self.cache),
            _ptr(self.slot_rows), _ptr(self.misses), _ptr(self.workspace),
            self.workspace.numel(), ctypes.c_void_p(_stream(stream))))
        return self.misses

    def attend(self, q_chunk: torch.Tensor, prefix_len: Sequence[int], budget: Sequence[int],
               out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """sparse_chunk_attn over the cache's rows; returns out [batch, h_q, C, d]."""
        if out is None:
            out = torch.empty_like(q_chunk)
        _check(lib().sparse_chunk_attn_selcache(
            ctypes.byref(self.shape), _ptr(q_chunk), _host_i32(prefix_len), _host_i32(budget),
            _ptr(self.cache), self.b_max, _ptr(out), _ptr(self.workspace), self.workspace.numel(),
            ctypes.c_void_p(_stream(stream))))
        return out


class KernelTimer:
    """Per-kernel device times of the library calls made inside a ``with`` block.

    Enqueues a short spin kernel and a start event on the stream, hands the library a pool
    of timing events (one is recorded after every kernel it launches from this thread,
    quoka_profile_events), and afterwards yields (kernel name, milliseconds) pairs in
    launch order.  The spin keeps the GPU busy while the host enqueues the calls, so each
    gap between events is one kernel's device time.  Eager calls only: not inside a
    stream capture.
    """

    def __init__(self, max_kernels: int = 64, stream: Optional[torch.cuda.Stream] = None):
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.start = torch.cuda.Event(enable_timing=True)
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(max_kernels)]
        for e in [self.start] + self.events:          # torch creates events on first record
            e.record(self.stream)
        self.stream.synchronize()
        self._handles = (ctypes.c_void_p * max_kernels)(*[e.cuda_event for e in self.events])
        self.times = []

    def __enter__(self):
        # a spin kernel ahead of the calls keeps the GPU busy while the host enqueues them,
        # so no host gap sits between the start event and the first kernel
        with torch.cuda.stream(self.stream):
            torch.cuda._sleep(4_000_000)
        self.start.record(self.stream)
        _check(lib().quoka_profile_events(self._handles, len(self.events)))
        return self

    def __exit__(self, *exc):
        n = int(lib().quoka_profile_marks(None, 0))
        names = (ctypes.c_char_p * max(n, 1))()
        lib().quoka_profile_marks(names, n)
        _check(lib().quoka_profile_events(None, 0))
        if exc[0] is None:
            self.stream.synchronize()
            prev = self.start
            for i in range(n):
                self.times.append((names[i].decode(), prev.elapsed_time(self.events[i])))
                prev = self.events[i]
        return False
