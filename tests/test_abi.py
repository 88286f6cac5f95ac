"""The C ABI library: it loads, exports every symbol include/quoka.h declares, and its
host-side validation rejects bad calls with the documented status before launching
anything.  The fake-pointer cases run only where no GPU is present (with a GPU the
same rejections are exercised with real buffers in test_kernels.py, test_prefill.py and
test_step.py)."""
import ctypes
import os
import re

import pytest
import torch

from query_oriented_sparse_b200 import binding as Bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "quoka.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", src)) -
                  {"if", "sizeof", "defined"})


def test_header_declares_the_boundary():
    fns = declared_functions()
    for name in ("quoka_select", "sparse_chunk_attn", "quoka_select_workspace_size",
                 "quoka_last_error", "quoka_device_error", "quoka_version",
                 "quoka_workspace_pooled_view"):
        assert name in fns


def test_library_loads_and_exports_every_declared_symbol():
    lib = Bd.lib()
    for name in declared_functions():
        assert hasattr(lib, name), f"libquoka.so does not export {name}"
    assert set(declared_functions()) == set(Bd.SIGNATURES), "binding and header disagree"
    assert Bd.version() == 101


def test_attn_workspace_size():
    s = Bd.make_shape(1, 32, 8, 128, 4096, torch.bfloat16)
    # compacted K and V: 8 heads x (16384 selected + 4096 chunk rows) x 256 B each
    assert Bd.attn_workspace_size(s, 16384) == 2 * 8 * (16384 + 4096) * 256
    # blocks are padded to a multiple of 128 rows
    assert Bd.attn_workspace_size(Bd.make_shape(1, 8, 4, 128, 96, torch.bfloat16), 200) == \
        2 * 4 * 384 * 256
    assert Bd.attn_workspace_size(Bd.make_shape(1, 4, 1, 64, 128, torch.float32), 128) == 0


def test_workspace_size_is_host_only():
    s = Bd.make_shape(1, 32, 8, 128, 4096, torch.bfloat16)
    n = Bd.select_workspace_size(s, 131072, 128)
    # kept queries (32*128 rows of 256 B) + their inverse norms + 8*131072 fp32 scores
    assert n >= 32 * 128 * 256 + 32 * 128 * 4 + 8 * 131072 * 4
    assert n % 256 == 0
    bad = Bd.make_shape(1, 32, 8, 96, 4096, torch.bfloat16)
    assert Bd.select_workspace_size(bad, 10, 4) == 0


no_gpu = pytest.mark.skipif(torch.cuda.is_available(),
                            reason="fake device pointers are only passed where there is no GPU")

FAKE = 0x10000  # never dereferenced: every case below must fail host-side validation


def _select(shape, q=FAKE, k=FAKE, kv_off=(0, 1024), prefix=(512,), nq=8, budget=(64,),
            b_max=64, idx=FAKE, kept=None, ws=FAKE, ws_bytes=1 << 30):
    lib = Bd.lib()
    return lib.quoka_select(ctypes.byref(shape), q, k, Bd._host_i64(kv_off), Bd._host_i32(prefix),
                            nq, Bd._host_i32(budget), b_max, idx, kept, ws, ws_bytes, None)


def _attn(shape, q=FAKE, k=FAKE, v=FAKE, kv_off=(0, 1024), prefix=(512,), budget=(64,),
          idx=FAKE, b_max=64, out=FAKE + 4096, ws=FAKE, ws_bytes=1 << 30):
    lib = Bd.lib()
    return lib.sparse_chunk_attn(ctypes.byref(shape), q, k, v, Bd._host_i64(kv_off),
                                 Bd._host_i32(prefix), Bd._host_i32(budget), idx, b_max, out, ws,
                                 ws_bytes, None)


@no_gpu
@pytest.mark.parametrize("case,status", [
    (dict(shape=dict(head_dim=96)), Bd.QUOKA_ERR_UNSUPPORTED),
    (dict(shape=dict(batch=65)), Bd.QUOKA_ERR_UNSUPPORTED),
    (dict(shape=dict(batch=0)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(shape=dict(h_q=6, h_kv=4)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(shape=dict(chunk=9000)), Bd.QUOKA_ERR_UNSUPPORTED),
    (dict(shape=dict(dtype=7)), Bd.QUOKA_ERR_UNSUPPORTED),
    (dict(q=FAKE + 2), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(idx=None), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(nq=0), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(prefix=(-1,)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(prefix=(1000,)), Bd.QUOKA_ERR_INVALID_ARG),        # prefix + chunk > rows
    (dict(budget=(65,)), Bd.QUOKA_ERR_INVALID_ARG),          # budget > b_max
    (dict(b_max=0, budget=(0,)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(ws=None), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws_bytes=100), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws=FAKE + 16), Bd.QUOKA_ERR_INVALID_ARG),          # workspace not 256-aligned
    (dict(kv_off=(-4, 1020)), Bd.QUOKA_ERR_INVALID_ARG),
])
def test_select_rejects(case, status):
    shp = dict(batch=1, h_q=8, h_kv=2, head_dim=128, chunk=256, dtype=Bd.QUOKA_BF16)
    shp.update(case.pop("shape", {}))
    shape = Bd.QuokaShape(**shp)
    assert _select(shape, **case) == status
    assert Bd.lib().quoka_last_error().decode()


@no_gpu
@pytest.mark.parametrize("case,status", [
    (dict(shape=dict(head_dim=32)), Bd.QUOKA_ERR_UNSUPPORTED),
    (dict(out=FAKE), Bd.QUOKA_ERR_INVALID_ARG),               # aliases q
    (dict(v=None), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(budget=(-1,)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(kv_off=(0, 600)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(ws=None), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws_bytes=1000), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws=FAKE + 64), Bd.QUOKA_ERR_INVALID_ARG),
])
def test_attn_rejects(case, status):
    shp = dict(batch=1, h_q=8, h_kv=2, head_dim=128, chunk=256, dtype=Bd.QUOKA_BF16)
    shp.update(case.pop("shape", {}))
    shape = Bd.QuokaShape(**shp)
    assert _attn(shape, **case) == status


def _step(shape, q=FAKE, k_new=FAKE + 0x2000, v_new=FAKE + 0x3000, k=FAKE + 0x4000,
          v=FAKE + 0x5000, kv_off=(0, 1024), prefix=(512,), nq=8, budget=(64,), b_max=64,
          idx=FAKE + 0x6000, out=FAKE + 0x7000, ws=FAKE, ws_bytes=1 << 30):
    return Bd.lib().quoka_step(ctypes.byref(shape), q, k_new, v_new, k, v, Bd._host_i64(kv_off),
                               Bd._host_i32(prefix), nq, Bd._host_i32(budget), b_max, idx, out,
                               ws, ws_bytes, None)


@no_gpu
@pytest.mark.parametrize("case,status", [
    (dict(shape=dict(head_dim=96)), Bd.QUOKA_ERR_UNSUPPORTED),
    (dict(k_new=None), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(v_new=FAKE + 0x3004), Bd.QUOKA_ERR_INVALID_ARG),       # misaligned
    (dict(out=FAKE), Bd.QUOKA_ERR_INVALID_ARG),                  # aliases q
    (dict(out=FAKE + 0x4000), Bd.QUOKA_ERR_INVALID_ARG),         # aliases the K cache
    (dict(budget=(65,)), Bd.QUOKA_ERR_INVALID_ARG),              # budget > b_max
    (dict(prefix=(900,)), Bd.QUOKA_ERR_INVALID_ARG),             # prefix + chunk > rows
    (dict(nq=0), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(ws=None), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws_bytes=1000), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws=FAKE + 64), Bd.QUOKA_ERR_INVALID_ARG),              # workspace not 256-aligned
])
def test_step_rejects(case, status):
    shp = dict(batch=1, h_q=8, h_kv=2, head_dim=128, chunk=256, dtype=Bd.QUOKA_BF16)
    shp.update(case.pop("shape", {}))
    assert _step(Bd.QuokaShape(**shp), **case) == status
    assert Bd.lib().quoka_last_error().decode()


def _prefill(shape, n_chunks=2, q=FAKE, k_new=FAKE + 0x2000, v_new=FAKE + 0x3000,
             k=FAKE + 0x4000, v=FAKE + 0x5000, kv_off=(0, 1024), nq=8, budgets=(0, 64), b_max=64,
             idx=FAKE + 0x6000, out=FAKE + 0x7000, ws=FAKE, ws_bytes=1 << 30):
    return Bd.lib().quoka_prefill(ctypes.byref(shape), n_chunks, q, k_new, v_new, k, v,
                                  Bd._host_i64(kv_off), nq,
                                  None if budgets is None else Bd._host_i32(budgets), b_max, idx,
                                  out, ws, ws_bytes, None)


@no_gpu
@pytest.mark.parametrize("case,status", [
    (dict(n_chunks=0, budgets=(0,)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(budgets=(0, 65)), Bd.QUOKA_ERR_INVALID_ARG),           # budget > b_max
    (dict(budgets=(0, -1)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(budgets=None), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(kv_off=(0, 500)), Bd.QUOKA_ERR_INVALID_ARG),           # fewer rows than the prompt
    (dict(n_chunks=5, budgets=(0, 8, 8, 8, 8)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(out=FAKE), Bd.QUOKA_ERR_INVALID_ARG),                  # aliases q
    (dict(q=FAKE + 2), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(ws=None), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws_bytes=100), Bd.QUOKA_ERR_WORKSPACE),
])
def test_prefill_rejects(case, status):
    shape = Bd.QuokaShape(batch=1, h_q=8, h_kv=2, head_dim=128, chunk=256, dtype=Bd.QUOKA_BF16)
    assert _prefill(shape, **case) == status
    assert Bd.lib().quoka_last_error().decode()


def test_step_and_prefill_workspace_sizes():
    s = Bd.make_shape(1, 32, 8, 128, 4096, torch.bfloat16)
    n_step = Bd.step_workspace_size(s, 131072, 128, 16384)
    assert n_step == (Bd.select_workspace_size(s, 131072, 128) + 255) // 256 * 256 + \
        Bd.attn_workspace_size(s, 16384)
    # 33 chunks: the last selects over 32 * 4096 prefix rows
    assert Bd.prefill_workspace_size(s, 33, 128, 16384) == n_step
    assert Bd.prefill_workspace_size(s, 0, 128, 16384) == 0
    assert Bd.step_workspace_size(s, -1, 128, 16384) == 0
    # decode (G * C <= 16): the attention scratch holds split partials, not a compacted cache
    d = Bd.make_shape(32, 32, 8, 128, 1, torch.bfloat16)
    parts = 32 * 8 * ((2048 + 1 + 255) // 256) * 4 * (128 + 4) * 4
    assert Bd.attn_workspace_size(d, 2048) == (parts + 255) // 256 * 256


def test_null_shape_rejected():
    lib = Bd.lib()
    assert lib.quoka_select(None, FAKE, FAKE, Bd._host_i64((0, 8)), Bd._host_i32((0,)), 1,
                            Bd._host_i32((0,)), 1, FAKE, None, FAKE, 1 << 20, None) == \
        Bd.QUOKA_ERR_INVALID_ARG
    assert "NULL" in lib.quoka_last_error().decode()


@no_gpu
def test_noalloc_rejects_oversize_before_launch():
    """A call whose scratch would not fit the built-in array is refused host-side."""
    lib = Bd.lib()
    shape = Bd.QuokaShape(64, 64, 8, 128, 64, Bd.QUOKA_BF16)
    need = lib.quoka_select_workspace_size(ctypes.byref(shape), 0, 64)
    assert need > (32 << 20)
    st = lib.quoka_select_noalloc(ctypes.byref(shape), FAKE, FAKE,
                                  Bd._host_i64([0] + [64 * (i + 1) for i in range(64)]),
                                  Bd._host_i32([0] * 64), 64, Bd._host_i32([1] * 64), 1, FAKE,
                                  None, None)
    assert st == Bd.QUOKA_ERR_WORKSPACE
    assert "built-in scratch" in lib.quoka_last_error().decode()


def test_profile_events_host_checks():
    """The timing hook checks its arguments on the host and starts with no marks."""
    lib = Bd.lib()
    assert lib.quoka_profile_events(None, 0) == Bd.QUOKA_OK
    assert lib.quoka_profile_marks(None, 0) == 0
    empty = (ctypes.c_void_p * 1)(None)
    assert lib.quoka_profile_events(empty, 1) == Bd.QUOKA_ERR_INVALID_ARG
    assert lib.quoka_profile_events(empty, 0) == Bd.QUOKA_ERR_INVALID_ARG
    assert lib.quoka_profile_marks(None, 0) == 0


def test_selcache_sizes():
    s = Bd.make_shape(2, 8, 2, 128, 96, torch.bfloat16)
    lib = Bd.lib()
    # K and V blocks of 2 x 2 (sequence, KV head) pairs x (200 + 96 -> 384 rows) x 256 B
    assert lib.quoka_selcache_bytes(ctypes.byref(s), 200) == 2 * 4 * 384 * 256
    assert lib.quoka_selcache_workspace_size(ctypes.byref(s), 200) > 2 * 4 * 200 * 4
    assert lib.quoka_selcache_bytes(ctypes.byref(s), 0) == 0
    bad = Bd.make_shape(1, 8, 2, 96, 96, torch.bfloat16)
    assert lib.quoka_selcache_bytes(ctypes.byref(bad), 64) == 0


def _selupd(shape, k=FAKE, v=FAKE + 0x1000, kv_off=(0, 1024), prefix=(512,), budget=(64,),
            idx=FAKE + 0x2000, b_max=64, cache=FAKE + 0x10000, slots=FAKE + 0x3000, misses=None,
            ws=FAKE + 0x4000, ws_bytes=1 << 30):
    return Bd.lib().quoka_selcache_update(
        ctypes.byref(shape), k, v, Bd._host_i64(kv_off), Bd._host_i32(prefix), Bd._host_i32(budget),
        idx, b_max, cache, slots, misses, ws, ws_bytes, None)


@no_gpu
@pytest.mark.parametrize("case,status", [
    (dict(shape=dict(head_dim=96)), Bd.QUOKA_ERR_UNSUPPORTED),
    (dict(idx=None), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(slots=None), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(cache=FAKE + 0x10010), Bd.QUOKA_ERR_INVALID_ARG),   # not 256-byte aligned
    (dict(cache=FAKE), Bd.QUOKA_ERR_INVALID_ARG),             # aliases k_cache
    (dict(budget=(65,)), Bd.QUOKA_ERR_INVALID_ARG),
    (dict(prefix=(1000,)), Bd.QUOKA_ERR_INVALID_ARG),         # prefix + chunk > rows
    (dict(ws=None), Bd.QUOKA_ERR_WORKSPACE),
    (dict(ws_bytes=64), Bd.QUOKA_ERR_WORKSPACE),
    (dict(kv_off=(0, 1 << 21), prefix=(1 << 21) - 300, b_max=1 << 19, budget=(1 << 19,)),
     Bd.QUOKA_ERR_UNSUPPORTED),                                # bitmaps beyond shared memory
])
def test_selcache_update_rejects(case, status):
    shp = dict(batch=1, h_q=8, h_kv=2, head_dim=128, chunk=256, dtype=Bd.QUOKA_BF16)
    shp.update(case.pop("shape", {}))
    if isinstance(case.get("prefix"), int):
        case["prefix"] = (case["prefix"],)
    assert _selupd(Bd.QuokaShape(**shp), **case) == status


@no_gpu
def test_selcache_attn_rejects():
    lib = Bd.lib()
    s = Bd.QuokaShape(1, 8, 2, 128, 256, Bd.QUOKA_BF16)

    def call(q=FAKE, budget=(64,), cache=FAKE + 0x10000, b_max=64, out=FAKE + 0x20000, ws=FAKE + 0x30000,
             ws_bytes=1 << 30):
        return lib.sparse_chunk_attn_selcache(ctypes.byref(s), q, Bd._host_i32((512,)), Bd._host_i32(budget),
                                              cache, b_max, out, ws, ws_bytes, None)
    assert call(out=FAKE) == Bd.QUOKA_ERR_INVALID_ARG            # aliases q
    assert call(budget=(65,)) == Bd.QUOKA_ERR_INVALID_ARG
    assert call(b_max=0, budget=(0,)) == Bd.QUOKA_ERR_INVALID_ARG
    assert call(cache=FAKE + 0x10008) == Bd.QUOKA_ERR_INVALID_ARG
    assert call(ws=None) == Bd.QUOKA_ERR_WORKSPACE
    assert call(ws_bytes=16) == Bd.QUOKA_ERR_WORKSPACE


def test_perq_tc_sizes_and_limits():
    lib = Bd.lib()
    s = Bd.make_shape(1, 32, 8, 128, 4096, torch.bfloat16)
    n = lib.sparse_perq_attn_tc_workspace_size(ctypes.byref(s), 512, 8192)
    # 8 KV heads x 64 pair tiles: union K/V blocks of 8192 rows of 256 B each, plus masks
    tiles = 8 * 64
    assert n >= tiles * 8192 * 256 * 2 + tiles * 256 * (8192 // 32) * 4
    assert lib.sparse_perq_attn_tc_workspace_size(ctypes.byref(s), 512, 1 << 20) == 0   # masks too large
    f32 = Bd.make_shape(1, 32, 8, 128, 4096, torch.float32)
    assert lib.sparse_perq_attn_tc_workspace_size(ctypes.byref(f32), 512, 8192) == 0
