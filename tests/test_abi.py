"""The C ABI library builds for sm_100a, loads without a GPU and exports every
function include/csa2.h declares; host-side argument checks return errors
before anything is launched (no GPU needed: nothing reaches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def capi():
    from fp4_sparse_attention_pack_b200 import _build
    _build.build()
    import fp4_sparse_attention_pack_b200 as m
    return m


def declared_functions():
    with open(os.path.join(ROOT, "include", "csa2.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("csa2_pack_cache", "csa2_index_topk", "csa2_sparse_attn", "csa2_layer_step",
              "csa2_window_append", "csa2_version", "csa2_strerror"):
        assert f in names


def test_library_exports_every_declared_symbol(capi):
    lib = capi.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.csa2_version() >= 1
    assert lib.csa2_strerror(-1) == b"invalid argument"


def test_argument_checks_fail_before_launch(capi):
    lib = capi.lib()
    c = capi.csa2_cache()
    # null cache pointers -> invalid argument, nothing enqueued
    assert lib.csa2_pack_cache(ctypes.byref(c), None, 0, None, None, 4, None) == -1
    c = capi.csa2_cache(*([16] * 10), 1, 1, 1, 2)
    assert lib.csa2_pack_cache(ctypes.byref(c), ctypes.c_void_p(16), 7, ctypes.c_void_p(16),
                               ctypes.c_void_p(16), 4, None) == -1          # bad dtype
    c2 = capi.csa2_cache(*([16] * 9 + [17]), 1, 1, 1, 2)
    assert lib.csa2_pack_cache(ctypes.byref(c2), ctypes.c_void_p(16), 0, ctypes.c_void_p(16),
                               ctypes.c_void_p(16), 4, None) == -2          # misaligned
    c3 = capi.csa2_cache(*([16] * 10), 1, 1, 1, 3)
    assert lib.csa2_pack_cache(ctypes.byref(c3), ctypes.c_void_p(16), 0, ctypes.c_void_p(16),
                               ctypes.c_void_p(16), 4, None) == -1          # bad ratio
    # K and H_idx ranges; workspace too small
    assert lib.csa2_index_topk(ctypes.byref(c), ctypes.c_void_p(16), ctypes.c_void_p(16), 65, 8,
                               ctypes.c_void_p(16), None, None, 0, None) == -1
    assert lib.csa2_index_topk(ctypes.byref(c), ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 4096,
                               ctypes.c_void_p(16), None, None, 0, None) == -1
    assert lib.csa2_index_topk(ctypes.byref(c), ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 8,
                               ctypes.c_void_p(16), None, None, 0, None) == -6
    w = capi.csa2_window(16, 16, 1)
    # more than 64 heads take the CUDA-core path, which needs a workspace
    assert lib.csa2_sparse_attn(None, ctypes.c_void_p(16), 100, None, 0, ctypes.byref(w), 0.1,
                                ctypes.c_void_p(16), None, 0, None) == -6
    assert capi.sparse_attn_workspace(1, 100, 0) > 0
    assert lib.csa2_sparse_attn(None, ctypes.c_void_p(16), 0, None, 0, ctypes.byref(w), 0.1,
                                ctypes.c_void_p(16), None, 0, None) == -1
    assert capi.index_topk_workspace(2, 1024, 64, 512) > 2 * 1024 * 4
    assert capi.sparse_attn_workspace(2, 64, 512) > 0
    # the bounded-wait self-test: a NULL or misaligned status word is refused
    f = lib.csa2_selftest_wait_timeout
    f.argtypes = [ctypes.c_void_p, ctypes.c_uint, ctypes.c_void_p]
    assert f(None, 10, None) == -1
    assert f(ctypes.c_void_p(18), 10, None) == -1


def test_cache_io_argument_checks(capi):
    lib = capi.lib()
    assert capi.seq_image_bytes(0) == 16 + 2048
    assert capi.seq_image_bytes(10) == 16 + 2048 + 10 * (256 + 32 + 64 + 4)
    assert lib.csa2_seq_image_bytes(-1) == 0
    c = capi.csa2_cache(*([16] * 10), 2, 1, 1, 2)
    img = ctypes.c_void_p(32)
    for f in (lib.csa2_cache_export, lib.csa2_cache_import):
        assert f(None, 0, img, 4, None) == -1                       # no cache
        assert f(ctypes.byref(c), 0, None, 4, None) == -1           # no image
        assert f(ctypes.byref(c), 2, img, 4, None) == -1            # seq outside [0, batch)
        assert f(ctypes.byref(c), -1, img, 4, None) == -1
        assert f(ctypes.byref(c), 0, img, -1, None) == -1           # negative capacity
        assert f(ctypes.byref(c), 0, ctypes.c_void_p(40), 4, None) == -2  # unaligned image
    c_bad = capi.csa2_cache(*([16] * 10), 2, 1, 1, 3)
    assert lib.csa2_cache_export(ctypes.byref(c_bad), 0, img, 4, None) == -1  # bad ratio


def test_mode_table_validation(capi):
    import numpy as np
    from fp4_sparse_attention_pack_b200 import workloads as W
    lib = capi.lib()

    def model(mode, src, idx_src, ratios=(2,)):
        L, S = len(mode), len(ratios)
        caches = (capi.csa2_cache * S)(*[capi.csa2_cache(*([16] * 10), 1, 1, 1, r) for r in ratios])
        wins = (capi.csa2_window * L)(*[capi.csa2_window(16, 16, 1) for _ in range(L)])
        ws = (ctypes.c_void_p * S)(*([16] * S))
        keep = [(ctypes.c_int32 * L)(*mode), (ctypes.c_int32 * L)(*src), (ctypes.c_int32 * L)(*idx_src)]
        m = capi.csa2_model(L, S, keep[0], keep[1], keep[2], caches, ws, wins, 1, 4, 4, 8, 0.04)
        return m, (caches, wins, ws, keep)

    ok, keep = model([W.SWA_ONLY, W.FULL, W.REINDEX, W.REUSE], [0, 0, 0, 0], [0, 1, 2, 2])
    assert capi.layer_step_workspace(ok) > 0
    for mode, src, idx_src in [
        ([W.REUSE, W.FULL], [0, 0], [1, 1]),            # reuse names a later layer
        ([W.FULL, W.FULL], [0, 0], [0, 1]),             # two writers of one source
        ([W.REINDEX, W.FULL], [0, 0], [0, 1]),          # reindex before the source exists
        ([W.FULL, 7], [0, 0], [0, 1]),                  # unknown mode
        ([W.SWA_ONLY], [0], [0]),                       # a source nobody writes
    ]:
        bad, keep2 = model(mode, src, idx_src)
        assert capi.layer_step_workspace(bad) == 0
        sin, sout = capi.csa2_step_in(), capi.csa2_step_out()
        assert lib.csa2_layer_step(ctypes.byref(bad), ctypes.byref(sin), ctypes.byref(sout),
                                   ctypes.c_void_p(256), 1 << 30, None) == -1


def test_pool_argument_checks(capi):
    lib = capi.lib()
    c = capi.csa2_cache(*([16] * 10), 1, 1, 1, 2)
    p16 = ctypes.c_void_p(16)
    assert capi.index_pool_workspace(2, 1024, 64, 512, 0) == 0
    assert capi.index_pool_workspace(2, 1024, 64, 512, capi.MAX_POOL_BLOCKS + 1) == 0
    # block maxima + pool counts on top of a scan whose rows hold max(entries, 8 * pool_blocks)
    assert capi.index_pool_workspace(2, 1024, 64, 512, 2048) > capi.index_topk_workspace(2, 8 * 2048, 64, 512)
    for pb in (0, capi.MAX_POOL_BLOCKS + 1):
        assert lib.csa2_index_topk_pool(ctypes.byref(c), p16, p16, 4, 8, p16, None, pb, p16, p16, 1 << 30,
                                        None) == -1
        assert lib.csa2_index_topk_in_pool(ctypes.byref(c), p16, p16, 4, 8, p16, pb, p16, None, p16, 1 << 30,
                                           None) == -1
    assert lib.csa2_index_topk_pool(ctypes.byref(c), p16, p16, 4, 8, p16, None, 4, None, p16, 1 << 30,
                                    None) == -1                                     # no pool_out
    assert lib.csa2_index_topk_in_pool(ctypes.byref(c), p16, p16, 4, 8, ctypes.c_void_p(20), 4, p16, None,
                                       p16, 1 << 30, None) == -2                    # unaligned pool
    assert lib.csa2_index_topk_in_pool(ctypes.byref(c), p16, p16, 4, 8, p16, 4, p16, None, p16, 16,
                                       None) == -6                                  # workspace too small


def test_model_pool_blocks_range(capi):
    from fp4_sparse_attention_pack_b200 import workloads as W
    caches = (capi.csa2_cache * 1)(capi.csa2_cache(*([16] * 10), 1, 1, 1, 2))
    wins = (capi.csa2_window * 3)(*[capi.csa2_window(16, 16, 1) for _ in range(3)])
    ws = (ctypes.c_void_p * 1)(16)
    keep = [(ctypes.c_int32 * 3)(W.FULL, W.REINDEX, W.REUSE), (ctypes.c_int32 * 3)(0, 0, 0),
            (ctypes.c_int32 * 3)(0, 1, 1)]
    sizes = {}
    for pb in (0, 16, -1, capi.MAX_POOL_BLOCKS + 1):
        m = capi.csa2_model(3, 1, keep[0], keep[1], keep[2], caches, ws, wins, 1, 4, 4, 8, 0.04, pb)
        sizes[pb] = capi.layer_step_workspace(m)
    assert sizes[-1] == 0 and sizes[capi.MAX_POOL_BLOCKS + 1] == 0
    assert sizes[16] > sizes[0] > 0


def test_layer_step_launch_counts(capi):
    """Host-side launch accounting (no launch happens): window append, cache write (2),
    indexer (3), attention (1 when there are at least as many (layer, sequence) units as
    SMs -- here 1 sequence, so the split path with a combine: 2); pools add the block
    maxima (1) and, with Reindex layers, the pool scans (4)."""
    from fp4_sparse_attention_pack_b200 import workloads as W
    lib = capi.lib()

    def count(table, pool_blocks, with_token=True):
        L, S = table.n_layers, table.n_sources
        caches = (capi.csa2_cache * S)(*[capi.csa2_cache(*([16] * 10), 1, 1, 1, r) for r in table.ratios])
        wins = (capi.csa2_window * L)(*[capi.csa2_window(16, 16, 1) for _ in range(L)])
        ws = (ctypes.c_void_p * S)(*([16] * S))
        keep = [(ctypes.c_int32 * L)(*table.mode), (ctypes.c_int32 * L)(*[max(s, 0) for s in table.src]),
                (ctypes.c_int32 * L)(*[max(s, 0) for s in table.idx_src])]
        m = capi.csa2_model(L, S, keep[0], keep[1], keep[2], caches, ws, wins, 1, 64, 64, 512, 0.04, pool_blocks)
        x = (ctypes.c_void_p * S)(*([16 if with_token else None] * S))
        sin = capi.csa2_step_in(x, x)
        return lib.csa2_layer_step_launches(ctypes.byref(m), ctypes.byref(sin))

    alt, pages, one = W.schedule_alternating_40(), W.schedule_pages_40(), W.single_full()
    base = 1 + 2 + 3 + 2
    assert count(alt, 0) == base
    assert count(alt, 0, with_token=False) == base - 2
    assert count(alt, 2048) == base + 1 + 4
    assert count(pages, 2048) == base + 1 + 4
    assert count(one, 2048) == base + 1            # a pool is built, no Reindex layer scans it
    assert count(alt, -1) < 0                      # invalid table: a negative status


def test_host_fault_hook_returns_cuda_error_before_launch(capi, monkeypatch):
    """CSA2_INJECT_FAULT makes the named entry points fail as a failed launch
    would (CSA2_ERR_CUDA), after the argument checks and before anything is
    enqueued, and csa2_injected_faults counts it.  No GPU is involved: the
    pointers are never dereferenced on the host."""
    lib = capi.lib()
    lib.csa2_injected_faults.restype = ctypes.c_int
    c = capi.csa2_cache(*([16] * 10), 2, 1, 1, 2)
    ws = capi.index_topk_workspace(2, 64, 4, 8)
    w = capi.csa2_window(16, 16, 2, 0)

    def topk():
        return lib.csa2_index_topk(ctypes.byref(c), ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 8,
                                   ctypes.c_void_p(16), None, ctypes.c_void_p(256), ctypes.c_size_t(ws), None)

    def append():
        return lib.csa2_window_append(ctypes.byref(w), ctypes.c_void_p(16), None)

    n0 = lib.csa2_injected_faults()
    monkeypatch.setenv("CSA2_INJECT_FAULT", "csa2_index_topk")
    assert topk() == -4                                   # CSA2_ERR_CUDA, injected
    assert lib.csa2_injected_faults() == n0 + 1
    # an argument error still wins over the hook, and is not counted
    assert lib.csa2_index_topk(ctypes.byref(c), ctypes.c_void_p(16), ctypes.c_void_p(16), 65, 8,
                               ctypes.c_void_p(16), None, None, 0, None) == -1
    assert lib.csa2_injected_faults() == n0 + 1
    # other entry points are not listed: the window append is not injected
    # (without a GPU it fails in CUDA itself, which the counter does not see)
    append()
    assert lib.csa2_injected_faults() == n0 + 1
    monkeypatch.setenv("CSA2_INJECT_FAULT", "csa2_pack_cache,csa2_window_append")
    assert append() == -4
    assert lib.csa2_injected_faults() == n0 + 2
    monkeypatch.setenv("CSA2_INJECT_FAULT", "*")
    assert topk() == -4 and append() == -4
    assert lib.csa2_injected_faults() == n0 + 4
    monkeypatch.delenv("CSA2_INJECT_FAULT")
    append()
    assert lib.csa2_injected_faults() == n0 + 4
