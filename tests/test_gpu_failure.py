"""Device-side failure paths made to fire without a GPU fault: a page id outside
the pool, an entry count outside the cache, and a bounded wait that runs out.
Each sets its CSA2_DEVERR_* bit, faults nothing, leaves the other sequences'
results exact and the context usable.  All calls go through the C ABI."""
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from fp4_sparse_attention_pack_b200 import workloads as W

from .oracle_models import ref_cache, ref_window
from .parity import ATTN_REL, attn_rel_err, check_topk
from .test_gpu_parity import _dev_cache_from_recipe, bf16_dev, csa, f32_dev  # noqa: F401 (fixture)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _windows(csa, wl, B, count):
    win = csa.engine.DeviceWindow(B, DEV)
    rings = []
    for b in range(B):
        ring, _ = ref_window(wl, 0, b, count)
        rings.append(ring)
        win.tokens[b] = bf16_dev(ring)
    win.count.fill_(count)
    return win, rings


def _run(csa, wl, dc, K, win):
    B = wl.B
    q, w, qm = W.query_idx(wl, 0, 0), W.head_weights(wl, 0, 0), W.query(wl, 0, 0)
    idx = torch.empty(B, K, dtype=torch.int32, device=DEV)
    ws = torch.empty(csa.index_topk_workspace(B, dc.max_pages * 64, wl.H_idx, K), dtype=torch.uint8, device=DEV)
    csa.index_topk(dc.desc, bf16_dev(q), f32_dev(w), K, idx, ws)
    out = torch.empty(B, wl.H, 512, dtype=torch.float32, device=DEV)
    wsa = torch.empty(max(csa.sparse_attn_workspace(B, wl.H, K), 16), dtype=torch.uint8, device=DEV)
    csa.sparse_attn(dc.desc, bf16_dev(qm), idx, K, win.desc, wl.scale, out, wsa)
    torch.cuda.synchronize()
    return q, w, qm, idx.cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("H_idx,H", [(64, 64), (16, 100)])  # tensor-core and CUDA-core kernels
def test_page_outside_pool_sets_status_and_spares_other_sequences(csa, H_idx, H):
    B, T, K, wc = 2, 4096, 256, 40
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H_idx=H_idx, H=H, K=K)
    dc = _dev_cache_from_recipe(csa, wl, 0, T, page_seed=5)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    n = T // 2
    bad = [3, 9]  # logical pages of sequence 1 pointed outside the pool
    dc.page_table[1, bad[0]] = dc.num_pages + 7
    dc.page_table[1, bad[1]] = -2
    win, rings = _windows(csa, wl, B, wc)
    q, w, qm, idx, out = _run(csa, wl, dc, K, win)
    assert dc.status_bits() & csa.DEVERR_PAGE
    # sequence 0 is exact
    check_topk(idx[0], rc.scores(0, q[0], w[0]), K)
    items = oracle.attention_items(rc.mc[0], rc.ms[0], n, idx[0], rings[0], wc)
    assert attn_rel_err(out[0], oracle.attention(qm[0], items, wl.scale)) <= ATTN_REL
    # sequence 1: valid indices; attention skips the entries of the bad pages
    g = idx[1][idx[1] >= 0]
    assert g.size == K and np.all(np.diff(g) > 0) and g.max() < n
    keep = g[~np.isin(g // 64, bad)]
    items = oracle.attention_items(rc.mc[1], rc.ms[1], n, keep, rings[1], wc)
    assert attn_rel_err(out[1], oracle.attention(qm[1], items, wl.scale)) <= ATTN_REL


def test_entry_count_outside_cache_sets_status(csa):
    B, T, K, wc = 2, 2048, 128, 7
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H_idx=64, H=64, K=K)
    dc = _dev_cache_from_recipe(csa, wl, 0, T, page_seed=6)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    n = T // 2
    win, rings = _windows(csa, wl, B, wc)
    # beyond the capacity: clamped to it (the pages there hold no entries yet)
    dc.n_entries[1] = dc.max_pages * 64 + 100
    q, w, qm, idx, out = _run(csa, wl, dc, K, win)
    assert dc.status_bits() & csa.DEVERR_COUNT
    check_topk(idx[0], rc.scores(0, q[0], w[0]), K)
    items = oracle.attention_items(rc.mc[0], rc.ms[0], n, idx[0], rings[0], wc)
    assert attn_rel_err(out[0], oracle.attention(qm[0], items, wl.scale)) <= ATTN_REL
    g = idx[1][idx[1] >= 0]
    assert g.size == K and np.all(np.diff(g) > 0) and g.max() < dc.max_pages * 64
    # negative: read as empty, so no entry is selected and only the window is attended
    dc.status.zero_()
    dc.n_entries[1] = -5
    q, w, qm, idx, out = _run(csa, wl, dc, K, win)
    assert dc.status_bits() & csa.DEVERR_COUNT
    assert np.all(idx[1] == -1)
    items = oracle.attention_items(rc.mc[1], rc.ms[1], 0, np.zeros(0, np.int32), rings[1], wc)
    assert attn_rel_err(out[1], oracle.attention(qm[1], items, wl.scale)) <= ATTN_REL
    check_topk(idx[0], rc.scores(0, q[0], w[0]), K)


def test_bounded_wait_runs_out_and_reports(csa):
    status = torch.zeros(4, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    csa.selftest_wait_timeout(status, 200000)  # 0.2 s
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert status[0].item() & csa.DEVERR_TIMEOUT
    assert dt >= 0.15
    # the context is still usable
    assert torch.arange(10, device=DEV).sum().item() == 45
    status.zero_()
    csa.selftest_wait_timeout(status, 1)
    torch.cuda.synchronize()
    assert status[0].item() == csa.DEVERR_TIMEOUT
