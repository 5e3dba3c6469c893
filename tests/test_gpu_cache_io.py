"""Prefix-cache export / import of one sequence (csa2_cache_export /
csa2_cache_import): byte-exact round trips between caches with different page
tables, through device memory and through pinned host memory, the image
layout, and the device-side error bits.  All calls go through the C ABI."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from fp4_sparse_attention_pack_b200 import workloads as W

from .oracle_models import ref_cache

pytestmark = pytest.mark.gpu

DEV = "cuda"
HDR, PEND = 16, 2048
ROW = 256 + 32 + 64 + 4


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from fp4_sparse_attention_pack_b200 import _build
    _build.build()
    import fp4_sparse_attention_pack_b200 as m
    from fp4_sparse_attention_pack_b200 import engine
    m.engine = engine
    return m


def filled_model(csa, B, T, seed):
    """A one-layer model whose source cache holds T tokens (ratio 2, odd T leaves
    a pending token) in shuffled pages."""
    wl = W.Workload("io", seed, B, T, W.single_full(), 8, 16, 64, 2)
    dm = csa.engine.DecodeModel(wl, DEV, page_seed=seed + 3)
    dm.fill(chunk_tokens=257)
    torch.cuda.synchronize()
    return wl, dm


def image_rows(img, cap, n):
    """(main codes, main scales, idx codes, idx scales) rows [0, n) of an image."""
    a = img.cpu().numpy()
    o = HDR + PEND
    mc = a[o:o + cap * 256].reshape(cap, 256)[:n]
    o += cap * 256
    ms = a[o:o + cap * 32].reshape(cap, 32)[:n]
    o += cap * 32
    kc = a[o:o + cap * 64].reshape(cap, 64)[:n]
    o += cap * 64
    ks = a[o:o + cap * 4].reshape(cap, 4)[:n]
    return mc, ms, kc, ks


def test_image_bytes(csa):
    assert csa.seq_image_bytes(0) == HDR + PEND
    assert csa.seq_image_bytes(1000) == HDR + PEND + 1000 * ROW


@pytest.mark.parametrize("T", [1201, 4096])
def test_export_import_round_trip(csa, T):
    wl, src = filled_model(csa, 3, T, 11)
    c_src = src.caches[0]
    n = T // 2
    cap = c_src.max_pages * 64
    img = torch.zeros(csa.seq_image_bytes(cap), dtype=torch.uint8, device=DEV)
    csa.cache_export(c_src.desc, 1, img, cap)
    torch.cuda.synchronize()
    # header and rows: the logical bytes of sequence 1
    hdr = img[:16].cpu().numpy()
    n_img, pend_valid, _, ratio = hdr.view(np.int32)
    assert (n_img, ratio) == (n, 2)
    assert pend_valid == c_src.pend_valid[1].item() == (T & 1)
    assert np.array_equal(img[16:16 + PEND].cpu().numpy().view(np.float32), c_src.pend_x[1].cpu().numpy())
    for got, want in zip(image_rows(img, cap, n), c_src.logical(1, 0, n)):
        assert np.array_equal(got, want)
    # ... which are the oracle's packed entries of that sequence (same seeded recipe)
    rc = ref_cache(wl, 0, [1], T, cap=n + 64)
    for got, want in zip(image_rows(img, cap, n), (rc.mc[0, :n], rc.ms[0, :n], rc.kc[0, :n], rc.ks[0, :n])):
        assert np.array_equal(got, want)
    assert rc.pend_valid[0] == pend_valid
    if pend_valid:
        assert np.array_equal(img[16:16 + PEND].cpu().numpy().view(np.float32), rc.pend_x[0])
    # into sequence 0 of a cache with another page permutation
    dst = csa.engine.DeviceCache(3, c_src.max_pages, 2, DEV, page_seed=77, spare_pages=5)
    csa.cache_import(dst.desc, 0, img, cap)
    torch.cuda.synchronize()
    assert dst.n_entries[0].item() == n and dst.n_entries[1].item() == 0
    assert dst.pend_valid[0].item() == c_src.pend_valid[1].item()
    assert dst.pend_g[0].item() == c_src.pend_g[1].item()
    assert torch.equal(dst.pend_x[0], c_src.pend_x[1])
    for got, want in zip(dst.logical(0, 0, n), c_src.logical(1, 0, n)):
        assert np.array_equal(got, want)
    assert dst.status_bits() == 0 and c_src.status_bits() == 0
    # the imported cache scans to the same Top-K
    q = torch.randn(1, 16, 128, device=DEV).to(torch.bfloat16)
    w = torch.rand(1, 16, device=DEV)
    ws = torch.empty(csa.index_topk_workspace(3, cap, 16, 64), dtype=torch.uint8, device=DEV)
    outs = []
    for cache, seq in ((c_src, 1), (dst, 0)):
        q3 = torch.zeros(3, 16, 128, dtype=torch.bfloat16, device=DEV)
        w3 = torch.zeros(3, 16, device=DEV)
        q3[seq], w3[seq] = q[0], w[0]
        idx = torch.empty(3, 64, dtype=torch.int32, device=DEV)
        csa.index_topk(cache.desc, q3, w3, 64, idx, ws)
        torch.cuda.synchronize()
        outs.append(idx[seq].cpu().numpy())
    assert np.array_equal(outs[0], outs[1])


def test_export_through_pinned_host_memory(csa):
    wl, src = filled_model(csa, 2, 777, 5)
    c = src.caches[0]
    n, cap = 777 // 2, c.max_pages * 64
    host = torch.zeros(csa.seq_image_bytes(cap), dtype=torch.uint8).pin_memory()
    csa.cache_export(c.desc, 0, host, cap)
    torch.cuda.synchronize()
    for got, want in zip(image_rows(host, cap, n), c.logical(0, 0, n)):
        assert np.array_equal(got, want)
    dst = csa.engine.DeviceCache(2, c.max_pages, 2, DEV, page_seed=9)
    csa.cache_import(dst.desc, 1, host, cap)
    torch.cuda.synchronize()
    for got, want in zip(dst.logical(1, 0, n), c.logical(0, 0, n)):
        assert np.array_equal(got, want)


def test_short_image_and_bad_header(csa):
    wl, src = filled_model(csa, 1, 501, 2)
    c = src.caches[0]
    n = 250
    cap = 100  # smaller than the sequence: 100 rows, CAPACITY bit
    img = torch.zeros(csa.seq_image_bytes(cap), dtype=torch.uint8, device=DEV)
    csa.cache_export(c.desc, 0, img, cap)
    torch.cuda.synchronize()
    assert img[:4].cpu().numpy().view(np.int32)[0] == cap
    assert c.status_bits() & csa.DEVERR_CAPACITY
    for got, want in zip(image_rows(img, cap, cap), c.logical(0, 0, cap)):
        assert np.array_equal(got, want)
    # an image of a ratio-2 source does not go into a ratio-1 cache
    dst = csa.engine.DeviceCache(1, c.max_pages, 1, DEV)
    before = dst.main_codes.clone()
    csa.cache_import(dst.desc, 0, img, cap)
    torch.cuda.synchronize()
    assert dst.status_bits() & csa.DEVERR_IMAGE
    assert dst.n_entries[0].item() == 0 and torch.equal(dst.main_codes, before)
    assert n > cap
