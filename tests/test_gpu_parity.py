"""GPU parity of every step of the path against the oracle, on small cases that
still span several tiles and ragged tails, plus rounding ties and edge cases.
All calls go through the C ABI (libcsa2.so)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from fp4_sparse_attention_pack_b200 import synth
from fp4_sparse_attention_pack_b200 import workloads as W

from .oracle_models import ref_cache, ref_model, ref_window, step_inputs
from .parity import ATTN_REL, attn_rel_err, check_topk

pytestmark = pytest.mark.gpu

DEV = "cuda"


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


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def f32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)


def compare_cache(dc, rc, b_dev, b_ref, n):
    mc, ms, kc, ks = dc.logical(b_dev, 0, n)
    assert np.array_equal(ms, rc.ms[b_ref, :n]), "main scales differ"
    assert np.array_equal(mc, rc.mc[b_ref, :n]), "main codes differ"
    assert np.array_equal(ks, rc.ks[b_ref, :n]), "indexer scales differ"
    assert np.array_equal(kc, rc.kc[b_ref, :n]), "indexer codes differ"


# ---------------------------------------------------------------- generator

def test_device_generator_matches_host(csa):
    wl = W.WORKLOADS[3]
    chan = W.chan_scale(wl, 0)
    k = synth.key(3, synth.TID_SRC_X, 0)
    d = torch.empty(3, 1536, dtype=torch.bfloat16, device=DEV)
    synth.dev_normal_bf16_rows(d, k, 512 * 7, synth.TSTRIDE * 512, 3, 1536, f32_dev(chan))
    h = synth.normal_bf16_rows(k, 512 * 7, synth.TSTRIDE * 512, 3, 1536, chan)
    assert np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16), h)
    g = torch.empty(2, 77, dtype=torch.float32, device=DEV)
    synth.dev_normal_f32_rows(g, k, 5, synth.TSTRIDE, 2, 77)
    assert np.array_equal(g.cpu().numpy(), synth.normal_f32_rows(k, 5, synth.TSTRIDE, 2, 77))
    u = torch.empty(1000, dtype=torch.float32, device=DEV)
    synth.dev_uniform_f32(u, k, 123)
    assert np.array_equal(u.cpu().numpy(), synth.uniform_f32(k, 123, 1000))
    q = torch.empty(4000, dtype=torch.bfloat16, device=DEV)
    synth.dev_normal_bf16(q, k, 99)
    assert np.array_equal(q.view(torch.int16).cpu().numpy().view(np.uint16), synth.normal_bf16(k, 99, 4000))


# ---------------------------------------------------------------- cache write

@pytest.mark.parametrize("x_f32", [False, True])
def test_pack_bit_exact_with_pending_slot(csa, x_f32):
    wl = W.WORKLOADS[0]  # B=1, 4096 tokens -> 2048 entries
    B, T = 1, wl.T
    dc = csa.engine.DeviceCache(B, 40, 2, DEV, page_seed=5, spare_pages=9)
    rc = oracle.RefCache(B, 40 * 64, 2, W.w_idx(wl, 0))
    Wd = f32_dev(W.w_idx(wl, 0))
    t0 = 0
    for n in [1, 1000, 3, 2047, 1045]:  # odd chunks exercise the pending token
        x = W.tokens(wl, 0, 0, t0, n)[None]
        g = W.gates(wl, 0, 0, t0, n)[None]
        xd = f32_dev(oracle.bf16_to_f32(x).reshape(1, n, 512)) if x_f32 else bf16_dev(x)
        csa.pack_cache(dc.desc, xd, f32_dev(g), Wd)
        rc.append(0, x[0], g[0])
        t0 += n
    torch.cuda.synchronize()
    assert t0 == T and dc.n_entries.item() == rc.n[0] == T // 2
    assert dc.pend_valid.item() == rc.pend_valid[0] == 0
    compare_cache(dc, rc, 0, 0, T // 2)
    assert dc.status_bits() == 0


def test_pack_ratio1_and_outliers_multiseq(csa):
    wl = W.small(W.WORKLOADS[3], B=3, T=333)
    T = wl.T
    for ratio in (1, 2):
        n_ent = T // ratio
        dc = csa.engine.DeviceCache(3, (n_ent + 63) // 64 + 1, ratio, DEV, page_seed=11)
        rc = oracle.RefCache(3, n_ent + 64, ratio, W.w_idx(wl, 0))
        x = np.stack([W.tokens(wl, 0, b, 0, T) for b in range(3)])
        g = np.stack([W.gates(wl, 0, b, 0, T) for b in range(3)])
        csa.pack_cache(dc.desc, bf16_dev(x), f32_dev(g), f32_dev(W.w_idx(wl, 0)))
        for b in range(3):
            rc.append(b, x[b], g[b])
        torch.cuda.synchronize()
        for b in range(3):
            assert dc.n_entries[b].item() == rc.n[b]
            compare_cache(dc, rc, b, b, n_ent)
        if ratio == 2:
            assert np.array_equal(dc.pend_x.cpu().numpy(), rc.pend_x)
            assert np.array_equal(dc.pend_g.cpu().numpy(), rc.pend_g)
            assert np.array_equal(dc.pend_valid.cpu().numpy(), rc.pend_valid)


def _crafted_entries():
    """Latent vectors whose blocks put E4M3 / E2M1 / MXFP4 decisions exactly on
    rounding midpoints (ties) and on saturation, all bf16-representable."""
    e4 = [oracle.e4m3_value(c) for c in range(0x7F)]
    e2mid = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    rows = []
    rng = np.random.default_rng(0)
    for r in range(24):
        e = np.zeros(512, np.float64)
        for j in range(32):
            kind = (r + j) % 4
            s = e4[int(rng.integers(8, 0x60))]
            blk = np.zeros(16)
            if kind == 0:      # E2M1 midpoints, scale exact (6s present)
                blk[0] = 6 * s
                blk[1:8] = np.array(e2mid) * s
                blk[8:15] = -np.array(e2mid) * s
                blk[15] = 0.1 * s
            elif kind == 1:    # E4M3 midpoint: amax/6 halfway between two scales
                c = int(rng.integers(8, 0x70))
                mid = (e4[c] + e4[c + 1]) / 2
                blk[:] = rng.uniform(-1, 1, 16) * mid
                blk[3] = 6 * mid
            elif kind == 2:    # power-of-two scales: MXFP4 ties downstream
                blk[:] = np.array([6, 0.25, 0.75, 1.5, 3, 0.5, 1, 2, 4, 0, 0.25, 0.75, 6, 1, 0.5, 3]) * 2.0 ** (j % 5 - 2)
            else:              # above the E4M3 range: saturation at 448 * 6
                blk[:] = rng.uniform(-3000, 3000, 16)
            e[16 * j:16 * j + 16] = blk
        f = e.astype(np.float32)
        bits = (f.view(np.uint32) >> 16).astype(np.uint16)  # truncation keeps what bf16 holds
        back = (bits.astype(np.uint32) << 16).view(np.float32)
        rows.append(bits if np.array_equal(back, f) else (back.view(np.uint32) >> 16).astype(np.uint16))
    return np.stack(rows)


def test_pack_rounding_ties(csa):
    # equal tokens with equal gates compress to themselves, so the packed
    # values are under direct control; an identity-like W makes the indexer
    # key the first 128 dequantised channels (MXFP4 ties)
    ent = _crafted_entries()
    n = ent.shape[0]
    x = np.repeat(ent, 2, axis=0)[None]           # pairs (v, v)
    g = np.zeros((1, 2 * n), np.float32)
    Wm = np.zeros((512, 128), np.float32)
    Wm[np.arange(128), np.arange(128)] = 1.0
    Wm[200, 5] = 0.5  # plus a few mixed columns
    Wm[300, 77] = -0.25
    dc = csa.engine.DeviceCache(1, 2, 2, DEV)
    csa.pack_cache(dc.desc, bf16_dev(x), f32_dev(g), f32_dev(Wm))
    rc = oracle.RefCache(1, 128, 2, Wm)
    rc.append(0, x[0], g[0])
    torch.cuda.synchronize()
    compare_cache(dc, rc, 0, 0, n)
    # saturated blocks really saturate at 448 * 6
    d = oracle.dequant_main(rc.mc[0, 0], rc.ms[0, 0])
    assert np.abs(d).max() <= 2688


def test_pack_capacity_error_sets_status(csa):
    wl = W.WORKLOADS[0]
    dc = csa.engine.DeviceCache(1, 1, 2, DEV)  # 64 entries
    Wd = f32_dev(W.w_idx(wl, 0))
    x = W.tokens(wl, 0, 0, 0, 140)[None]
    g = W.gates(wl, 0, 0, 0, 140)[None]
    csa.pack_cache(dc.desc, bf16_dev(x[:, :100]), f32_dev(g[:, :100]), Wd)  # 50 entries
    torch.cuda.synchronize()
    assert dc.n_entries.item() == 50 and dc.status_bits() == 0
    csa.pack_cache(dc.desc, bf16_dev(x[:, 100:]), f32_dev(g[:, 100:]), Wd)  # 20 more: full
    torch.cuda.synchronize()
    assert dc.status_bits() & csa.DEVERR_CAPACITY
    assert dc.n_entries.item() == 50  # that sequence is left unchanged
    # an append more than twice the capacity is refused on the host, nothing launched
    with pytest.raises(csa.Csa2Error):
        csa.pack_cache(dc.desc, bf16_dev(W.tokens(wl, 0, 0, 0, 200)[None]),
                       f32_dev(W.gates(wl, 0, 0, 0, 200)[None]), Wd)


# ---------------------------------------------------------------- indexer

def _dev_cache_from_recipe(csa, wl, s, T, page_seed=None):
    r = wl.table.ratios[s]
    max_pages = (T // r + 63) // 64 + 1
    dc = csa.engine.DeviceCache(wl.B, max_pages, r, DEV, page_seed=page_seed)
    x = np.stack([W.tokens(wl, s, b, 0, T) for b in range(wl.B)])
    g = np.stack([W.gates(wl, s, b, 0, T) for b in range(wl.B)])
    csa.pack_cache(dc.desc, bf16_dev(x), f32_dev(g), f32_dev(W.w_idx(wl, s)))
    return dc


@pytest.mark.parametrize("B,T,H_idx,K", [(1, 4096, 4, 256), (3, 1401, 64, 512), (2, 2000, 64, 1024),
                                         (2, 256, 16, 100)])
def test_index_topk_parity(csa, B, T, H_idx, K):
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H_idx=H_idx, K=K)
    dc = _dev_cache_from_recipe(csa, wl, 0, T, page_seed=3)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    q = W.query_idx(wl, 0, 0)
    w = W.head_weights(wl, 0, 0)
    idx = torch.empty(B, K, dtype=torch.int32, device=DEV)
    sc = torch.empty(B, K, dtype=torch.float32, device=DEV)
    ws = torch.empty(csa.index_topk_workspace(B, dc.max_pages * 64, H_idx, K), dtype=torch.uint8, device=DEV)
    csa.index_topk(dc.desc, bf16_dev(q), f32_dev(w), K, idx, ws, score_out=sc)
    torch.cuda.synchronize()
    n = T // 2
    compare_cache(dc, rc, 0, 0, n)
    for b in range(B):
        ref = rc.scores(b, q[b], w[b])
        gi = idx[b].cpu().numpy()
        check_topk(gi, ref, K)
        m = min(K, n)
        got = sc[b].cpu().numpy()[:m].astype(np.float64)
        want = ref[gi[:m]]
        assert np.all(np.abs(got - want) <= 1e-5 * np.maximum(np.abs(want), 1e-6)), "scores"


def test_index_topk_empty_and_short(csa):
    wl = W.small(W.WORKLOADS[0], B=2, T=0)
    dc = csa.engine.DeviceCache(2, 2, 2, DEV)
    q = W.query_idx(wl, 0, 0)
    w = W.head_weights(wl, 0, 0)
    K = 16
    idx = torch.zeros(2, K, dtype=torch.int32, device=DEV)
    ws = torch.empty(csa.index_topk_workspace(2, 128, wl.H_idx, K), dtype=torch.uint8, device=DEV)
    csa.index_topk(dc.desc, bf16_dev(q), f32_dev(w), K, idx, ws)
    torch.cuda.synchronize()
    assert (idx.cpu().numpy() == -1).all()
    # five entries, K = 16: all five then padding
    x = np.stack([W.tokens(wl, 0, b, 0, 11) for b in range(2)])
    g = np.stack([W.gates(wl, 0, b, 0, 11) for b in range(2)])
    csa.pack_cache(dc.desc, bf16_dev(x), f32_dev(g), f32_dev(W.w_idx(wl, 0)))
    csa.index_topk(dc.desc, bf16_dev(q), f32_dev(w), K, idx, ws)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    assert (got[:, :5] == np.arange(5)).all() and (got[:, 5:] == -1).all()


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("H,K,win_count", [(16, 256, 4096), (64, 512, 5), (8, 100, 1), (16, 0, 300)])
def test_sparse_attn_parity(csa, H, K, win_count):
    B, T = 2, 2 * max(K, 8) + 50
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H=H, K=max(K, 1))
    dc = _dev_cache_from_recipe(csa, wl, 0, T)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    n = T // 2
    rng = np.random.default_rng(K)
    idx = np.full((B, max(K, 1)), -1, np.int32)
    for b in range(B):
        sel = np.sort(rng.choice(n, size=min(K, n) - 3 if K > 3 else K, replace=False))
        idx[b, :sel.size] = sel
        if K > 3:
            idx[b, sel.size] = n + 7  # beyond n_entries: skipped
    win = csa.engine.DeviceWindow(B, DEV)
    rings = []
    for b in range(B):
        ring, cnt = ref_window(wl, 0, b, win_count)
        rings.append(ring)
        win.tokens[b] = bf16_dev(ring)
    win.count.fill_(win_count)
    q = W.query(wl, 0, 0)
    out = torch.empty(B, H, 512, dtype=torch.float32, device=DEV)
    ws = torch.empty(csa.sparse_attn_workspace(B, H, K), dtype=torch.uint8, device=DEV)
    idx_d = torch.from_numpy(idx).to(DEV)
    csa.sparse_attn(dc.desc if K else None, bf16_dev(q), idx_d, K, win.desc, wl.scale, out, ws)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    wl_len = min(win_count, 128)
    for b in range(B):
        items = oracle.attention_items(rc.mc[b], rc.ms[b], n, idx[b, :K], rings[b], wl_len)
        ref = oracle.attention(q[b], items, wl.scale)
        assert attn_rel_err(o[b], ref) <= ATTN_REL


@pytest.mark.parametrize("H,K,win_count,qexp", [(64, 512, 130, 17), (16, 100, 5, 17), (64, 256, 40, -20)])
def test_sparse_attn_query_magnitude(csa, H, K, win_count, qexp):
    """Queries 2^qexp times larger (|q| near 1e5, beyond fp16's range) or smaller
    (near fp16's subnormals) with the scale 2^-qexp times smaller: the same
    softmax, so the same output within the usual tolerance."""
    B, T = 2, 2 * K + 50
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H=H, K=K)
    dc = _dev_cache_from_recipe(csa, wl, 0, T)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    n = T // 2
    rng = np.random.default_rng(K + 1)
    idx = np.stack([np.sort(rng.choice(n, size=K, replace=False)) for _ in range(B)]).astype(np.int32)
    win = csa.engine.DeviceWindow(B, DEV)
    rings = []
    for b in range(B):
        ring, _ = ref_window(wl, 0, b, win_count)
        rings.append(ring)
        win.tokens[b] = bf16_dev(ring)
    win.count.fill_(win_count)
    q0 = np.asarray(W.query(wl, 0, 0), np.uint16)
    f = (q0.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** qexp)
    q = (f.view(np.uint32) >> 16).astype(np.uint16)  # exact: a power-of-two multiple of bf16 values
    assert np.array_equal((q.astype(np.uint32) << 16).view(np.float32), f)
    scale = float(np.float32(wl.scale) * np.float32(2.0 ** -qexp))
    out = torch.empty(B, H, 512, dtype=torch.float32, device=DEV)
    ws = torch.empty(csa.sparse_attn_workspace(B, H, K), dtype=torch.uint8, device=DEV)
    csa.sparse_attn(dc.desc, bf16_dev(q), torch.from_numpy(idx).to(DEV), K, win.desc, scale, out, ws)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    assert np.isfinite(o).all()
    for b in range(B):
        items = oracle.attention_items(rc.mc[b], rc.ms[b], n, idx[b], rings[b], min(win_count, 128))
        ref = oracle.attention(q[b], items, scale)
        assert attn_rel_err(o[b], ref) <= ATTN_REL


def test_sparse_attn_cuda_core_selected_at_64_heads(csa, monkeypatch):
    """CSA2_ATTN_CUDA_CORE=1 runs the CUDA-core kernel at 64 heads (the tensor-core
    one's comparison point): same parity bar, workspace sized for it."""
    monkeypatch.setenv("CSA2_ATTN_CUDA_CORE", "1")
    test_sparse_attn_parity(csa, 64, 512, 130)


def test_sparse_attn_tail_tiles_merged(csa):
    """More (sequence) units than SMs: after one unit per CTA, the remaining
    units run tile by tile as partials merged by the tail kernel; every
    sequence, those included, matches the oracle."""
    B, T, K, H, wc = 150, 600, 256, 16, 40
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H=H, K=K)
    dc = _dev_cache_from_recipe(csa, wl, 0, T)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    n = T // 2
    rng = np.random.default_rng(7)
    idx = np.stack([np.sort(rng.choice(n, size=K, replace=False)) for _ in range(B)]).astype(np.int32)
    win = csa.engine.DeviceWindow(B, DEV)
    rings = []
    for b in range(B):
        ring, _ = ref_window(wl, 0, b, wc)
        rings.append(ring)
        win.tokens[b] = bf16_dev(ring)
    win.count.fill_(wc)
    q = W.query(wl, 0, 0)
    out = torch.empty(B, H, 512, dtype=torch.float32, device=DEV)
    ws = torch.empty(max(csa.sparse_attn_workspace(B, H, K), 16), dtype=torch.uint8, device=DEV)
    csa.sparse_attn(dc.desc, bf16_dev(q), torch.from_numpy(idx).to(DEV), K, win.desc, wl.scale, out, ws)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    for b in (0, 1, 146, 147, 148, 149):
        items = oracle.attention_items(rc.mc[b], rc.ms[b], n, idx[b], rings[b], wc)
        assert attn_rel_err(o[b], oracle.attention(q[b], items, wl.scale)) <= ATTN_REL, b


def test_sparse_attn_window_beyond_fp16_saturates(csa):
    """Tensor-core attention: bf16 window values beyond fp16's range saturate at
    +-65504 (the header's contract): outputs stay finite and equal the oracle's
    on the clamped window."""
    B, T, K, H, wc = 2, 600, 128, 64, 20
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H=H, K=K)
    dc = _dev_cache_from_recipe(csa, wl, 0, T)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    n = T // 2
    rng = np.random.default_rng(11)
    idx = np.stack([np.sort(rng.choice(n, size=K, replace=False)) for _ in range(B)]).astype(np.int32)
    win = csa.engine.DeviceWindow(B, DEV)
    rings, clamped = [], []
    for b in range(B):
        ring, _ = ref_window(wl, 0, b, wc)
        f = (np.asarray(ring, np.uint16).astype(np.uint32) << 16).view(np.float32).copy()
        f[3, :64] *= np.float32(2.0 ** 20)   # one token with channels near 1e5 .. 1e6
        bits = (f.view(np.uint32) >> 16).astype(np.uint16)
        rings.append(bits)
        c = np.clip((bits.astype(np.uint32) << 16).view(np.float32), -65504.0, 65504.0)
        clamped.append(c)
        win.tokens[b] = bf16_dev(bits)
    win.count.fill_(wc)
    q = W.query(wl, 0, 0)
    scale = float(np.float32(wl.scale) * np.float32(2.0 ** -12))  # keep the softmax away from one-hot
    out = torch.empty(B, H, 512, dtype=torch.float32, device=DEV)
    ws = torch.empty(max(csa.sparse_attn_workspace(B, H, K), 16), dtype=torch.uint8, device=DEV)
    csa.sparse_attn(dc.desc, bf16_dev(q), torch.from_numpy(idx).to(DEV), K, win.desc, scale, out, ws)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    assert np.isfinite(o).all()
    for b in range(B):
        items = oracle.attention_items(rc.mc[b], rc.ms[b], n, idx[b], rings[b], wc)
        items[K:K + wc] = clamped[b][:wc]  # the window rows as the kernel reads them
        assert attn_rel_err(o[b], oracle.attention(q[b], items, scale)) <= ATTN_REL


def test_window_append_ring(csa):
    B = 3
    win = csa.engine.DeviceWindow(B, DEV)
    win.count.copy_(torch.tensor([0, 127, 300], dtype=torch.int32))
    tok = torch.randn(B, 512, device=DEV).to(torch.bfloat16)
    csa.window_append(win.desc, tok)
    torch.cuda.synchronize()
    assert win.count.cpu().tolist() == [1, 128, 301]
    for b, slot in enumerate([0, 127, 300 % 128]):
        assert torch.equal(win.tokens[b, slot], tok[b])


# ---------------------------------------------------------------- layer step

def _reindex16_table():
    """16 layers over one ratio-2 source: Full, 13 Reindex, 2 Reuse.  Fourteen
    scans read one cache, more than one grouped work item holds (two subsets of
    seven problems, each ending in a single-problem MMA pass)."""
    mode = (W.FULL,) + (W.REINDEX,) * 13 + (W.REUSE,) * 2
    return W.ModeTable(mode, (0,) * 16, tuple(range(14)) + (13, 13), (2,))


@pytest.mark.parametrize("table_name,H_idx", [("alternating", 16), ("pages", 16), ("alternating", 64),
                                              ("pages", 64), ("reindex16", 64)])
def test_layer_step_parity(csa, table_name, H_idx):
    table = {"alternating": W.schedule_alternating_40, "pages": W.schedule_pages_40,
             "reindex16": _reindex16_table}[table_name]()
    wl = W.Workload("small40", 7, 2, 601, table, 8, H_idx, 64, 3)
    dm = csa.engine.DecodeModel(wl, DEV, page_seed=21)
    dm.fill(chunk_tokens=256)
    rm = ref_model(wl)
    for st in range(wl.steps):
        dm.gen_step_inputs(st)
        dm.step()
        torch.cuda.synchronize()
        out_ref, idx_ref = rm.step(**step_inputs(wl, st))
        gidx = dm.idx.cpu().numpy()
        gout = dm.out.cpu().numpy()
        for l in range(table.n_layers):
            m = table.mode[l]
            for b in range(wl.B):
                if m in (W.FULL, W.REINDEX):
                    c = rm.caches[table.src[l]]
                    ref_scores = c.scores(b, W.query_idx(wl, l, st)[b], W.head_weights(wl, l, st)[b])
                    check_topk(gidx[l, b], ref_scores, wl.K)
                # attention checked on the GPU's own indices
                src_l = table.idx_src[l] if m == W.REUSE else l
                if m == W.SWA_ONLY:
                    ref = rm.layer_attention(l, b, W.query(wl, l, st)[b], None)
                else:
                    ref = rm.layer_attention(l, b, W.query(wl, l, st)[b], gidx[src_l, b])
                assert attn_rel_err(gout[l, b], ref) <= ATTN_REL, (l, b)
        for s in range(table.n_sources):
            n = int(rm.caches[s].n[0])
            for b in range(wl.B):
                assert dm.caches[s].n_entries[b].item() == rm.caches[s].n[b]
                compare_cache(dm.caches[s], rm.caches[s], b, b, n)
    assert dm.status_bits() == 0
