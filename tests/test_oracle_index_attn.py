"""Pins of the oracle's indexer scan, Top-K, attention and mode-table semantics."""
import numpy as np
import pytest
from scipy.special import softmax

from fp4_sparse_attention_pack_b200 import workloads as W


def _bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _keys(ref, rng, N):
    kc = np.zeros((N, 64), np.uint8)
    ks = np.zeros((N, 4), np.uint8)
    for e in range(N):
        kc[e], ks[e] = ref.mxfp4_quant(rng.normal(size=128).astype(np.float32))
    return kc, ks


def test_scores_brute_force(ref):
    # matrix form with a library matmul over the dequantised MXFP4 operands
    rng = np.random.default_rng(0)
    N, H = 37, 5
    kc, ks = _keys(ref, rng, N)
    q = _bf16(rng.normal(size=(H, 128)))
    w = rng.uniform(0, 1, H).astype(np.float32)
    got = ref.index_scores(kc, ks, N, q, w)
    qc, qs = ref.quantize_queries(q)
    Qd = np.stack([ref.mxfp4_dequant(qc[h], qs[h]) for h in range(H)])
    Kd = np.stack([ref.mxfp4_dequant(kc[e], ks[e]) for e in range(N)])
    want = np.maximum(Kd @ Qd.T, 0.0) @ w.astype(np.float64)
    np.testing.assert_allclose(got, want, rtol=1e-13)


def test_scores_relu_all_negative(ref):
    rng = np.random.default_rng(1)
    kc, ks = ref.mxfp4_quant(np.abs(rng.normal(size=128)).astype(np.float32))
    q = _bf16(-np.abs(rng.normal(size=(3, 128))))
    s = ref.index_scores(kc[None], ks[None], 1, q, np.ones(3, np.float32))
    assert s[0] == 0.0


def test_topk_equals_full_sort(ref):
    rng = np.random.default_rng(2)
    for N, K in [(10, 4), (50, 50), (7, 12), (1, 1), (64, 16), (300, 37)]:
        s = rng.integers(0, 6, N).astype(np.float64)  # many forced ties
        got = ref.topk(s, K)
        order = sorted(range(N), key=lambda i: (-s[i], i))[:min(K, N)]
        assert list(got[:len(order)]) == sorted(order)
        assert np.all(got[len(order):] == -1)
    assert np.all(ref.topk(np.zeros(0), 5) == -1)


def test_attention_single_item_and_uniform(ref):
    rng = np.random.default_rng(3)
    q = _bf16(rng.normal(size=(4, 512)))
    item = rng.normal(size=(1, 512)).astype(np.float32)
    out = ref.attention(q, item, 0.044)
    assert np.array_equal(out, np.repeat(item, 4, 0))
    items = rng.normal(size=(9, 512)).astype(np.float32)
    out = ref.attention(np.zeros((2, 512), np.uint16), items, 0.044)
    np.testing.assert_allclose(out, np.repeat(items.astype(np.float64).mean(0, keepdims=True), 2, 0),
                               rtol=1e-6, atol=1e-7)
    assert not ref.attention(q, np.zeros((0, 512), np.float32), 0.1).any()


def test_attention_matches_softmax_matrix_form(ref):
    rng = np.random.default_rng(4)
    for M in (1, 5, 130):
        q = _bf16(rng.normal(size=(6, 512)))
        items = (rng.normal(size=(M, 512)) * 3).astype(np.float32)
        sc = 1 / np.sqrt(512)
        qf = ref.bf16_to_f32(q).reshape(6, 512).astype(np.float64)
        P = softmax(sc * qf @ items.T.astype(np.float64), axis=1)
        np.testing.assert_allclose(ref.attention(q, items, sc), P @ items, rtol=1e-5, atol=1e-6)


def test_gather_items_skips_padding_and_counts_window(ref):
    rng = np.random.default_rng(5)
    mc = rng.integers(0, 256, (6, 256)).astype(np.uint8)
    ms = rng.integers(0, 0x7F, (6, 32)).astype(np.uint8)
    win = _bf16(rng.normal(size=(128, 512)))
    items = ref.attention_items(mc, ms, 6, np.array([4, -1, 0, -1], np.int32), win, 3)
    assert items.shape == (5, 512)
    assert np.array_equal(items[0], ref.dequant_main(mc[4], ms[4]))
    assert np.array_equal(items[1], ref.dequant_main(mc[0], ms[0]))
    assert np.array_equal(items[2:], ref.bf16_to_f32(win[:3]).reshape(3, 512))


def _tiny_model(ref, table, B=2, T=40, H=4, Hi=4, K=6, seed=11):
    rng = np.random.default_rng(seed)
    Ws = [(rng.normal(size=(512, 128)) / np.sqrt(512)).astype(np.float32) for _ in table.ratios]
    m = ref.RefModel(table, B, [64] * table.n_sources, Ws, H, Hi, K, 1 / np.sqrt(512))
    for s in range(table.n_sources):
        for b in range(B):
            m.caches[s].append(b, _bf16(rng.normal(size=(T, 512))), rng.normal(size=T).astype(np.float32))
    L = table.n_layers
    inputs = dict(
        x_new=[[_bf16(rng.normal(size=512)) for _ in range(B)] for _ in table.ratios],
        g_new=[rng.normal(size=B).astype(np.float32) for _ in table.ratios],
        q=[[_bf16(rng.normal(size=(H, 512))) for _ in range(B)] for _ in range(L)],
        qidx=[[_bf16(rng.normal(size=(Hi, 128))) for _ in range(B)] for _ in range(L)],
        wh=[[rng.uniform(0, 1, Hi).astype(np.float32) for _ in range(B)] for _ in range(L)],
        wtok=[[_bf16(rng.normal(size=512)) for _ in range(B)] for _ in range(L)],
    )
    return m, inputs


def test_modes_reuse_and_reindex(ref):
    t = W.ModeTable((W.SWA_ONLY, W.FULL, W.REINDEX, W.REUSE, W.REINDEX), (-1, 0, 0, 0, 0),
                    (-1, 1, 2, 2, 4), (2,))
    m, inp = _tiny_model(ref, t)
    # layer 4 (Reindex) gets layer 1's (Full) indexer query: same indices
    inp["qidx"][4] = inp["qidx"][1]
    inp["wh"][4] = inp["wh"][1]
    out, idx = m.step(**inp)
    for b in range(2):
        assert idx[0][b] is None
        assert np.array_equal(idx[3][b], idx[2][b])   # Reuse = its source's indices
        assert np.array_equal(idx[4][b], idx[1][b])   # Reindex with the Full query
        assert all(out[l][b] is not None for l in range(5))
    # Reuse attention equals attention over the source's selection with its own q/window
    wl = m.win_len(3, 0)
    c = m.caches[0]
    items = ref.attention_items(c.mc[0], c.ms[0], int(c.n[0]), idx[2][0], m.win[3, 0], wl)
    assert np.array_equal(out[3][0], ref.attention(inp["q"][3][0], items, m.scale))


def test_mode_table_validation(ref):
    bad = W.ModeTable((W.REUSE, W.FULL), (0, 0), (1, 1), (2,))
    with pytest.raises(ValueError):
        _tiny_model(ref, bad)


def test_swa_only_reads_only_the_window(ref):
    t = W.ModeTable((W.SWA_ONLY,), (-1,), (-1,), (2,))
    m, inp = _tiny_model(ref, t, B=1)
    out, _ = m.step(**inp)
    items = ref.bf16_to_f32(m.win[0, 0, :1]).reshape(1, 512)
    assert np.array_equal(out[0][0], np.repeat(items, 4, 0))  # one window token: output = token
