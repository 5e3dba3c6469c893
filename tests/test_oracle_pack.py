"""Pins of the oracle's cache write: compression, main pack, projection, MXFP4 keys,
pending-slot bookkeeping and the pages' byte accounting."""
import numpy as np
import pytest

from fp4_sparse_attention_pack_b200 import workloads as W


def _e2m1_vals(ref):
    return np.array([ref.e2m1_value(c) for c in range(16)])


def test_compress_equal_gates_is_mean(ref):
    rng = np.random.default_rng(0)
    x0, x1 = rng.normal(size=512).astype(np.float32), rng.normal(size=512).astype(np.float32)
    for g in (0.0, 1.7, -3.25):
        e = ref.compress_pair(x0, g, x1, g)
        assert np.array_equal(e, ((x0.astype(np.float64) + x1) / 2).astype(np.float32))


def test_compress_saturated_gates_pick_one_token(ref):
    rng = np.random.default_rng(1)
    x0, x1 = rng.normal(size=512).astype(np.float32), rng.normal(size=512).astype(np.float32)
    assert np.array_equal(ref.compress_pair(x0, 30.0, x1, 0.0), x0)
    e = ref.compress_pair(x0, 0.0, x1, 30.0)
    np.testing.assert_allclose(e, x1, rtol=2 ** -22, atol=1e-12)


def test_compress_is_softmax_weighted_sum(ref):
    rng = np.random.default_rng(2)
    for _ in range(20):
        x0, x1 = rng.normal(size=512).astype(np.float32), rng.normal(size=512).astype(np.float32)
        g0, g1 = rng.normal(size=2).astype(np.float32)
        w = np.exp([float(g0), float(g1)])
        w /= w.sum()
        np.testing.assert_allclose(ref.compress_pair(x0, g0, x1, g1), w[0] * x0 + w[1] * x1,
                                   rtol=1e-6, atol=1e-6)


def test_pack_roundtrip_of_representable_blocks(ref):
    # a block whose values are E2M1 x s, with 6s present, packs back to itself exactly
    rng = np.random.default_rng(3)
    vals = _e2m1_vals(ref)
    e4 = np.array([ref.e4m3_value(c) for c in range(0x7F)])
    e = np.zeros(512, np.float32)
    want_scales = np.zeros(32, np.uint8)
    for j in range(32):
        sc = int(rng.integers(1, 0x7F))
        s = e4[sc]
        codes = rng.integers(0, 16, 16)
        codes[rng.integers(0, 16)] = rng.choice([7, 15])  # +-6 present
        e[16 * j:16 * j + 16] = vals[codes] * s
        want_scales[j] = sc
    codes, scales = ref.pack_main(e)
    assert np.array_equal(scales, want_scales)
    d = ref.dequant_main(codes, scales)
    assert np.array_equal(d, e) or np.array_equal(np.abs(d), np.abs(e))
    assert np.array_equal(d[e != 0], e[e != 0])


def test_pack_error_bound_with_outliers(ref):
    # |x - xhat| <= half the E2M1 spacing at x/s, times s, unless x/s saturates
    rng = np.random.default_rng(4)
    for trial in range(30):
        e = rng.normal(size=512).astype(np.float32)
        if trial % 3 == 0:
            e[rng.choice(512, 5, replace=False)] *= 64.0
        codes, scales = ref.pack_main(e)
        d = ref.dequant_main(codes, scales)
        for j in range(32):
            s = ref.e4m3_value(int(scales[j]))
            blk = slice(16 * j, 16 * j + 16)
            r = np.abs(e[blk].astype(np.float64)) / s
            half = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
            err = np.abs(d[blk].astype(np.float64) - e[blk])
            ok = (err <= half * s * (1 + 1e-6)) | (r > 6)
            assert ok.all()
            # saturation only when the scale was rounded down; then xhat = +-6s
            sat = r > 6
            assert np.all(np.abs(d[blk][sat]) == 6 * s)


def test_pack_tiny_block_scale_zero(ref):
    e = np.zeros(512, np.float32)
    e[:16] = 1e-3  # amax / 6 below half the smallest E4M3 subnormal
    codes, scales = ref.pack_main(e)
    assert scales[0] == 0 and not codes[:8].any()


def test_dequant_is_exact_product(ref):
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, 256).astype(np.uint8)
    scales = rng.integers(0, 0x7F, 32).astype(np.uint8)
    d = ref.dequant_main(codes, scales)
    vals = _e2m1_vals(ref)
    lo, hi = codes & 15, codes >> 4
    q = np.empty(512, np.int64)
    q[0::2], q[1::2] = lo, hi
    want = vals[q] * np.repeat([ref.e4m3_value(int(s)) for s in scales], 16)
    assert np.array_equal(d.astype(np.float64), want)


def test_bits_per_channel_and_entry_bytes(ref, golden):
    codes, scales = ref.pack_main(np.ones(512, np.float32))
    kc, ks = ref.mxfp4_quant(np.ones(128, np.float32))
    assert (codes.size, scales.size) == (golden["main_code_bytes"]["value"], golden["main_scale_bytes"]["value"])
    assert (kc.size, ks.size) == (golden["idx_code_bytes"]["value"], golden["idx_scale_bytes"]["value"])
    assert codes.size + scales.size == golden["main_entry_bytes"]["value"]
    assert kc.size + ks.size == golden["idx_entry_bytes"]["value"]
    assert (codes.size + scales.size) * 8 / 512 == golden["bits_per_channel_main"]["value"]
    assert (kc.size + ks.size) * 8 / 128 == golden["bits_per_channel_idx"]["value"]
    assert golden["v4_fp8_entry_bytes"]["value"] == 512 * 8 // 8


def test_global_cache_bytes_per_token(ref, golden):
    # recompute the pages' 890 B/token from the mode table and the packed sizes
    codes, scales = ref.pack_main(np.ones(512, np.float32))
    kc, ks = ref.mxfp4_quant(np.ones(128, np.float32))
    entry = codes.size + scales.size + kc.size + ks.size
    t = W.schedule_pages_40()
    writers = [l for l, m in enumerate(t.mode) if m == W.FULL]
    assert writers == golden["full_layers"]["value"]
    assert [l for l, m in enumerate(t.mode) if m == W.SWA_ONLY] == golden["swa_only_layers"]["value"]
    assert t.n_layers == golden["n_layers"]["value"]
    per_token = sum(1 / t.ratios[t.src[l]] for l in writers)
    assert per_token == golden["entries_per_token"]["value"]
    assert per_token * entry == golden["global_kv_bytes_per_token"]["value"]
    gib = per_token * entry * golden["cache_gib_at_1m_tokens"]["tokens"] / 2 ** 30
    assert round(gib, 2) == golden["cache_gib_at_1m_tokens"]["value"]
    assert len(t.scan_layers()) == golden["pages_schedule_scans_per_step"]["value"]
    # the all-ratio-2 schedule of the 40-layer benchmark: 2 entries per token
    t2 = W.schedule_alternating_40()
    assert sum(1 / t2.ratios[t2.src[l]] for l, m in enumerate(t2.mode) if m == W.FULL) * entry == 712
    assert len(t2.scan_layers()) == 23


def test_mode_tables_follow_the_page_table(golden):
    # Full computes all three; Reindex recomputes only the indices; Reuse nothing
    for t in (W.schedule_pages_40(), W.schedule_alternating_40()):
        for l, m in enumerate(t.mode):
            if m == W.FULL:
                assert t.idx_src[l] == l and t.src[l] in range(t.n_sources)
            elif m == W.REINDEX:
                assert t.idx_src[l] == l and t.mode[[j for j in range(l) if t.src[j] == t.src[l]][0]] == W.FULL
            elif m == W.REUSE:
                j = t.idx_src[l]
                assert j < l and t.mode[j] in (W.FULL, W.REINDEX) and t.src[j] == t.src[l]
                assert all(t.mode[i] == W.REUSE for i in range(j + 1, l))
    assert golden["mode_table"]["value"]["reuse"] == ["reused"] * 3


def test_projection_column_selection_is_exact(ref):
    rng = np.random.default_rng(6)
    e = rng.normal(size=512).astype(np.float32)
    codes, scales = ref.pack_main(e)
    deq = ref.dequant_main(codes, scales)
    sel = rng.choice(512, 128, replace=False)
    Wm = np.zeros((512, 128), np.float32)
    Wm[sel, np.arange(128)] = 1.0
    kc, ks = ref.index_key(codes, scales, Wm)
    # a sum starting from +0 turns -0 into +0 (IEEE), hence the + 0.0
    want_c, want_s = ref.mxfp4_quant(deq[sel] + np.float32(0.0))
    assert np.array_equal(kc, want_c) and np.array_equal(ks, want_s)
    # with a power-of-two weight the projection is still exact
    Wm[sel, np.arange(128)] = 0.25
    kc, ks = ref.index_key(codes, scales, Wm)
    want_c, want_s = ref.mxfp4_quant(deq[sel] * np.float32(0.25) + np.float32(0.0))
    assert np.array_equal(kc, want_c) and np.array_equal(ks, want_s)


def test_projection_close_to_fp64_matmul(ref):
    rng = np.random.default_rng(8)
    e = rng.normal(size=512).astype(np.float32)
    Wm = (rng.normal(size=(512, 128)) / np.sqrt(512)).astype(np.float32)
    codes, scales = ref.pack_main(e)
    kc, ks = ref.index_key(codes, scales, Wm)
    k64 = ref.dequant_main(codes, scales).astype(np.float64) @ Wm.astype(np.float64)
    kq = ref.mxfp4_dequant(kc, ks)
    # MXFP4 error: at most half an E2M1 step (<= 1 unit at scale 2^X) per element
    X = np.repeat([ref.e8m0_value(int(s)) for s in ks], 32)
    assert np.all(np.abs(kq - k64) <= X * 1.0 + 1e-9)


def test_mxfp4_roundtrip(ref):
    rng = np.random.default_rng(9)
    vals = _e2m1_vals(ref)
    for _ in range(50):
        v = np.zeros(128, np.float32)
        xs = rng.integers(-20, 20, 4)
        for j in range(4):
            c = rng.integers(0, 16, 32)
            c[rng.integers(0, 32)] = rng.choice([6, 7, 14, 15])  # |max| in {4, 6}
            v[32 * j:32 * j + 32] = vals[c] * 2.0 ** xs[j]
        codes, scales = ref.mxfp4_quant(v)
        assert np.array_equal(scales.astype(int) - 127, xs)
        assert np.array_equal(ref.mxfp4_dequant(codes, scales).astype(np.float32)[v != 0], v[v != 0])


def test_mxfp4_zero_block(ref):
    v = np.zeros(64, np.float32)
    v[32:] = 1.0
    codes, scales = ref.mxfp4_quant(v)
    assert scales[0] == 0 and not codes[:16].any()
    assert scales[1] == 127 - 2


def test_append_pending_slot(ref):
    # appending tokens one by one equals appending them all at once (ratio 2 pairs
    # are disjoint and taken in arrival order); ratio 1 makes one entry per token
    rng = np.random.default_rng(10)
    T = 9
    x = (rng.normal(size=(T, 512)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    g = rng.normal(size=T).astype(np.float32)
    Wm = (rng.normal(size=(512, 128)) / 20).astype(np.float32)
    a = ref.RefCache(1, 8, 2, Wm)
    a.append(0, x, g)
    b = ref.RefCache(1, 8, 2, Wm)
    for t in range(T):
        b.append(0, x[t:t + 1], g[t:t + 1])
    assert a.n[0] == b.n[0] == 4 and a.pend_valid[0] == b.pend_valid[0] == 1
    for arr in ("mc", "ms", "kc", "ks"):
        assert np.array_equal(getattr(a, arr), getattr(b, arr))
    xf = ref.bf16_to_f32(x).reshape(T, 512)
    e = ref.compress_pair(xf[2], g[2], xf[3], g[3])
    c, s = ref.pack_main(e)
    assert np.array_equal(a.mc[0, 1], c) and np.array_equal(a.ms[0, 1], s)
    r1 = ref.RefCache(1, 16, 1, Wm)
    r1.append(0, x, g)
    assert r1.n[0] == T
    c, s = ref.pack_main(xf[5])
    assert np.array_equal(r1.mc[0, 5], c) and np.array_equal(r1.ms[0, 5], s)
    with pytest.raises(ValueError):
        ref.RefCache(1, 3, 2, Wm).append(0, x, g)


def test_pack_scale_is_nearest_even_e4m3_of_amax_over_6(ref):
    """The main scale byte is E4M3 round-to-nearest-even of fp32 amax / 6 (the
    reading of "Le cache KV en FP4" in which the scale is the plain NVFP4-style
    nearest value): pinned at every exact midpoint between two adjacent positive
    E4M3 values, one fp32 ulp either side of it, and on the values themselves,
    against the library float8 cast, independently of the GPU path."""
    import torch
    rng = np.random.default_rng(11)
    vals = np.array([ref.e4m3_value(c) for c in range(0x7F)], np.float64)  # 0 .. 448
    amaxes = []
    for k in range(1, 0x7E):
        lo, hi = vals[k], vals[k + 1]
        for target in (lo, (lo + hi) / 2):
            a = np.float32(target * 6.0)  # exact: few significant bits
            assert float(a) == target * 6.0
            amaxes += [a, np.nextafter(a, np.float32(np.inf)), np.nextafter(a, np.float32(0))]
    amaxes = np.array(amaxes, np.float32)
    amaxes = amaxes[(amaxes > 0) & (amaxes / np.float32(6) <= np.float32(448))]
    want = torch.from_numpy(amaxes / np.float32(6)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for i0 in range(0, len(amaxes), 32):
        blk = amaxes[i0:i0 + 32]
        e = np.zeros(512, np.float32)
        for j, a in enumerate(blk):
            # one element carries +-amax, the others are strictly smaller
            v = (rng.random(16) * 0.99 * a).astype(np.float32) * rng.choice([-1, 1], 16)
            v[rng.integers(0, 16)] = a * rng.choice([-1, 1])
            e[16 * j:16 * j + 16] = v
        _, scales = ref.pack_main(e)
        assert np.array_equal(scales[:len(blk)], want[i0:i0 + 32])
    # the midpoints themselves went to the even code (ties-to-even, not round-up)
    mids = np.array([np.float32((vals[k] + vals[k + 1]) / 2 * 6) for k in range(1, 0x7E)], np.float32)
    e = np.zeros(512, np.float32)
    for j in range(32):
        e[16 * j] = mids[j]
    _, scales = ref.pack_main(e)
    for j in range(32):
        assert scales[j] % 2 == 0
