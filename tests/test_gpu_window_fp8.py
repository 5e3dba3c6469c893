"""GPU parity of the FP8 SWA window (E4M3 codes, 512 B a token) against the
oracle: the ring write bit-exact, attention over an FP8 window on both attention
paths (tcgen05 up to 64 heads, CUDA cores above), and the layer step with FP8
windows.  All calls go through the C ABI."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
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


def _bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_window_append_fp8_codes_bit_exact(csa):
    B = 3
    win = csa.engine.DeviceWindow(B, DEV, fp8=True)
    win.count.copy_(torch.tensor([0, 120, 300], dtype=torch.int32))
    rng = np.random.default_rng(8)
    special = np.array([0.0, -0.0, 448.0, 464.0, 1e6, -1e6, 2.0 ** -10, -(2.0 ** -10), 1.0625, 1.1875,
                        2.0 ** -9, 2.0 ** -7 * 1.5, -240.0, 3e38], np.float32)
    toks = []
    for i in range(10):  # wraps the second ring
        x = (rng.normal(size=(B, 512)) * 10 ** rng.uniform(-4, 2.7, (B, 512))).astype(np.float32)
        x[:, :special.size] = special
        t = _bf16(x)
        toks.append(t)
        csa.window_append(win.desc, bf16_dev(t))
    torch.cuda.synchronize()
    assert win.count.cpu().tolist() == [10, 130, 310]
    ring = win.tokens.cpu().numpy()
    for b, c0 in enumerate([0, 120, 300]):
        for i in range(10):
            assert np.array_equal(ring[b, (c0 + i) % 128], oracle.window_fp8(toks[i][b])), (b, i)


@pytest.mark.parametrize("H,K,win_count", [(64, 512, 300), (16, 256, 5), (100, 64, 200), (64, 0, 128)])
def test_sparse_attn_fp8_window_parity(csa, H, K, win_count):
    B, T = 2, 2 * max(K, 8) + 50
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H=H, K=max(K, 1))
    max_pages = (T // 2 + 63) // 64 + 1
    dc = csa.engine.DeviceCache(B, max_pages, 2, DEV, page_seed=4)
    x = np.stack([W.tokens(wl, 0, b, 0, T) for b in range(B)])
    g = np.stack([W.gates(wl, 0, b, 0, T) for b in range(B)])
    csa.pack_cache(dc.desc, bf16_dev(x), f32_dev(g), f32_dev(W.w_idx(wl, 0)))
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    n = T // 2
    rng = np.random.default_rng(K + 1)
    idx = np.full((B, max(K, 1)), -1, np.int32)
    for b in range(B):
        sel = np.sort(rng.choice(n, size=min(K, n) - 3 if K > 3 else K, replace=False))
        idx[b, :sel.size] = sel
    # the window: the last min(win_count, 128) tokens appended through the library
    win = csa.engine.DeviceWindow(B, DEV, fp8=True)
    wlen = min(win_count, 128)
    win.count.fill_(win_count - wlen)
    for p in range(win_count - wlen, win_count):
        tok = np.stack([W.window_tokens(wl, 0, b, p, 1)[0] for b in range(B)])
        csa.window_append(win.desc, bf16_dev(tok))
    q = W.query(wl, 0, 0)
    out = torch.empty(B, H, 512, dtype=torch.float32, device=DEV)
    ws = torch.empty(csa.sparse_attn_workspace(B, H, K), dtype=torch.uint8, device=DEV)
    csa.sparse_attn(dc.desc if K else None, bf16_dev(q), torch.from_numpy(idx).to(DEV), K, win.desc, wl.scale,
                    out, ws)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    for b in range(B):
        ring, _ = ref_window(wl, 0, b, win_count)
        items = oracle.attention_items_fp8(rc.mc[b], rc.ms[b], n, idx[b, :K], oracle.window_fp8(ring), wlen)
        ref = oracle.attention(q[b], items, wl.scale)
        assert attn_rel_err(o[b], ref) <= ATTN_REL


@pytest.mark.parametrize("table_name,H_idx", [("alternating", 64), ("pages", 16)])
def test_layer_step_fp8_windows(csa, table_name, H_idx):
    table = {"alternating": W.schedule_alternating_40, "pages": W.schedule_pages_40}[table_name]()
    wl = W.Workload("small40w8", 3, 2, 611, table, 8, H_idx, 48, 2, win_fp8=True)
    dm = csa.engine.DecodeModel(wl, DEV, page_seed=17)
    dm.fill(chunk_tokens=256)
    rm = ref_model(wl)
    for l in range(table.n_layers):  # the filled rings hold the oracle's codes
        assert np.array_equal(dm.windows[l].tokens.cpu().numpy(), rm.win8[l]), l
    for st in range(wl.steps):
        dm.gen_step_inputs(st)
        dm.step()
        torch.cuda.synchronize()
        inp = step_inputs(wl, st)
        rm.step(**inp)
        gidx = dm.idx.cpu().numpy()
        gout = dm.out.cpu().numpy()
        for l in range(table.n_layers):
            m = table.mode[l]
            assert np.array_equal(dm.windows[l].tokens.cpu().numpy(), rm.win8[l]), (st, l)
            for b in range(wl.B):
                if m in (W.FULL, W.REINDEX):
                    c = rm.caches[table.src[l]]
                    check_topk(gidx[l, b], c.scores(b, inp["qidx"][l][b], inp["wh"][l][b]), wl.K)
                src_l = table.idx_src[l] if m == W.REUSE else l
                idx_l = None if m == W.SWA_ONLY else gidx[src_l, b]
                ref = rm.layer_attention(l, b, inp["q"][l][b], idx_l)
                assert attn_rel_err(gout[l, b], ref) <= ATTN_REL, (l, b)
    assert dm.status_bits() == 0
