"""GPU parity of the hierarchical sparse indexer against the oracle: the pool a
Full-layer scan builds (csa2_index_topk_pool), the pool-restricted scan and Top-K
of a deeper layer (csa2_index_topk_in_pool) on both scan paths (tcgen05 at 64
indexer heads, CUDA cores otherwise), the edge cases, and the layer step with
pools.  All calls go through the C ABI."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from fp4_sparse_attention_pack_b200 import workloads as W

from .oracle_models import ref_cache, ref_model, step_inputs
from .parity import ATTN_REL, TOPK_REL, attn_rel_err, check_topk, check_topk_in_pool

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


def dev_cache(csa, wl, T, page_seed=5):
    max_pages = (T // 2 + 63) // 64 + 1
    dc = csa.engine.DeviceCache(wl.B, max_pages, 2, DEV, page_seed=page_seed)
    if T > 0:
        x = np.stack([W.tokens(wl, 0, b, 0, T) for b in range(wl.B)])
        g = np.stack([W.gates(wl, 0, b, 0, T) for b in range(wl.B)])
        csa.pack_cache(dc.desc, bf16_dev(x), f32_dev(g), f32_dev(W.w_idx(wl, 0)))
    return dc


def run_pool(csa, dc, wl, P, l_full=0, l_deep=1, pool=None):
    """Full-layer scan with pool, then a deeper layer's scan restricted to it
    (the given pool instead, when one is passed).  Returns host arrays."""
    B, K, cap = wl.B, wl.K, dc.max_pages * 64
    ws = torch.empty(csa.index_pool_workspace(B, cap, wl.H_idx, K, P), dtype=torch.uint8, device=DEV)
    idx = torch.empty(B, K, dtype=torch.int32, device=DEV)
    pool_d = torch.empty(B, P, dtype=torch.int32, device=DEV)
    csa.index_topk_pool(dc.desc, bf16_dev(W.query_idx(wl, l_full, 0)), f32_dev(W.head_weights(wl, l_full, 0)),
                        K, idx, pool_d, ws)
    if pool is not None:
        pool_d = torch.from_numpy(np.ascontiguousarray(pool, np.int32)).to(DEV)
    idx2 = torch.empty(B, K, dtype=torch.int32, device=DEV)
    sc2 = torch.empty(B, K, dtype=torch.float32, device=DEV)
    csa.index_topk_in_pool(dc.desc, bf16_dev(W.query_idx(wl, l_deep, 0)), f32_dev(W.head_weights(wl, l_deep, 0)),
                           K, pool_d, idx2, ws, score_out=sc2)
    torch.cuda.synchronize()
    assert dc.status_bits() == 0
    return idx.cpu().numpy(), pool_d.cpu().numpy(), idx2.cpu().numpy(), sc2.cpu().numpy()


@pytest.mark.parametrize("B,T,H_idx,K,P", [
    (2, 3001, 64, 64, 40),      # tcgen05 scan: ragged last block and tile, pool < blocks
    (3, 1401, 16, 100, 20),     # CUDA-core scan
    (2, 65536, 64, 512, 2048),  # the pages' pool size: 128 gathered tiles per sequence, several items
    (1, 20000, 64, 256, 300),   # pool tiles end in a partial tile (300 * 8 = 2400 positions)
    (2, 777, 64, 32, 3),        # pool smaller than K: padding after 24 entries
])
def test_pool_and_restricted_topk_parity(csa, B, T, H_idx, K, P):
    wl = W.small(W.WORKLOADS[0], B=B, T=T, H_idx=H_idx, K=K)
    dc = dev_cache(csa, wl, T)
    rc = ref_cache(wl, 0, range(B), T, cap=T // 2 + 64)
    idx, pool, idx2, sc2 = run_pool(csa, dc, wl, P)
    n = T // 2
    q0, w0 = W.query_idx(wl, 0, 0), W.head_weights(wl, 0, 0)
    q1, w1 = W.query_idx(wl, 1, 0), W.head_weights(wl, 1, 0)
    for b in range(B):
        s0 = rc.scores(b, q0[b], w0[b])
        check_topk(idx[b], s0, K)                                  # the Full layer's own Top-K
        check_topk(pool[b], oracle.block_maxima(s0), P)            # the pool over block maxima
        s1 = rc.scores(b, q1[b], w1[b])
        cand = oracle.pool_entries(pool[b], n)
        check_topk_in_pool(idx2[b], s1, cand, K)
        m = min(K, cand.size)
        want = s1[idx2[b, :m]]
        assert np.all(np.abs(sc2[b, :m] - want) <= 1e-5 * np.maximum(np.abs(want), 1e-6)), "scores"
        assert np.all(sc2[b, m:] == 0)


def test_pool_covering_every_block_is_plain_topk(csa):
    wl = W.small(W.WORKLOADS[0], B=2, T=2 * 43, H_idx=64, K=16)   # 43 entries: 6 blocks, the last of 3
    dc = dev_cache(csa, wl, wl.T)
    rc = ref_cache(wl, 0, range(2), wl.T, cap=200)
    idx, pool, idx2, _ = run_pool(csa, dc, wl, 10)
    q1, w1 = W.query_idx(wl, 1, 0), W.head_weights(wl, 1, 0)
    for b in range(2):
        assert list(pool[b]) == [0, 1, 2, 3, 4, 5, -1, -1, -1, -1]
        check_topk(idx2[b], rc.scores(b, q1[b], w1[b]), 16)


def test_given_pool_stops_at_blocks_beyond_the_sequence(csa):
    wl = W.small(W.WORKLOADS[0], B=2, T=2 * 43, H_idx=16, K=12)
    dc = dev_cache(csa, wl, wl.T)
    rc = ref_cache(wl, 0, range(2), wl.T, cap=200)
    given = np.array([[1, 3, 1000, -1], [0, 5, -1, -1]], np.int32)   # block 5 holds entries 40..42
    _, _, idx2, _ = run_pool(csa, dc, wl, 4, pool=given)
    q1, w1 = W.query_idx(wl, 1, 0), W.head_weights(wl, 1, 0)
    for b in range(2):
        s1 = rc.scores(b, q1[b], w1[b])
        cand = oracle.pool_entries(given[b], 43)
        assert list(cand) == ([8 + i for i in range(8)] + [24 + i for i in range(8)] if b == 0 else
                              list(range(8)) + [40, 41, 42])
        check_topk_in_pool(idx2[b], s1, cand, 12)


def test_pool_of_empty_sequences(csa):
    wl = W.small(W.WORKLOADS[0], B=2, T=0, H_idx=64, K=8)
    dc = dev_cache(csa, wl, 0)
    idx, pool, idx2, sc2 = run_pool(csa, dc, wl, 5)
    assert (idx == -1).all() and (pool == -1).all() and (idx2 == -1).all() and (sc2 == 0).all()


@pytest.mark.parametrize("table_name,H_idx,P", [("alternating", 64, 12), ("pages", 64, 12), ("alternating", 16, 9)])
def test_layer_step_with_pools(csa, table_name, H_idx, P):
    table = {"alternating": W.schedule_alternating_40, "pages": W.schedule_pages_40}[table_name]()
    wl = W.Workload("small40p", 9, 2, 1203, table, 8, H_idx, 32, 2, pool_blocks=P)
    dm = csa.engine.DecodeModel(wl, DEV, page_seed=13)
    dm.fill(chunk_tokens=256)
    rm = ref_model(wl)
    for st in range(wl.steps):
        dm.gen_step_inputs(st)
        dm.step()
        torch.cuda.synchronize()
        inp = step_inputs(wl, st)
        out_ref, idx_ref = rm.step(**inp)
        gidx = dm.idx.cpu().numpy()
        gout = dm.out.cpu().numpy()
        for l in range(table.n_layers):
            m = table.mode[l]
            for b in range(wl.B):
                if m in (W.FULL, W.REINDEX):
                    c = rm.caches[table.src[l]]
                    s = c.scores(b, inp["qidx"][l][b], inp["wh"][l][b])
                    if m == W.FULL:
                        check_topk(gidx[l, b], s, wl.K)
                    else:
                        # the oracle's pool of this source must be unambiguous for the check
                        lf = _full_of(table, table.src[l])
                        s_full = c.scores(b, inp["qidx"][lf][b], inp["wh"][lf][b])
                        bm = oracle.block_maxima(s_full)
                        pool = rm.pools[(table.src[l], b)]
                        valid = pool[pool >= 0]
                        if valid.size < bm.size:
                            kth = np.sort(bm)[::-1][valid.size - 1]
                            band = np.abs(bm - kth) <= TOPK_REL * abs(kth)
                            assert band.sum() == 1, "ambiguous pool boundary in the test data"
                        check_topk_in_pool(gidx[l, b], s, oracle.pool_entries(pool, int(c.n[b])), wl.K)
                src_l = table.idx_src[l] if m == W.REUSE else l
                idx_l = None if m == W.SWA_ONLY else gidx[src_l, b]
                ref = rm.layer_attention(l, b, inp["q"][l][b], idx_l)
                assert attn_rel_err(gout[l, b], ref) <= ATTN_REL, (l, b)
    assert dm.status_bits() == 0


def _full_of(table, s):
    return next(l for l in range(table.n_layers) if table.mode[l] == W.FULL and table.src[l] == s)
