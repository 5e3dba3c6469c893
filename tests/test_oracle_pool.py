"""Pins of the oracle's hierarchical sparse indexer: the block pool built from a
Full layer's scores and the Top-K of a deeper layer restricted to that pool
("DeepSeek-V4.1-Flash, expliqué pas à pas", CSA2 chapter, hierarchical indexer
paragraph; video-summary page: blocks of 8 positions)."""
import numpy as np
import pytest

from fp4_sparse_attention_pack_b200 import workloads as W


def _brute_pool(scores, P):
    """Pure-Python: blocks of 8 ranked by (max desc, block asc), first P, sorted."""
    n = len(scores)
    blocks = []
    for b in range((n + 7) // 8):
        blocks.append((-max(scores[8 * b:min(n, 8 * b + 8)]), b))
    chosen = sorted(b for _, b in sorted(blocks)[:P])
    return chosen + [-1] * (P - len(chosen))


def _brute_in_pool(scores, pool, K):
    cand = [(-scores[e], e) for b in pool if b >= 0 for e in range(8 * b, min(len(scores), 8 * b + 8))]
    chosen = sorted(e for _, e in sorted(cand)[:K])
    return chosen + [-1] * (K - len(chosen))


@pytest.mark.parametrize("n,P,K", [(1, 1, 1), (7, 2, 3), (8, 1, 8), (61, 3, 5), (200, 6, 16), (203, 40, 9)])
def test_pool_and_restricted_topk_brute_force(ref, n, P, K):
    rng = np.random.default_rng(n * 31 + P)
    s = rng.normal(size=n)
    s[rng.random(n) < 0.3] = 0.0  # ReLU'd scores: many exact zeros, so ties decide
    pool = ref.block_pool(s, P)
    assert pool.dtype == np.int32 and list(pool) == _brute_pool(list(s), P)
    got = ref.topk_in_pool(s, pool, K)
    assert got.dtype == np.int32 and list(got) == _brute_in_pool(list(s), list(pool), K)


def test_ties_take_the_lower_block_and_entry(ref):
    s = np.zeros(40)
    assert list(ref.block_pool(s, 3)) == [0, 1, 2]
    assert list(ref.topk_in_pool(s, [3, 1, -1], 4)) == [8, 9, 10, 11]
    s[37] = 1.0  # the ragged last block (entries 32..39) wins outright
    assert list(ref.block_pool(s, 2)) == [0, 4]


def test_ragged_tail_and_padding(ref):
    s = np.arange(19, dtype=np.float64)      # blocks 0..2, the last holds 16..18
    assert list(ref.block_pool(s, 5)) == [0, 1, 2, -1, -1]
    assert list(ref.topk_in_pool(s, [2], 5)) == [16, 17, 18, -1, -1]   # never an entry >= n
    assert list(ref.pool_entries([2, 0], 19)) == [0, 1, 2, 3, 4, 5, 6, 7, 16, 17, 18]


def test_empty(ref):
    assert list(ref.block_pool(np.zeros(0), 4)) == [-1] * 4
    assert list(ref.topk_in_pool(np.zeros(0), [-1] * 4, 3)) == [-1] * 3


def test_pool_of_all_blocks_is_plain_topk(ref):
    rng = np.random.default_rng(3)
    s = rng.normal(size=1001)
    pool = ref.block_pool(s, 126)           # 126 blocks cover all 1,001 entries
    assert list(pool) == list(range(126))
    assert np.array_equal(ref.topk_in_pool(s, pool, 50), ref.topk(s, 50))


@pytest.mark.parametrize("P", [64, 65, 200])
def test_pool_contains_the_full_topk_when_it_has_k_blocks(ref, P):
    # distinct scores: every block ranked above the block of a Top-K entry holds an
    # entry ranked above it, so P >= K blocks always hold the whole Top-K
    rng = np.random.default_rng(P)
    s = rng.permutation(4096).astype(np.float64)
    full = ref.topk(s, 64)
    assert np.array_equal(ref.topk_in_pool(s, ref.block_pool(s, P), 64), full)


def test_small_pool_misses_part_of_the_full_topk(ref):
    # the pool really restricts: one block's worth of pool, Top-K spread over blocks
    s = np.zeros(64)
    s[[3, 12, 21, 30]] = [4.0, 3.0, 2.0, 1.0]
    pool = ref.block_pool(s, 2)
    assert list(pool) == [0, 1]
    assert list(ref.topk_in_pool(s, pool, 4)) == [0, 1, 3, 12]   # zeros of the pool fill in
    assert list(ref.topk(s, 4)) == [3, 12, 21, 30]


def _model(ref, table, P, B=2, T=150, H=4, Hi=4, K=6, seed=7):
    rng = np.random.default_rng(seed)
    Ws = [(rng.normal(size=(512, 128)) / np.sqrt(512)).astype(np.float32) for _ in table.ratios]
    m = ref.RefModel(table, B, [128] * table.n_sources, Ws, H, Hi, K, 1 / np.sqrt(512), pool_blocks=P)
    bf = lambda x: (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    for s in range(table.n_sources):
        for b in range(B):
            m.caches[s].append(b, bf(rng.normal(size=(T, 512))), rng.normal(size=T).astype(np.float32))
    L = table.n_layers
    inp = dict(
        x_new=[[bf(rng.normal(size=512)) for _ in range(B)] for _ in table.ratios],
        g_new=[rng.normal(size=B).astype(np.float32) for _ in table.ratios],
        q=[[bf(rng.normal(size=(H, 512))) for _ in range(B)] for _ in range(L)],
        qidx=[[bf(rng.normal(size=(Hi, 128))) for _ in range(B)] for _ in range(L)],
        wh=[[rng.uniform(0, 1, Hi).astype(np.float32) for _ in range(B)] for _ in range(L)],
        wtok=[[bf(rng.normal(size=512)) for _ in range(B)] for _ in range(L)],
    )
    return m, inp


def test_model_reindex_layers_search_the_full_layers_pool(ref):
    t = W.ModeTable((W.FULL, W.REINDEX, W.REUSE, W.REINDEX), (0, 0, 0, 0), (0, 1, 1, 3), (2,))
    m, inp = _model(ref, t, P=2)
    out, idx = m.step(**inp)
    c = m.caches[0]
    for b in range(2):
        s_full = c.scores(b, inp["qidx"][0][b], inp["wh"][0][b])
        pool = ref.block_pool(s_full, 2)
        assert np.array_equal(m.pools[(0, b)], pool)
        assert np.array_equal(idx[0][b], ref.topk(s_full, 6))          # the Full layer is not restricted
        for l in (1, 3):
            s = c.scores(b, inp["qidx"][l][b], inp["wh"][l][b])
            assert np.array_equal(idx[l][b], ref.topk_in_pool(s, pool, 6))
            assert all(e // 8 in set(pool) for e in idx[l][b] if e >= 0)
        assert np.array_equal(idx[2][b], idx[1][b])                     # Reuse is unchanged


def test_model_pool_of_all_blocks_equals_unpooled(ref):
    t = W.ModeTable((W.FULL, W.REINDEX, W.REINDEX), (0, 0, 0), (0, 1, 2), (2,))
    m0, inp = _model(ref, t, P=0)
    m1, _ = _model(ref, t, P=1000)
    out0, idx0 = m0.step(**inp)
    out1, idx1 = m1.step(**inp)
    for l in range(3):
        for b in range(2):
            assert np.array_equal(idx0[l][b], idx1[l][b])
            assert np.array_equal(out0[l][b], out1[l][b])
