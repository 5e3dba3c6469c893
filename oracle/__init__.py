"""CSA2 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The CUDA library never calls it and
shares no code with it; the per-entry arithmetic lives in ``csa2_ref.c``
(plain C, fp32 where a float decides an integer code, fp64 elsewhere) and the
per-layer mode table is orchestrated here in plain Python.

Mode table ("Résumé exécutif", CSA2 table; CSA2 chapter of "DeepSeek-V4.1-Flash,
expliqué pas à pas"):
  Full    -- computes the main cache, the indexer keys and its Top-K indices;
  Reindex -- reuses the main cache and indexer keys of its source, recomputes
             the Top-K with its own indexer query;
  Reuse   -- reuses the cache and the indices of the nearest preceding
             Full/Reindex layer of its group;
every layer keeps its own main query and its own 128-token sliding window and
produces its own attention output; layers 0-1 are sliding-window only.

Every function here has a pin in ``tests/test_oracle_*.py`` (closed forms, page
figures, library routines, brute force); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(_HERE, "libcsa2_ref.so")
SWA_ONLY, FULL, REINDEX, REUSE = 0, 1, 2, 3
D, D_IDX, WIN = 512, 128, 128


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "csa2_ref.c")
    hdr = os.path.join(_HERE, "csa2_ref.h")
    stale = (not os.path.exists(SO) or os.path.getmtime(SO) < max(os.path.getmtime(src),
                                                                    os.path.getmtime(hdr)))
    if force or stale:
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", src, "-o", SO, "-lm"])
    return SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp, ci, cf, cd, cu = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_uint
        for name, res, args in [
            ("ref_e2m1_value", cd, [cu]), ("ref_e4m3_value", cd, [cu]), ("ref_e8m0_value", cd, [cu]),
            ("ref_e2m1_encode", cu, [cf]), ("ref_e4m3_encode", cu, [cf]),
            ("ref_window_fp8", None, [vp, ci, vp]),
            ("ref_mx_shared_exp", ci, [cf]), ("ref_spec_exp", cf, [cf]),
            ("ref_compress_pair", None, [vp, cf, vp, cf, vp]),
            ("ref_pack_main", None, [vp, vp, vp]), ("ref_dequant_main", None, [vp, vp, vp]),
            ("ref_mxfp4_quant", None, [vp, ci, vp, vp]),
            ("ref_index_key", None, [vp, vp, vp, vp, vp]),
            ("ref_append_tokens", ci, [ci, vp, vp, ci, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci]),
            ("ref_index_scores", None, [vp, vp, ci, vp, vp, vp, ci, vp]),
            ("ref_topk", None, [vp, ci, ci, vp]),
            ("ref_gather_items", ci, [vp, vp, ci, vp, ci, vp, ci, vp]),
            ("ref_attention", None, [vp, ci, vp, ci, cd, vp]),
            ("ref_threads", ci, []),
        ]:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def threads() -> int:
    return int(lib().ref_threads())


def bf16_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- per-op API

def e2m1_value(code: int) -> float:
    return lib().ref_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().ref_e4m3_value(code)


def e8m0_value(code: int) -> float:
    return lib().ref_e8m0_value(code)


def e2m1_encode(v: float) -> int:
    return lib().ref_e2m1_encode(float(np.float32(v)))


def e4m3_encode(v: float) -> int:
    return lib().ref_e4m3_encode(float(np.float32(v)))


def window_fp8(tok_bf16) -> np.ndarray:
    """E4M3 codes of bf16 window tokens, one per channel, same shape (the FP8
    SWA window: "Le cache KV en FP4", the SWA KV stays in FP8)."""
    x = np.ascontiguousarray(bf16_to_f32(tok_bf16), np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().ref_window_fp8(_p(x), x.size, _p(out))
    return out


_E4M3_VALUES = None


def e4m3_values(codes) -> np.ndarray:
    """fp32 values of E4M3 codes (each exact in fp32), from ref_e4m3_value."""
    global _E4M3_VALUES
    if _E4M3_VALUES is None:
        _E4M3_VALUES = np.array([e4m3_value(c) for c in range(256)], np.float32)
    return _E4M3_VALUES[np.asarray(codes, np.uint8)]


def mx_shared_exp(amax: float) -> int:
    return lib().ref_mx_shared_exp(float(np.float32(amax)))


def spec_exp(x) -> np.ndarray:
    x = np.asarray(x, np.float32).ravel()
    return np.array([lib().ref_spec_exp(float(v)) for v in x], np.float32)


def compress_pair(x0, g0, x1, g1) -> np.ndarray:
    x0 = np.ascontiguousarray(x0, np.float32)
    x1 = np.ascontiguousarray(x1, np.float32)
    e = np.empty(D, np.float32)
    lib().ref_compress_pair(_p(x0), float(np.float32(g0)), _p(x1), float(np.float32(g1)), _p(e))
    return e


def pack_main(e):
    e = np.ascontiguousarray(e, np.float32)
    codes, scales = np.empty(256, np.uint8), np.empty(32, np.uint8)
    lib().ref_pack_main(_p(e), _p(codes), _p(scales))
    return codes, scales


def dequant_main(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    out = np.empty(D, np.float32)
    lib().ref_dequant_main(_p(codes), _p(scales), _p(out))
    return out


def mxfp4_quant(v):
    v = np.ascontiguousarray(v, np.float32).ravel()
    codes, scales = np.empty(v.size // 2, np.uint8), np.empty(v.size // 32, np.uint8)
    lib().ref_mxfp4_quant(_p(v), v.size, _p(codes), _p(scales))
    return codes, scales


def mxfp4_dequant(codes, scales) -> np.ndarray:
    codes = np.asarray(codes, np.uint8).ravel()
    n = codes.size * 2
    q = np.empty(n, np.uint8)
    q[0::2], q[1::2] = codes & 15, codes >> 4
    vals = np.array([e2m1_value(c) for c in range(16)])[q]
    sc = np.array([e8m0_value(int(s)) for s in np.asarray(scales).ravel()])
    return vals * np.repeat(sc, 32)


def index_key(codes, scales, W):
    W = np.ascontiguousarray(W, np.float32)
    kc, ks = np.empty(64, np.uint8), np.empty(4, np.uint8)
    lib().ref_index_key(_p(np.ascontiguousarray(codes, np.uint8)),
                        _p(np.ascontiguousarray(scales, np.uint8)), _p(W), _p(kc), _p(ks))
    return kc, ks


def quantize_queries(qidx_bf16):
    """MXFP4 of each indexer-query head: bf16 [H][128] -> codes [H][64], scales [H][4]."""
    q = bf16_to_f32(qidx_bf16).reshape(-1, D_IDX)
    H = q.shape[0]
    qc, qs = np.empty((H, 64), np.uint8), np.empty((H, 4), np.uint8)
    for h in range(H):
        qc[h], qs[h] = mxfp4_quant(q[h])
    return qc, qs


def index_scores(kc, ks, N, qidx_bf16, w) -> np.ndarray:
    qc, qs = quantize_queries(qidx_bf16)
    w = np.ascontiguousarray(w, np.float32)
    out = np.empty(max(N, 1), np.float64)
    lib().ref_index_scores(_p(np.ascontiguousarray(kc)), _p(np.ascontiguousarray(ks)), N, _p(qc),
                           _p(qs), _p(w), qc.shape[0], _p(out))
    return out[:N]


def topk(scores, K) -> np.ndarray:
    scores = np.ascontiguousarray(scores, np.float64)
    out = np.empty(K, np.int32)
    lib().ref_topk(_p(scores) if scores.size else None, scores.size, K, _p(out))
    return out


# Hierarchical sparse indexer ("DeepSeek-V4.1-Flash, expliqué pas à pas", CSA2
# chapter, hierarchical indexer paragraph: in the CED decoder the shallow
# indexer's information restricts the candidates of the deeper indexers, so only
# the first Full layer keeps scanning the whole context; the video-summary page
# gives the pool as blocks of 8 positions, 2,048 of them at a million tokens,
# built by the first decoder layer).  The step list itself did not survive on
# the page; the reading taken here: a block is 8 consecutive entries, its score
# the largest score of its entries under the Full layer's indexer; the pool is
# the pool_blocks best blocks (ties: lower block); a deeper Reindex layer scores
# only the pool's entries and keeps its Top-K among them.
POOL_BLOCK = 8


def block_maxima(scores) -> np.ndarray:
    """Score of every block: the largest score among its (up to 8) entries."""
    scores = np.asarray(scores, np.float64)
    if scores.size == 0:
        return np.zeros(0, np.float64)
    return np.maximum.reduceat(scores, np.arange(0, scores.size, POOL_BLOCK))


def block_pool(scores, pool_blocks: int) -> np.ndarray:
    """Block ids of the pool, increasing, padded with -1 (int32[pool_blocks])."""
    bmax = block_maxima(scores)
    if bmax.size == 0:
        return np.full(pool_blocks, -1, np.int32)
    return topk(bmax, pool_blocks)


def pool_entries(pool, n: int) -> np.ndarray:
    """Entries of the pool's blocks below n, increasing (int64)."""
    blocks = np.asarray(pool, np.int64)
    blocks = blocks[blocks >= 0]
    ents = np.sort((blocks[:, None] * POOL_BLOCK + np.arange(POOL_BLOCK)[None, :]).reshape(-1))
    return ents[ents < n]


def topk_in_pool(scores, pool, K: int) -> np.ndarray:
    """Top-K over the pool's entries only (score desc, entry asc), increasing,
    padded with -1 (int32[K])."""
    scores = np.asarray(scores, np.float64)
    ents = pool_entries(pool, scores.size)
    sel = topk(scores[ents], K)
    if ents.size == 0:
        return sel
    return np.where(sel >= 0, ents[np.maximum(sel, 0)], -1).astype(np.int32)


def attention_items(mc, ms, n_entries, idx, win_bf16, win_len) -> np.ndarray:
    idx = np.ascontiguousarray(idx, np.int32)
    win = np.ascontiguousarray(win_bf16, np.uint16)
    items = np.empty((idx.size + win_len, D), np.float32)
    m = lib().ref_gather_items(_p(mc), _p(ms), n_entries, _p(idx) if idx.size else None, idx.size,
                               _p(win), win_len, _p(items))
    return items[:m]


def attention_items_fp8(mc, ms, n_entries, idx, win_codes, win_len) -> np.ndarray:
    """attention_items for an FP8 window: the selected entries, then the E4M3
    values of the first win_len window slots."""
    ents = attention_items(mc, ms, n_entries, idx, np.zeros((1, D), np.uint16), 0)
    w = e4m3_values(np.asarray(win_codes, np.uint8).reshape(-1, D)[:win_len])
    return np.concatenate([ents, w.astype(np.float32)])


def attention(q_bf16, items, scale) -> np.ndarray:
    q = np.ascontiguousarray(bf16_to_f32(q_bf16).reshape(-1, D))
    items = np.ascontiguousarray(items, np.float32)
    H = q.shape[0]
    out = np.empty((H, D), np.float32)
    lib().ref_attention(_p(q), H, _p(items) if items.size else None, items.shape[0], float(scale),
                        _p(out))
    return out


# ---------------------------------------------------------------- state objects

class RefCache:
    """One source's compressed cache for B sequences (logical, unpaged layout)."""

    def __init__(self, B: int, cap: int, ratio: int, W):
        self.B, self.cap, self.ratio = B, cap, ratio
        self.W = np.ascontiguousarray(W, np.float32)
        self.mc = np.zeros((B, cap, 256), np.uint8)
        self.ms = np.zeros((B, cap, 32), np.uint8)
        self.kc = np.zeros((B, cap, 64), np.uint8)
        self.ks = np.zeros((B, cap, 4), np.uint8)
        self.n = np.zeros(B, np.int32)
        self.pend_valid = np.zeros(B, np.int32)
        self.pend_x = np.zeros((B, D), np.float32)
        self.pend_g = np.zeros(B, np.float32)

    def append(self, b: int, x_bf16, g):
        x = np.ascontiguousarray(bf16_to_f32(x_bf16).reshape(-1, D))
        g = np.ascontiguousarray(g, np.float32).ravel()
        pv = self.pend_valid[b:b + 1]
        px = self.pend_x[b]
        pg = self.pend_g[b:b + 1]
        n = lib().ref_append_tokens(self.ratio, _p(x), _p(g), x.shape[0], _p(self.W), _p(pv), _p(px),
                                    _p(pg), _p(self.mc[b]), _p(self.ms[b]), _p(self.kc[b]),
                                    _p(self.ks[b]), int(self.n[b]), self.cap)
        if n < 0:
            raise ValueError("cache capacity exceeded")
        self.n[b] = n

    def scores(self, b: int, qidx_bf16, w) -> np.ndarray:
        return index_scores(self.kc[b], self.ks[b], int(self.n[b]), qidx_bf16, w)


class RefModel:
    """All layers of one decode model: per-source caches and per-layer windows."""

    def __init__(self, table, B: int, caps, Ws, H: int, H_idx: int, K: int, scale: float,
                 pool_blocks: int = 0, win_fp8: bool = False):
        self.t = table
        self.B, self.H, self.H_idx, self.K, self.scale = B, H, H_idx, K, scale
        self.pool_blocks = pool_blocks  # > 0: Reindex layers search the Full layer's pool
        self.win_fp8 = win_fp8          # windows keep E4M3 codes (win8) instead of bf16
        self.caches = [RefCache(B, caps[s], table.ratios[s], Ws[s]) for s in range(table.n_sources)]
        L = table.n_layers
        self.win = np.zeros((L, B, WIN, D), np.uint16)
        self.win8 = np.zeros((L, B, WIN, D), np.uint8) if win_fp8 else None
        self.win_count = np.zeros((L, B), np.int64)
        for l in range(L):
            m = table.mode[l]
            if m == REUSE:
                j = table.idx_src[l]
                if not (0 <= j < l and table.mode[j] in (FULL, REINDEX) and table.src[j] == table.src[l]):
                    raise ValueError(f"layer {l}: Reuse must name an earlier Full/Reindex layer "
                                     "of the same source")

    def window_append(self, l: int, b: int, tok_bf16):
        slot = int(self.win_count[l, b] % WIN)
        self.win[l, b, slot] = np.asarray(tok_bf16, np.uint16).reshape(D)
        if self.win_fp8:
            self.win8[l, b, slot] = window_fp8(self.win[l, b, slot])
        self.win_count[l, b] += 1

    def win_len(self, l: int, b: int) -> int:
        return int(min(self.win_count[l, b], WIN))

    def layer_attention(self, l: int, b: int, q_bf16, idx) -> np.ndarray:
        wl = self.win_len(l, b)
        gather = attention_items_fp8 if self.win_fp8 else attention_items
        win = self.win8[l, b] if self.win_fp8 else self.win[l, b]
        if self.t.mode[l] == SWA_ONLY or idx is None:
            items = gather(np.zeros((1, 256), np.uint8), np.zeros((1, 32), np.uint8), 0,
                           np.zeros(0, np.int32), win, wl)
        else:
            c = self.caches[self.t.src[l]]
            items = gather(c.mc[b], c.ms[b], int(c.n[b]), idx, win, wl)
        return attention(q_bf16, items, self.scale)

    def step(self, x_new, g_new, q, qidx, wh, wtok, want=None):
        """One decode step of every layer.  Order: window append (all layers),
        source cache write, then per layer Top-K (Full/Reindex) or index reuse
        (Reuse), then attention.  ``want``: optional set of (layer, seq) whose
        attention output is computed (others are None) to bound the work.
        Returns (out[l][b] or None, idx[l][b] or None)."""
        L, B = self.t.n_layers, self.B
        for l in range(L):
            for b in range(B):
                self.window_append(l, b, wtok[l][b])
        for s in range(self.t.n_sources):
            for b in range(B):
                self.caches[s].append(b, x_new[s][b], g_new[s][b:b + 1])
        idx = [[None] * B for _ in range(L)]
        out = [[None] * B for _ in range(L)]
        self.pools = {}  # (source, seq) -> pool of the source's Full layer this step
        for l in range(L):
            m = self.t.mode[l]
            for b in range(B):
                if m in (FULL, REINDEX):
                    c = self.caches[self.t.src[l]]
                    sc = c.scores(b, qidx[l][b], wh[l][b])
                    pool = self.pools.get((self.t.src[l], b)) if self.pool_blocks > 0 else None
                    if m == REINDEX and pool is not None:
                        idx[l][b] = topk_in_pool(sc, pool, self.K)
                    else:
                        idx[l][b] = topk(sc, self.K)
                    if m == FULL and self.pool_blocks > 0:
                        self.pools[(self.t.src[l], b)] = block_pool(sc, self.pool_blocks)
                elif m == REUSE:
                    idx[l][b] = idx[self.t.idx_src[l]][b]
                if want is None or (l, b) in want:
                    out[l][b] = self.layer_attention(l, b, q[l][b], idx[l][b])
        return out, idx
