"""Build oracle state from a workload's seeded recipe (host generator only).

The oracle never receives anything the CUDA path produced: every input here
comes from :mod:`fp4_sparse_attention_pack_b200.workloads` (host generator).
"""
import numpy as np

import oracle
from fp4_sparse_attention_pack_b200 import workloads as W

WIN = 128


def ref_cache(wl, s, seqs, T, cap=None, chunk=65536):
    """Oracle cache of source s for the sequences `seqs`, holding tokens [0, T)."""
    r = wl.table.ratios[s]
    cap = cap if cap is not None else wl.capacity_entries(s)
    c = oracle.RefCache(len(seqs), cap, r, W.w_idx(wl, s))
    for i, b in enumerate(seqs):
        for t0 in range(0, T, chunk):
            n = min(chunk, T - t0)
            c.append(i, W.tokens(wl, s, b, t0, n), W.gates(wl, s, b, t0, n))
    return c


def ref_window(wl, l, b, T):
    """Ring contents (bf16 bits [128][512]) and count after tokens [0, T)."""
    ring = np.zeros((WIN, 512), np.uint16)
    n = min(T, WIN)
    toks = W.window_tokens(wl, l, b, T - n, n)
    for i, p in enumerate(range(T - n, T)):
        ring[p % WIN] = toks[i]
    return ring, T


def ref_model(wl, T=None):
    """Full oracle model (all sequences) after tokens [0, T)."""
    T = wl.T if T is None else T
    t = wl.table
    m = oracle.RefModel(t, wl.B, [wl.capacity_entries(s) for s in range(t.n_sources)],
                        [W.w_idx(wl, s) for s in range(t.n_sources)], wl.H, wl.H_idx, wl.K, wl.scale,
                        pool_blocks=wl.pool_blocks, win_fp8=wl.win_fp8)
    for s in range(t.n_sources):
        m.caches[s] = ref_cache(wl, s, range(wl.B), T)
    for l in range(t.n_layers):
        for b in range(wl.B):
            ring, cnt = ref_window(wl, l, b, T)
            m.win[l, b] = ring
            if wl.win_fp8:
                m.win8[l, b] = oracle.window_fp8(ring)
            m.win_count[l, b] = cnt
    return m


def step_inputs(wl, st):
    """Host inputs of decode step st (token position T + append + st)."""
    t = wl.table
    p = wl.T + wl.append + st
    B = wl.B
    return dict(
        x_new=[[W.tokens(wl, s, b, p, 1)[0] for b in range(B)] for s in range(t.n_sources)],
        g_new=[np.array([W.gates(wl, s, b, p, 1)[0] for b in range(B)], np.float32)
               for s in range(t.n_sources)],
        q=[list(W.query(wl, l, st)) for l in range(t.n_layers)],
        qidx=[list(W.query_idx(wl, l, st)) for l in range(t.n_layers)],
        wh=[list(W.head_weights(wl, l, st)) for l in range(t.n_layers)],
        wtok=[[W.window_tokens(wl, l, b, p, 1)[0] for b in range(B)] for l in range(t.n_layers)],
    )
