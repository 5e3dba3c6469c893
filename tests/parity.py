"""Parity criteria of the CUDA path against the oracle (stated once, used by all GPU tests).

* packed caches: bit-exact, byte for byte, in logical entry order;
* Top-K: the GPU's index set equals the oracle's except for entries whose
  oracle score lies within TOPK_REL of the oracle's K-th score (their count is
  returned); indices distinct, within [0, n), increasing, padded with -1;
* hierarchical indexer: the pool by the Top-K criterion over the oracle's block
  maxima; a pool-restricted Top-K by the Top-K criterion over the oracle's
  scores of the pool's entries;
* attention: per (sequence, head) row, max_c |o - r| / max_c |r| <= ATTN_REL,
  the oracle evaluated on the GPU's own index set.
"""
import numpy as np

TOPK_REL = 1e-5
ATTN_REL = 2e-3


def check_topk(gpu_idx: np.ndarray, ref_scores: np.ndarray, K: int) -> int:
    """Assert the Top-K criterion for one sequence; return how many indices differ
    from the oracle's set (each of them inside the tie band)."""
    return topk_tie_report(gpu_idx, ref_scores, K)["differ"]


def topk_tie_report(gpu_idx: np.ndarray, ref_scores: np.ndarray, K: int) -> dict:
    """Assert the Top-K criterion for one sequence and report the tie band:
    band = entries whose oracle score lies within TOPK_REL of the oracle's K-th
    score (the entries on which the two sides may legitimately differ), differ =
    indices in exactly one of the two sets (all of them inside the band)."""
    n = ref_scores.size
    gpu_idx = np.asarray(gpu_idx, np.int64)
    m = min(K, n)
    assert np.all(gpu_idx[m:] == -1), "padding must be -1"
    g = gpu_idx[:m]
    assert np.all((g >= 0) & (g < n)), "index out of range"
    assert np.all(np.diff(g) > 0), "indices must be distinct and increasing"
    if m == 0:
        return {"band": 0, "differ": 0}
    order = sorted(range(n), key=lambda i: (-ref_scores[i], i)) if n < 4096 else \
        np.lexsort((np.arange(n), -ref_scores))
    ref_set = set(int(i) for i in order[:m])
    kth = ref_scores[order[m - 1]]
    band = np.abs(ref_scores - kth) <= TOPK_REL * max(abs(kth), 1e-30)
    diff = ref_set.symmetric_difference(set(int(i) for i in g))
    bad = [i for i in diff if not band[i]]
    assert not bad, f"{len(bad)} Top-K entries differ outside the tie band, e.g. {bad[:5]}"
    return {"band": int(band.sum()), "differ": len(diff)}


def attn_rel_err(out: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of max_c |o - r| / max_c |r| (rows = all leading dims)."""
    o = np.asarray(out, np.float64).reshape(-1, out.shape[-1])
    r = np.asarray(ref, np.float64).reshape(-1, ref.shape[-1])
    den = np.maximum(np.abs(r).max(axis=1), 1e-30)
    return float((np.abs(o - r).max(axis=1) / den).max())


def check_topk_in_pool(gpu_idx: np.ndarray, ref_scores: np.ndarray, cand: np.ndarray, K: int) -> int:
    """Top-K criterion restricted to the candidate entries `cand` (increasing)."""
    gpu_idx = np.asarray(gpu_idx, np.int64)
    cand = np.asarray(cand, np.int64)
    m = min(K, cand.size)
    g = gpu_idx[:m]
    pos = np.searchsorted(cand, g)
    assert np.all(pos < cand.size) and np.array_equal(cand[np.minimum(pos, cand.size - 1)], g), \
        "index outside the pool"
    return check_topk(np.concatenate([pos, gpu_idx[m:]]), ref_scores[cand], K)
