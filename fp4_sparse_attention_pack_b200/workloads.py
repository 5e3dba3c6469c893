"""Workload definitions: shapes, per-layer mode tables and the seeded input recipe.

Nothing here computes a step of the CSA2 method; both the CUDA path and the
oracle receive these values as inputs.

Sources (DeepSeek-V4.1-Flash course pages):
  * "DeepSeek-V4.1-Flash, expliqué pas à pas", CSA2 chapter (three modes, the
    exact mode split of section 4.2.1 of the report, SWA n_win = 128, top 512);
  * "Résumé exécutif", CSA2 table (Full / Reindex / Reuse: what each layer
    computes or reuses) and "only layers 2, 8, 14 and 20 write a cache".
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import synth

# per-layer modes
SWA_ONLY, FULL, REINDEX, REUSE = 0, 1, 2, 3
MODE_NAMES = {SWA_ONLY: "swa", FULL: "full", REINDEX: "reindex", REUSE: "reuse"}

D = 512        # main latent channels
D_IDX = 128    # indexer key / query dim
WIN = 128      # SWA window (n_win)
PAGE = 64      # entries per cache page


@dataclasses.dataclass(frozen=True)
class ModeTable:
    mode: tuple   # per layer
    src: tuple    # per layer: source cache index (-1 for SWA_ONLY)
    idx_src: tuple  # per layer: layer whose Top-K indices are used (-1 for SWA_ONLY)
    ratios: tuple   # per source: tokens per entry (1 or 2)

    @property
    def n_layers(self):
        return len(self.mode)

    @property
    def n_sources(self):
        return len(self.ratios)

    def scan_layers(self):
        return [l for l, m in enumerate(self.mode) if m in (FULL, REINDEX)]


def single_full() -> ModeTable:
    """One Full-mode layer writing and reading source 0 (ratio 2)."""
    return ModeTable((FULL,), (0,), (0,), (2,))


def _groups_table(groups, n_layers, ratios, pattern):
    mode = [SWA_ONLY] * n_layers
    src = [-1] * n_layers
    idx_src = [-1] * n_layers
    for s, (a, b) in enumerate(groups):
        last_indexer = -1
        for l in range(a, b):
            m = pattern(s, l - a)
            mode[l] = m
            src[l] = s
            if m in (FULL, REINDEX):
                last_indexer = l
            idx_src[l] = last_indexer
    return ModeTable(tuple(mode), tuple(src), tuple(idx_src), tuple(ratios))


def schedule_alternating_40() -> ModeTable:
    """40 layers; layers 0-1 SWA only; sources at layers 2, 8, 14 (encoder) and 20
    (decoder), all ratio 2.  In each source's group the first layer is Full, the
    next Reindex, then Reuse and Reindex alternate; a Reuse layer takes the indices
    of the nearest preceding Full/Reindex layer of its group.  23 scans per step."""
    def pat(_s, j):
        if j == 0:
            return FULL
        return REINDEX if j % 2 == 1 else REUSE
    return _groups_table([(2, 8), (8, 14), (14, 20), (20, 40)], 40, (2, 2, 2, 2), pat)


def schedule_pages_40() -> ModeTable:
    """The report's split (section 4.2.1): encoder layers 2-19 in 3 groups of
    1 Full + 5 Reuse at ratio 2; decoder layers 20-39 at ratio 1, first group of 4
    is 1 Full + 3 Reuse, the next four groups are 1 Reindex + 3 Reuse over the
    decoder's Full cache.  8 scans per step."""
    def pat(s, j):
        if s < 3:
            return FULL if j == 0 else REUSE
        if j == 0:
            return FULL
        return REINDEX if j % 4 == 0 else REUSE
    return _groups_table([(2, 8), (8, 14), (14, 20), (20, 40)], 40, (2, 2, 2, 1), pat)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    T: int              # tokens cached per sequence per source before the steps
    table: ModeTable
    H: int
    H_idx: int
    K: int
    steps: int          # decode steps of the workload
    outliers: bool = False
    append: int = 0     # tokens appended per sequence before the decode steps
    pool_blocks: int = 0  # > 0: hierarchical indexer, Reindex layers scan their source's pool
    win_fp8: bool = False  # SWA windows kept as E4M3 codes instead of bf16

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / np.sqrt(D)))

    def entries(self, s: int, tokens: int | None = None) -> int:
        t = self.T if tokens is None else tokens
        return t // self.table.ratios[s]

    def capacity_entries(self, s: int) -> int:
        """Entries a sequence can hold: everything the workload ever appends."""
        return self.entries(s, self.T + self.append + self.steps + 2)

    def max_pages(self, s: int) -> int:
        return (self.capacity_entries(s) + PAGE - 1) // PAGE


WORKLOADS = {
    0: Workload("cfg0_1layer_b1_4k", 0, 1, 4096, single_full(), 16, 4, 256, 1),
    1: Workload("cfg1_1layer_b8_64k", 1, 8, 65536, single_full(), 64, 64, 512, 100),
    2: Workload("cfg2_40layer_b16_128k", 2, 16, 131072, schedule_alternating_40(), 64, 64, 512, 100),
    3: Workload("cfg3_1layer_b4_1m_outliers", 3, 4, 1048576, single_full(), 64, 64, 1024, 1,
                outliers=True),
    4: Workload("cfg4_prefix_append_b16_256k", 4, 16, 262144, schedule_alternating_40(), 64, 64, 512,
                64, append=8192),
    # the pages' own schedule and ratios (8 scans per step, decoder source at ratio 1)
    5: Workload("cfg5_pages40_b16_128k", 5, 16, 131072, schedule_pages_40(), 64, 64, 512, 100),
    # the hierarchical indexer on both schedules: pools of 2,048 blocks of 8 entries
    6: Workload("cfg6_alternating40_b16_128k_pool2048", 2, 16, 131072, schedule_alternating_40(), 64, 64,
                512, 100, pool_blocks=2048),
    7: Workload("cfg7_pages40_b16_128k_pool2048", 5, 16, 131072, schedule_pages_40(), 64, 64, 512, 100,
                pool_blocks=2048),
    # the 40-layer step with the SWA windows in FP8 (E4M3, 512 B a token)
    8: Workload("cfg8_40layer_b16_128k_fp8win", 2, 16, 131072, schedule_alternating_40(), 64, 64, 512, 100,
                win_fp8=True),
}


# Profiling cases: one kernel at a size whose inputs exceed L2 (126 MB) while the
# device holds a few GB at most.
PROFILE_WORKLOADS = {
    # one Full layer over 32 sequences x 65,536 entries: 142 MB of indexer keys per scan
    "scan32": Workload("scan32_1layer_b32_128k", 5, 32, 131072, single_full(), 64, 64, 512, 4),
    # the 40-layer step at batch 4: 160 attention units (about one wave), 410 MB of keys per step
    "step_b4": Workload("step_b4_40layer_128k", 6, 4, 131072, schedule_alternating_40(), 64, 64, 512, 4),
    # the same step with the hierarchical indexer (pools of 2,048 blocks)
    "step_b4_pool": Workload("step_b4_pool2048_40layer_128k", 6, 4, 131072, schedule_alternating_40(), 64, 64,
                             512, 4, pool_blocks=2048),
}


def small(wl: Workload, **kw) -> Workload:
    """A reduced copy of a workload (same recipe, smaller sizes)."""
    return dataclasses.replace(wl, **kw)


# ---------------------------------------------------------------- input recipe

def _choose(seed: int, tensor_sub: int, n: int, k: int) -> np.ndarray:
    """k distinct values of range(n): partial Fisher-Yates driven by SplitMix64."""
    u = synth.u64(synth.key(seed, synth.TID_OUTLIER, tensor_sub), 0, k)
    perm = np.arange(n)
    for i in range(k):
        j = i + int(u[i] % np.uint64(n - i))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:k])


def outlier_channels(wl: Workload, s: int) -> np.ndarray:
    """1 % of the latent channels (5 of 512), scaled by 64 in the source values."""
    return _choose(wl.seed, 2 * s, D, 5) if wl.outliers else np.zeros(0, np.int64)


def outlier_columns(wl: Workload, s: int) -> np.ndarray:
    """1 % of the indexer-key columns (2 of 128), scaled by 64 in W_idx."""
    return _choose(wl.seed, 2 * s + 1, D_IDX, 2) if wl.outliers else np.zeros(0, np.int64)


def chan_scale(wl: Workload, s: int) -> np.ndarray:
    """Per-channel lognormal(0, 0.5) scale of source s (fp32[512])."""
    z = synth.normal_f32(synth.key(wl.seed, synth.TID_CHAN, s), 0, D).astype(np.float64)
    sc = np.exp(0.5 * z).astype(np.float32)
    sc[outlier_channels(wl, s)] *= np.float32(64.0)
    return sc


def w_idx(wl: Workload, s: int) -> np.ndarray:
    """Indexer projection of source s: fp32 [512][128], N(0, 1/512)."""
    w = synth.normal_scaled_f32(synth.key(wl.seed, synth.TID_W, s), 0, D * D_IDX,
                                np.float32(1.0 / np.sqrt(D))).reshape(D, D_IDX)
    cols = outlier_columns(wl, s)
    if cols.size:
        w[:, cols] *= np.float32(64.0)
    return w


def tokens(wl: Workload, s: int, b: int, t0: int, n: int) -> np.ndarray:
    """Source tokens t0..t0+n-1 of sequence b, bf16 bits [n][512]."""
    k = synth.key(wl.seed, synth.TID_SRC_X, s)
    return synth.normal_bf16(k, (b * synth.TSTRIDE + t0) * D, n * D, chan_scale(wl, s)).reshape(n, D)


def gates(wl: Workload, s: int, b: int, t0: int, n: int) -> np.ndarray:
    """Gate logits of tokens t0..t0+n-1 of sequence b, fp32 [n], N(0,1)."""
    return synth.normal_f32(synth.key(wl.seed, synth.TID_SRC_G, s), b * synth.TSTRIDE + t0, n)


def query(wl: Workload, l: int, st: int) -> np.ndarray:
    """Main query of layer l at step st, bf16 bits [B][H][512], N(0,1)."""
    n = wl.B * wl.H * D
    return synth.normal_bf16(synth.key(wl.seed, synth.TID_Q, l), st * n, n).reshape(wl.B, wl.H, D)


def query_idx(wl: Workload, l: int, st: int) -> np.ndarray:
    """Indexer query of layer l at step st, bf16 bits [B][H_idx][128], N(0,1)."""
    n = wl.B * wl.H_idx * D_IDX
    return synth.normal_bf16(synth.key(wl.seed, synth.TID_QIDX, l), st * n, n).reshape(
        wl.B, wl.H_idx, D_IDX)


def head_weights(wl: Workload, l: int, st: int) -> np.ndarray:
    """Indexer head weights of layer l at step st, fp32 [B][H_idx], U(0,1)."""
    n = wl.B * wl.H_idx
    return synth.uniform_f32(synth.key(wl.seed, synth.TID_WH, l), st * n, n).reshape(wl.B, wl.H_idx)


def window_tokens(wl: Workload, l: int, b: int, p0: int, n: int) -> np.ndarray:
    """SWA tokens at positions p0..p0+n-1 of layer l, sequence b, bf16 bits [n][512]."""
    k = synth.key(wl.seed, synth.TID_WIN, l)
    return synth.normal_bf16(k, (b * synth.TSTRIDE + p0) * D, n * D).reshape(n, D)
