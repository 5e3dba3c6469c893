"""The benchmark's algorithmic-byte accounting (the roofline numerators) against the
per-unit figures: 68 B per indexer key, 4 B per score, 64 x 72 B of query and
weights per (scan, sequence), 292 B per selected entry, 1,024 B (bf16) or 512 B
(FP8) per window token, 64 KiB of bf16 query and 128 KiB of fp32 output per
(layer, sequence)."""
import bench
from fp4_sparse_attention_pack_b200 import workloads as W


def _n(wl):
    return [[wl.entries(s)] * wl.B for s in range(wl.table.n_sources)]


def test_configuration_2_bytes():
    wl = W.WORKLOADS[2]
    kb = bench.kernel_bytes(wl, _n(wl))
    B, N, scans = 16, 65536, 23
    assert kb["index_scan"] == 4 * B * N * 68 + scans * B * 64 * 72 + scans * B * N * 4
    assert kb["topk"] == scans * B * N * 4 + scans * B * 512 * 4
    per_entry_layer = 512 * 292 + 128 * 1024 + 64 * 512 * 2 + 64 * 512 * 4
    per_window_layer = 128 * 1024 + 64 * 512 * 2 + 64 * 512 * 4
    assert kb["attention"] == B * (38 * per_entry_layer + 2 * per_window_layer)
    # at exactly 65,536 entries (the benchmark counts the entries present after its steps)
    assert kb["index_scan"] == 383_377_408 and kb["attention"] == 300_613_632


def test_fp8_windows_halve_the_window_bytes():
    a = bench.kernel_bytes(W.WORKLOADS[2], _n(W.WORKLOADS[2]))
    b = bench.kernel_bytes(W.WORKLOADS[8], _n(W.WORKLOADS[8]))
    assert a["attention"] - b["attention"] == 40 * 16 * 128 * 512
    assert a["index_scan"] == b["index_scan"]


def test_pooled_step_splits_the_indexer_phase():
    wl = W.WORKLOADS[6]
    kb = bench.kernel_bytes(wl, _n(wl))
    B, N, P = 16, 65536, 2048 * 8
    full, reidx = 4, 19
    scores = full * B * N * 4
    assert kb["index_scan"] == full * B * N * 68 + full * B * 64 * 72 + scores
    blocks = full * B * (N // 8) * 4
    pool = scores + 2 * blocks + full * B * 2048 * 4
    pscan = 4 * B * P * 68 + reidx * B * 64 * 72 + reidx * B * P * 4
    ptopk = reidx * B * P * 4 + reidx * B * 512 * 4
    assert kb["topk"] == scores + full * B * 512 * 4 + pool + pscan + ptopk
