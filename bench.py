#!/usr/bin/env python3
"""CSA2 decode benchmark: 40-layer decode step, batch 16, 131,072-token context.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 2]

One step = one CSA2 decode step of every layer of the workload (window append,
source cache write, every Full/Reindex scan + Top-K, every layer's attention)
for the whole batch, through the C ABI's csa2_layer_step, replayed from a CUDA
graph.  Metric: layer-steps/s (one layer x one decode step for the batch).
Multi-GPU: one process per GPU, each with its own batch (the path shards by
sequence, no collective): weak scaling, value = all ranks' layer-steps / max time.

``--impl reference`` times the CPU oracle (the plain C reference) on the host
cores on a bounded sample of the same workload; it prints the same JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode layer-steps/s at 128K ctx"
UNIT = "layer-steps/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--workload", default=None,
                    help="a profiling case of workloads.PROFILE_WORKLOADS instead of --config")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-layer", action="store_true",
                    help="skip the layer-by-layer timing of the indexer and attention")
    ap.add_argument("--profile-steps", type=int, default=5)
    ap.add_argument("--measure", choices=["step", "cache_io"], default="step",
                    help="cache_io: prefix-cache export/import throughput of one source's sequences")
    return ap.parse_args()


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.samples = []  # (t, sm, smax, reasons set)
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            reasons = {n for n, v in zip(names, parts[5:9]) if v.lower() == "active"}
            self.samples.append((time.time(), sm, smax, reasons))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        where = "timed"
        if len(win) < 3:
            win = [s for s in self.samples if s[0] <= t1]
            where = "warmup+timed"
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": "none"}
        reasons = sorted(set().union(*[s[3] for s in win]))
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": max(s[2] for s in win),
                "reasons": reasons, "samples": len(win), "window": where}


# ---------------------------------------------------------------- helpers

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


KERNEL_SOURCES = {"index_scan": "scan_mma.cu", "attention": "attn_mma.cu", "topk": "topk.cu"}


def kernel_traffic(kernel: str):
    """Per-launch DRAM bytes (read + write) of a kernel at the bench workload from
    the committed ncu summary profiles/<kernel>_traffic.json, only while the
    kernel's source is unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")
    src = os.path.join(ROOT, "fp4_sparse_attention_pack_b200", "csrc", KERNEL_SOURCES[kernel])
    try:
        with open(p) as f:
            d = json.load(f)
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        return d.get("bytes_per_launch_at_workload") if d.get("source_sha") == sha else None
    except (OSError, ValueError):
        return None


def workload_config(wl, world):
    """The workload keys of the JSON line's config (both arms)."""
    cfg = {"workload": wl.name, "global_batch": wl.B * world, "seq_len": wl.T,
           "layers": wl.table.n_layers, "scans_per_step": len(wl.table.scan_layers()), "H": wl.H,
           "H_idx": wl.H_idx, "top_k": wl.K, "parallelism": f"dp{world} (replicas, no collective)",
           "cache_format": "E2M1+E4M3/16 main, MXFP4 indexer keys"}
    if wl.pool_blocks > 0:
        cfg["pool_blocks"] = wl.pool_blocks
    cfg["window"] = "fp8 e4m3 (512 B a token)" if wl.win_fp8 else "bf16 (1,024 B a token)"
    return cfg


def kernel_bytes(wl, n_entries):
    """Algorithmic HBM bytes per launch of each kernel in one decode step (our
    accounting of the path; every launch covers all layers of the step):
      index_scan  each scanned source's indexer keys once (64 code + 4 scale
                  bytes per entry), every scan's query (64 x (64 + 4) bytes) and
                  head weights, one fp32 score per (scan, entry) written;
      topk        the scores read, K indices written per (scan, sequence);
      attention   per (layer, sequence) the K selected entries (256 code + 32
                  scale bytes) and their indices, the 128-token window (bf16, or
                  one E4M3 byte a channel), the bf16 query, the fp32 output;
      step        all kernels, plus the cache write of the new tokens.
    With pools (hierarchical indexer) index_scan covers the Full layers only,
    and topk the rest of the indexer phase: the Full layers' Top-K, the block
    maxima (scores read, one fp32 per 8 entries written), the pool Top-K (block
    maxima read, pool written), the Reindex layers' pool scans (per source the
    keys of its pools' positions once, their queries, one fp32 score per
    position written) and their Top-K (those scores read, K indices written)."""
    from fp4_sparse_attention_pack_b200 import workloads as W
    t = wl.table
    B, H, Hi, K = wl.B, wl.H, wl.H_idx, wl.K
    scans = t.scan_layers()
    n_src = {s: sum(n_entries[s]) for s in range(t.n_sources)}
    qbytes = B * Hi * (64 + 4 + 4)
    if wl.pool_blocks > 0:
        full = [l for l in scans if t.mode[l] == W.FULL]
        reidx = [l for l in scans if t.mode[l] == W.REINDEX]
        score_bytes = sum(n_src[t.src[l]] * 4 for l in full)
        scan = sum(n_src[t.src[l]] * 68 for l in full) + len(full) * qbytes + score_bytes
        pos = {s: sum(min(8 * wl.pool_blocks, n) for n in n_entries[s]) for s in range(t.n_sources)}
        blocks = sum((n_src[t.src[l]] + 7) // 8 * 4 for l in full)
        pool = score_bytes + blocks + blocks + len(full) * B * wl.pool_blocks * 4
        pscan = (sum(pos[s] * 68 for s in sorted({t.src[l] for l in reidx})) + len(reidx) * qbytes +
                 sum(pos[t.src[l]] * 4 for l in reidx))
        ptopk = sum(pos[t.src[l]] * 4 for l in reidx) + len(reidx) * B * K * 4
        topk = score_bytes + len(full) * B * K * 4 + pool + pscan + ptopk
    else:
        scanned = sorted({t.src[l] for l in scans})
        score_bytes = sum(n_src[t.src[l]] * 4 for l in scans)
        scan = (sum(n_src[s] * 68 for s in scanned) + len(scans) * qbytes + score_bytes)
        topk = score_bytes + len(scans) * B * K * 4
    attn = 0
    win_b = 1 if wl.win_fp8 else 2  # bytes a window channel
    for m in t.mode:
        attn += B * (WIN * 512 * win_b + H * 512 * 2 + H * 512 * 4)
        if m != 0:
            attn += B * K * (288 + 4)
    cache_write = t.n_sources * B * (512 * 2 + 4 + 288 + 68)
    return {"index_scan": scan, "topk": topk, "attention": attn,
            "step": scan + topk + attn + cache_write + t.n_layers * B * 1024}


WIN = 128


def survey_bytes(wl, n_entries):
    """HBM bytes per step under the per-scan accounting (every scan reads its
    source's keys, as a decoder that scans layer by layer must):
      reads  per sequence: scans x (n 68 + H_idx 128 2 + H_idx 4) + attention
             layers x K (288 + 4) + layers x (128 512 2 + H 512 2);
      writes layers x H 512 4 (fp32 output) + scans x K 4 (indices) per sequence;
    the scores are not counted.  index_scan = the scans' reads, attention = the
    attention reads and the output."""
    t = wl.table
    scans = t.scan_layers()
    B, H, Hi, K = wl.B, wl.H, wl.H_idx, wl.K
    scan = sum(n * 68 + Hi * 128 * 2 + Hi * 4 for l in scans for n in n_entries[t.src[l]])
    attn_layers = sum(1 for m in t.mode if m != 0)
    win_b = 1 if wl.win_fp8 else 2
    attn = B * (attn_layers * K * (288 + 4) + t.n_layers * (WIN * 512 * win_b + H * 512 * 2) +
                t.n_layers * H * 512 * 4)
    idx = B * len(scans) * K * 4
    return {"index_scan": scan, "attention": attn, "step": scan + attn + idx}


def per_layer_path(dm, wl, stream, reps=10):
    """Device ms of the step's indexer and attention done layer by layer, as a
    decoder whose layer l + 1 query depends on layer l's output must: per layer,
    csa2_index_topk for a Full / Reindex layer (its own scan of the source's
    keys), then csa2_sparse_attn; replayed from a CUDA graph."""
    import torch
    import fp4_sparse_attention_pack_b200 as csa
    from fp4_sparse_attention_pack_b200 import workloads as W
    t = wl.table
    io = dm.io
    q, q_idx, w, out, idx = io.tensors[2], io.tensors[3], io.tensors[4], io.tensors[6], io.tensors[7]
    nmax = max(max(c.n_entries.cpu().tolist()) for c in dm.caches) + 64
    ws_scan = torch.empty(max(csa.index_topk_workspace(wl.B, nmax, wl.H_idx, wl.K), 16), dtype=torch.uint8,
                          device=dm.dev)
    ws_attn = torch.empty(max(csa.sparse_attn_workspace(wl.B, wl.H, wl.K), 16), dtype=torch.uint8,
                          device=dm.dev)

    def run():
        for l in range(t.n_layers):
            m = t.mode[l]
            if m in (W.FULL, W.REINDEX):
                csa.index_topk(dm.caches[t.src[l]].desc, q_idx[l], w[l], wl.K, idx[l], ws_scan,
                               stream=torch.cuda.current_stream())
            if m == W.SWA_ONLY:
                csa.sparse_attn(None, q[l], idx[l], 0, dm.windows[l].desc, wl.scale, out[l], ws_attn,
                                stream=torch.cuda.current_stream())
            else:
                src_l = t.idx_src[l] if m == W.REUSE else l
                csa.sparse_attn(dm.caches[t.src[l]].desc, q[l], idx[src_l], wl.K, dm.windows[l].desc, wl.scale,
                                out[l], ws_attn, stream=torch.cuda.current_stream())

    with torch.cuda.stream(stream):
        run()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / reps, len(t.scan_layers()) + t.n_layers


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(wl, seqs=(0,), layers=None, scores_out=None):
    """Time the oracle on `layers` for `seqs` (caches built untimed).  Returns
    (seconds per (scan layer, sequence), seconds per (attention-only layer,
    sequence), threads, description).  scores_out (a dict, optional) receives the
    oracle's fp64 indexer scores of every scan layer of the first sequence."""
    import numpy as np
    import oracle
    from fp4_sparse_attention_pack_b200 import workloads as W
    from tests.oracle_models import ref_cache, ref_window
    t = wl.table
    layers = layers if layers is not None else list(range(2, 8))
    srcs = sorted({t.src[l] for l in layers if t.mode[l] != W.SWA_ONLY})
    caches = {s: ref_cache(wl, s, list(seqs), wl.T, cap=wl.T // t.ratios[s] + 64) for s in srcs}
    t_scan, t_attn = [], []
    for i, b in enumerate(seqs):
        idx = {}
        for l in layers:
            m = t.mode[l]
            ring, cnt = ref_window(wl, l, b, wl.T)
            t0 = time.perf_counter()
            if m in (W.FULL, W.REINDEX):
                c = caches[t.src[l]]
                sc = c.scores(i, W.query_idx(wl, l, 0)[b], W.head_weights(wl, l, 0)[b])
                idx[l] = oracle.topk(sc, wl.K)
                if scores_out is not None and i == 0:
                    scores_out[l] = sc
            sel = idx.get(l if m != W.REUSE else t.idx_src[l])
            if m == W.SWA_ONLY:
                items = oracle.attention_items(np.zeros((1, 256), np.uint8), np.zeros((1, 32), np.uint8),
                                               0, np.zeros(0, np.int32), ring, min(cnt, WIN))
            else:
                c = caches[t.src[l]]
                items = oracle.attention_items(c.mc[i], c.ms[i], int(c.n[i]), sel, ring, min(cnt, WIN))
            oracle.attention(W.query(wl, l, 0)[b], items, wl.scale)
            dt = time.perf_counter() - t0
            (t_scan if m in (W.FULL, W.REINDEX) else t_attn).append(dt)
    n_scan = len(t.scan_layers())
    desc = (f"oracle on layers {layers[0]}-{layers[-1]} x sequences {list(seqs)} of the {t.n_layers}-layer "
            f"step (Top-K scan over {wl.T // t.ratios[t.src[layers[0]]]} entries, {wl.H_idx} heads, attention "
            f"over K + 128 items); per-layer-step time = {wl.B} x ({n_scan} scan-layer + "
            f"{t.n_layers - n_scan} attention-only-layer) sequence times")
    return (statistics.mean(t_scan) if t_scan else 0.0, statistics.mean(t_attn) if t_attn else 0.0,
            oracle.threads(), desc)


def cpu_baseline(wl, gpu_first_idx=None):
    """The oracle's sampled rate; with gpu_first_idx ([layers][K] indices of the
    GPU's first step for sequence 0), also the Top-K parity of those layers
    against the oracle's scores, with the tie-band counts."""
    scores = {}
    ts, ta, thr, desc = oracle_sample(wl, scores_out=scores)
    n_scan = len(wl.table.scan_layers())
    n_attn = wl.table.n_layers - n_scan
    step_s = wl.B * (n_scan * ts + n_attn * ta)
    base = {"value": wl.table.n_layers / step_s, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": desc}
    parity = None
    if gpu_first_idx is not None and scores:
        from tests.parity import TOPK_REL, topk_tie_report
        band = differ = 0
        ok = True
        for l, sc in sorted(scores.items()):
            try:
                r = topk_tie_report(gpu_first_idx[l], sc, wl.K)
                band += r["band"]
                differ += r["differ"]
            except AssertionError:
                ok = False
        parity = {"topk_rows_checked": len(scores), "topk_sets_match": ok, "tie_band_rel": TOPK_REL,
                  "tie_band_entries": band, "indices_differ": differ,
                  "rows": f"sequence 0 of layers {sorted(scores)} at the first decode step, GPU indices "
                          f"against the oracle's fp64 scores"}
    return base, parity


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank):
    import numpy as np
    from fp4_sparse_attention_pack_b200 import workloads as W
    import oracle
    from tests.oracle_models import ref_cache, ref_window
    if rank != 0:
        return
    wl = W.WORKLOADS[args.config]
    t = wl.table
    # untimed set-up: the oracle packs one sequence of every source
    caches = {s: ref_cache(wl, s, [0], wl.T, cap=wl.T // t.ratios[s] + 64) for s in range(t.n_sources)}
    rings = {l: ref_window(wl, l, 0, wl.T) for l in range(t.n_layers)}
    idx = {}

    def one(i):
        l = i % t.n_layers
        m = t.mode[l]
        if m in (W.FULL, W.REINDEX):
            c = caches[t.src[l]]
            idx[l] = oracle.topk(c.scores(0, W.query_idx(wl, l, 0)[0], W.head_weights(wl, l, 0)[0]), wl.K)
        ring, cnt = rings[l]
        if m == W.SWA_ONLY:
            items = oracle.attention_items(np.zeros((1, 256), np.uint8), np.zeros((1, 32), np.uint8), 0,
                                           np.zeros(0, np.int32), ring, min(cnt, WIN))
        else:
            c = caches[t.src[l]]
            sel = idx.get(l if m != W.REUSE else t.idx_src[l])
            if sel is None:  # a Reuse layer whose source was not run in this window
                src = t.idx_src[l]
                cs = caches[t.src[src]]
                sel = idx[src] = oracle.topk(cs.scores(0, W.query_idx(wl, src, 0)[0],
                                                       W.head_weights(wl, src, 0)[0]), wl.K)
            items = oracle.attention_items(c.mc[0], c.ms[0], int(c.n[0]), sel, ring, min(cnt, WIN))
        oracle.attention(W.query(wl, l, 0)[0], items, wl.scale)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(args.warmup + i)
    dt = time.perf_counter() - t0
    # each sample step is one layer for one of the batch's sequences: 1/B layer-step
    value = (args.steps / wl.B) / dt
    desc = (f"each step: the oracle on one layer (cycling through the 40-layer schedule) for one of the "
            f"{wl.B} sequences; value = (steps / {wl.B}) / seconds")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, 1),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import ctypes
    import torch
    import fp4_sparse_attention_pack_b200 as csa
    from fp4_sparse_attention_pack_b200 import engine, replicas, workloads as W

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    base = W.PROFILE_WORKLOADS[args.workload] if args.workload else W.WORKLOADS[args.config]
    wl = replicas.rank_workload(base, rank)  # each rank: its own batch of sequences
    extra = args.warmup + args.steps + 2 * args.profile_steps + 8
    dm = engine.DecodeModel(wl, dev, steps_capacity=extra)
    dm.fill()
    dm.gen_step_inputs(0)
    torch.cuda.synchronize()

    def barrier():
        replicas.barrier(world)

    stream = torch.cuda.Stream()
    torch.cuda.current_stream().wait_stream(torch.cuda.default_stream())
    # one eager step (also validates arguments), then capture
    with torch.cuda.stream(stream):
        dm.step(stream)
    stream.synchronize()
    first_idx = dm.idx[:, 0].cpu().numpy() if world == 1 else None  # the oracle sample's step
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        dm.step(torch.cuda.current_stream())
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            g.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    time.sleep(0.25)
    clocks.stop()
    ms = replicas.max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world, dev)
    n_ent = [dm.caches[s].n_entries.cpu().tolist() for s in range(dm.S)]
    status = dm.status_bits()

    # per-phase device times of the same step (eager launches with events)
    names = ["window_append", "cache_write", "query_quant", "index_scan", "topk", "attention",
             "attn_combine"]
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8 * args.profile_steps)]
    lib = csa.lib()
    lib.csa2_layer_step_profiled.restype = ctypes.c_int
    lib.csa2_layer_step_profiled.argtypes = [ctypes.POINTER(csa.csa2_model), ctypes.POINTER(csa.csa2_step_in),
                                             ctypes.POINTER(csa.csa2_step_out), ctypes.c_void_p,
                                             ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    phase = [[] for _ in names]
    for x in evs:  # torch creates the CUDA event on first record
        x.record(stream)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.profile_steps):
            e = evs[8 * i:8 * i + 8]
            arr = (ctypes.c_void_p * 8)(*[x.cuda_event for x in e])
            rc = lib.csa2_layer_step_profiled(ctypes.byref(dm.model), ctypes.byref(dm._in),
                                              ctypes.byref(dm._out), dm.ws.data_ptr(),
                                              dm.ws.numel(), stream.cuda_stream, arr)
            if rc != 0:
                raise csa.Csa2Error(rc, "csa2_layer_step_profiled")
    torch.cuda.synchronize()
    for i in range(args.profile_steps):
        e = evs[8 * i:8 * i + 8]
        for k in range(7):
            phase[k].append(e[k].elapsed_time(e[k + 1]))
    phase_ms = {n: statistics.mean(v) for n, v in zip(names, phase)}
    if wl.pool_blocks > 0:
        phase_note = ("hierarchical indexer: index_scan = the Full layers' scans; topk = their Top-K, "
                      "the pool build and the Reindex layers' pool scans with their Top-K")

    # End to end: every step copies its inputs from pinned host memory and reads its
    # outputs back, through csa2_layer_step.  Two device buffer sets and two copy
    # streams let step k's host->device copy and step k-1's device->host read overlap
    # step k-1's / k's compute (the steps themselves stay in order on one stream).
    e2e = None
    ios = [dm.io, dm.new_io()]
    host_in = [t.cpu().pin_memory() for t in dm.io.inputs]
    host_out = [[torch.empty_like(t, device="cpu").pin_memory() for t in io.outputs] for io in ios]
    h2d = sum(t.numel() * t.element_size() for t in dm.io.inputs)
    d2h = sum(t.numel() * t.element_size() for t in dm.io.outputs)
    e2e_steps = 0 if args.no_e2e else max(3, min(args.steps, 30))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in ios]
    comp_done = [torch.cuda.Event() for _ in ios]
    out_done = [torch.cuda.Event() for _ in ios]
    for e in comp_done + out_done:
        e.record(stream)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for k in range(e2e_steps):
        i = k & 1
        io = ios[i]
        with torch.cuda.stream(s_in):  # inputs of step k (buffer free once step k-2 ran)
            s_in.wait_event(comp_done[i])
            for d, h in zip(io.inputs, host_in):
                d.copy_(h, non_blocking=True)
            in_done[i].record(s_in)
        stream.wait_event(in_done[i])
        stream.wait_event(out_done[i])  # outputs of step k-2 have been read back
        dm.step(stream, io)
        comp_done[i].record(stream)
        with torch.cuda.stream(s_out):  # outputs of step k
            s_out.wait_event(comp_done[i])
            for d, h in zip(io.outputs, host_out[i]):
                h.copy_(d, non_blocking=True)
            out_done[i].record(s_out)
    stream.wait_stream(s_out)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = replicas.max_over_ranks(f0.elapsed_time(f1) / e2e_steps if e2e_steps else float("nan"), world, dev)
    barrier()
    if rank != 0:
        return
    # the same indexer + attention work layer by layer (no grouping of scans)
    pl_ms, pl_calls = per_layer_path(dm, wl, stream) if world == 1 and not args.no_per_layer else (None, None)

    L = wl.table.n_layers
    value = replicas.job_rate(L, world, ms / 1e3)
    kb = kernel_bytes(wl, n_ent)
    sb = survey_bytes(wl, n_ent)
    peak, peak_kind = measured_peaks()
    # roofline of the kernel with the largest share of the step
    dom = max(("index_scan", "attention", "topk"), key=lambda k: phase_ms[k])
    kernels = {k: {"algorithmic_bytes_per_launch": kb[k], "launch_ms": phase_ms[k],
                   "achieved_gbs": kb[k] / (phase_ms[k] / 1e3) / 1e9,
                   "frac_of_measured_hbm": kb[k] / (phase_ms[k] / 1e3) / 1e9 / peak,
                   "dram_bytes_per_launch": kernel_traffic(k)}
               for k in ("index_scan", "topk", "attention")}
    achieved = kernels[dom]["achieved_gbs"]
    launches_per_step = csa.layer_step_launches(dm.model, dm._in)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
        "config": dict(workload_config(wl, world),
                       l2="inputs larger than L2: %.2f GB read per step" % (kb["step"] / 1e9),
                       cuda_graph=True),
        "hbm": {"step_algorithmic_bytes": kb["step"],
                "achieved_gbs": kb["step"] / (ms / 1e3) / 1e9,
                "frac_of_measured": kb["step"] / (ms / 1e3) / (peak * 1e9),
                "accounting": "distinct bytes: each source's keys once per step for all its scans",
                "per_scan_accounting": {
                    "step_bytes": sb["step"], "achieved_gbs": sb["step"] / (ms / 1e3) / 1e9,
                    "frac_of_peak": sb["step"] / (ms / 1e3) / (peak * 1e9),
                    "index_scan_bytes": sb["index_scan"],
                    "index_scan_frac": sb["index_scan"] / (phase_ms["index_scan"] / 1e3) / (peak * 1e9),
                    "attention_bytes": sb["attention"],
                    "attention_frac": sb["attention"] / (phase_ms["attention"] / 1e3) / (peak * 1e9),
                    "note": "every scan reads its source's keys (a decoder scanning layer by layer); "
                            "the grouped step reads them once per source, so this fraction counts bytes "
                            "the kernel shares between scans"}},
        "per_layer_path": ({"ms_per_step": pl_ms, "launch_calls_per_step": pl_calls,
                            "grouped_ms_same_phases": phase_ms["query_quant"] + phase_ms["index_scan"] +
                            phase_ms["topk"] + phase_ms["attention"] + phase_ms["attn_combine"],
                            "per_scan_frac_of_peak": (sb["index_scan"] + sb["attention"]) /
                            (pl_ms / 1e3) / (peak * 1e9) if pl_ms else None,
                            "note": "csa2_index_topk per Full/Reindex layer then csa2_sparse_attn per layer, "
                                    "in layer order, replayed from a CUDA graph; excludes the window append "
                                    "and cache write of the step"}
                           if pl_ms is not None else None),
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": kernels[dom]["dram_bytes_per_launch"],
                     "peak_source": peak_kind, "algorithmic_bytes_per_launch": kb[dom],
                     "launch_ms": phase_ms[dom]},
        "kernels": kernels,
        "phase_ms": phase_ms,
        **({"phase_note": phase_note} if wl.pool_blocks > 0 else {}),
        "e2e": {"value": replicas.job_rate(L, world, e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "method": "csa2_layer_step with every step's inputs copied from pinned host memory and "
                          "its outputs read back; two buffer sets, copies on their own streams overlap "
                          "the neighbouring steps' compute"},
        "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_per_step": launches_per_step,
        "clocks": clocks.summary(t_wall0, t_wall1),
        "device_status": status,
    }
    if world == 1 and not args.no_cpu_baseline and not args.workload:
        line["cpu_baseline"], parity = cpu_baseline(W.WORKLOADS[args.config],
                                                    first_idx if wl.pool_blocks == 0 else None)
        if parity is not None:
            line["parity"] = parity
    print(json.dumps(line), flush=True)


def run_cache_io(args):
    """Prefix-cache export / import (csa2_cache_export / csa2_cache_import) of
    every sequence of one source at the workload's context, into device images
    and into pinned host images, and back into a cache with another page
    permutation.  Prints one JSON line (GB/s of image bytes moved)."""
    import torch
    import fp4_sparse_attention_pack_b200 as csa
    from fp4_sparse_attention_pack_b200 import engine, workloads as W
    wl = W.WORKLOADS[args.config]
    dm = engine.DecodeModel(wl, "cuda")
    dm.fill()
    src = dm.caches[0]
    B, cap = wl.B, src.max_pages * 64
    nbytes = csa.seq_image_bytes(cap)
    dst = engine.DeviceCache(B, src.max_pages, src.ratio, "cuda", page_seed=99)
    dev_img = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(B)]
    host_img = [torch.empty(nbytes, dtype=torch.uint8).pin_memory() for _ in range(B)]
    torch.cuda.synchronize()

    def timed(fn, reps):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / reps

    used = sum(356 * n for n in src.n_entries.cpu().tolist())  # bytes of the sequences' entries
    res = {}
    for name, imgs, reps in (("device", dev_img, 20), ("pinned_host", host_img, 5)):
        t_exp = timed(lambda: [csa.cache_export(src.desc, b, imgs[b], cap) for b in range(B)], reps)
        t_imp = timed(lambda: [csa.cache_import(dst.desc, b, imgs[b], cap) for b in range(B)], reps)
        res[name] = {"export_gbs": used / t_exp / 1e9, "import_gbs": used / t_imp / 1e9,
                     "export_ms": t_exp * 1e3, "import_ms": t_imp * 1e3}
    import numpy as np
    ok = all(np.array_equal(a, b) for a, b in zip(dst.logical(0, 0, 1024), src.logical(0, 0, 1024)))
    peak, peak_kind = measured_peaks()
    ach = 2 * used / (res["device"]["export_ms"] / 1e3) / 1e9  # entries read + image written
    line = {"metric": "prefix-cache image throughput", "unit": "GB/s", "value": res["device"]["export_gbs"],
            "higher_is_better": True, "n_gpus": 1, "data": "synthetic",
            "config": {"workload": wl.name, "source": 0, "sequences": B, "entries_per_sequence": wl.entries(0),
                       "entry_bytes": 356, "image_bytes_per_sequence": nbytes},
            "results": res, "status": src.status_bits() | dst.status_bits(),
            "round_trip_first_1024_entries_equal": ok,
            "roofline": {"kernel": "k_export", "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                         "frac": ach / peak, "peak_source": peak_kind, "traffic": None}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.measure == "cache_io":
        run_cache_io(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
