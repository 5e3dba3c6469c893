"""The multi-GPU path on CPU: two gloo ranks run the replica plumbing the
benchmark uses (per-rank sequences, barrier, max-over-ranks time, whole-job
rate).  The decode path shards by sequence with no exchange step, so this is
all the cross-rank logic there is."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

from fp4_sparse_attention_pack_b200 import replicas
from fp4_sparse_attention_pack_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = replicas.rank_workload(W.WORKLOADS[2], rank)
        tok = W.tokens(wl, 0, 0, 0, 2)              # this rank's first source tokens (host generator)
        replicas.barrier(world)
        ms = replicas.max_over_ranks(1.5 + rank, world)  # per-rank step times 1.5 and 2.5 ms
        rate = replicas.job_rate(wl.table.n_layers, world, ms / 1e3)
        out[rank] = (wl.seed, wl.B, wl.T, tok.tobytes(), ms, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_by_sequence_and_time_by_the_slowest():
    world = 2
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    (s0, b0, t0, tok0, ms0, r0), (s1, b1, t1, tok1, ms1, r1) = res[0], res[1]
    assert (b0, t0) == (b1, t1) == (16, 131072)                # same shapes on every rank
    assert s1 - s0 == replicas.RANK_SEED_STRIDE and tok0 != tok1  # different sequences
    assert ms0 == ms1 == 2.5                                     # both ranks see the slowest time
    assert r0 == r1 == pytest.approx(40 * 2 / 2.5e-3)            # all ranks' layer-steps over that time


def test_single_rank_needs_no_process_group():
    assert replicas.max_over_ranks(3.0, 1) == 3.0
    replicas.barrier(1)
    assert replicas.job_rate(40, 1, 0.5e-3) == pytest.approx(80000)
    wl = replicas.rank_workload(W.WORKLOADS[2], 0)
    assert wl == W.WORKLOADS[2]
