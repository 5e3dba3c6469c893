"""Device state for the CSA2 C ABI: caches, windows, model tables, step buffers.

torch provides the device memory and the stream; every computation is a call
into libcsa2.so.  ``DecodeModel`` holds one workload's state (per-source paged
caches, per-layer windows, per-step inputs/outputs, workspace) and fills it
with the seeded recipe of :mod:`.workloads` using the device generator.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import (WIN_BF16, WIN_FP8, csa2_cache, csa2_model, csa2_step_in, csa2_step_out, csa2_window,
               layer_step, layer_step_workspace, pack_cache, synth, window_append, workloads as W)

D, D_IDX, WIN, PAGE = 512, 128, 128, 64


def _u8(n, dev):
    return torch.zeros(n, dtype=torch.uint8, device=dev)


class DeviceCache:
    """One source's paged cache for ``B`` sequences.  ``page_seed`` shuffles the
    physical pages (a seeded permutation) to exercise the page table."""

    def __init__(self, B: int, max_pages: int, ratio: int, device="cuda", page_seed=None,
                 spare_pages: int = 0):
        self.B, self.max_pages, self.ratio = B, max_pages, ratio
        self.num_pages = B * max_pages + spare_pages
        n = self.num_pages * PAGE
        self.main_codes = _u8(n * 256, device)
        self.main_scales = _u8(n * 32, device)
        self.idx_codes = _u8(n * 64, device)
        self.idx_scales = _u8(n * 4, device)
        pt = np.arange(B * max_pages, dtype=np.int32)
        if page_seed is not None:
            pt = np.random.default_rng(page_seed).permutation(self.num_pages)[:B * max_pages].astype(np.int32)
        self.page_table_host = pt.reshape(B, max_pages)
        self.page_table = torch.from_numpy(self.page_table_host.copy()).to(device)
        self.n_entries = torch.zeros(B, dtype=torch.int32, device=device)
        self.pend_x = torch.zeros(B, D, dtype=torch.float32, device=device)
        self.pend_g = torch.zeros(B, dtype=torch.float32, device=device)
        self.pend_valid = torch.zeros(B, dtype=torch.int32, device=device)
        self.status = torch.zeros(4, dtype=torch.int32, device=device)
        self.desc = csa2_cache(self.main_codes.data_ptr(), self.main_scales.data_ptr(),
                               self.idx_codes.data_ptr(), self.idx_scales.data_ptr(),
                               self.page_table.data_ptr(), self.n_entries.data_ptr(),
                               self.pend_x.data_ptr(), self.pend_g.data_ptr(),
                               self.pend_valid.data_ptr(), self.status.data_ptr(), B, max_pages,
                               self.num_pages, ratio)

    def logical(self, b: int, lo: int, hi: int):
        """Entries [lo, hi) of sequence b in logical layout (host numpy)."""
        e = np.arange(lo, hi)
        rows = self.page_table_host[b, e // PAGE].astype(np.int64) * PAGE + e % PAGE
        idx = torch.from_numpy(rows).to(self.main_codes.device)
        mc = self.main_codes.view(-1, 256)[idx].cpu().numpy()
        ms = self.main_scales.view(-1, 32)[idx].cpu().numpy()
        kc = self.idx_codes.view(-1, 64)[idx].cpu().numpy()
        ks = self.idx_scales.view(-1, 4)[idx].cpu().numpy()
        return mc, ms, kc, ks

    def status_bits(self) -> int:
        return int(self.status[0].item())


class DeviceWindow:
    """One layer's SWA ring: bf16 tokens, or E4M3 codes when fp8."""

    def __init__(self, B: int, device="cuda", fp8: bool = False):
        self.fp8 = fp8
        dt = torch.uint8 if fp8 else torch.bfloat16
        self.tokens = torch.zeros(B, WIN, D, dtype=dt, device=device)
        self.count = torch.zeros(B, dtype=torch.int32, device=device)
        self.desc = csa2_window(self.tokens.data_ptr(), self.count.data_ptr(), B, WIN_FP8 if fp8 else WIN_BF16)


def _ptr_array(tensors):
    arr = (ctypes.c_void_p * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = None if t is None else t.data_ptr()
    return arr


class DecodeModel:
    """All device state of one workload (see :class:`workloads.Workload`)."""

    def __init__(self, wl: W.Workload, device="cuda", page_seed=None, steps_capacity=None):
        self.wl, self.dev = wl, device
        t = wl.table
        self.L, self.S, B = t.n_layers, t.n_sources, wl.B
        extra = wl.steps if steps_capacity is None else steps_capacity
        self.caches = []
        for s in range(self.S):
            cap_tokens = wl.T + wl.append + extra + 2
            max_pages = (cap_tokens // t.ratios[s] + PAGE - 1) // PAGE
            self.caches.append(DeviceCache(B, max_pages, t.ratios[s], device,
                                           None if page_seed is None else page_seed + s))
        self.windows = [DeviceWindow(B, device, wl.win_fp8) for _ in range(self.L)]
        self.W = [torch.from_numpy(W.w_idx(wl, s)).to(device) for s in range(self.S)]
        self.chan = [torch.from_numpy(W.chan_scale(wl, s)).to(device) for s in range(self.S)]
        # model table (host arrays kept alive with the struct)
        self._mode = (ctypes.c_int32 * self.L)(*t.mode)
        self._src = (ctypes.c_int32 * self.L)(*[max(s, 0) for s in t.src])
        self._idx_src = (ctypes.c_int32 * self.L)(*[max(s, 0) for s in t.idx_src])
        self._caches = (csa2_cache * self.S)(*[c.desc for c in self.caches])
        self._w = (ctypes.c_void_p * self.S)(*[w.data_ptr() for w in self.W])
        self._wins = (csa2_window * self.L)(*[w.desc for w in self.windows])
        self.model = csa2_model(self.L, self.S, self._mode, self._src, self._idx_src, self._caches,
                                self._w, self._wins, B, wl.H, wl.H_idx, wl.K, wl.scale, wl.pool_blocks)
        self.ws = torch.empty(max(layer_step_workspace(self.model), 16), dtype=torch.uint8, device=device)
        # per-step buffers
        self.io = self.new_io()
        (self.x_new, self.g_new, self.q, self.q_idx, self.w, self.win_tok, self.out,
         self.idx) = self.io.tensors
        self._in, self._out = self.io.step_in, self.io.step_out
        self.position = wl.T  # tokens already in every stream

    class IO:
        """One set of per-step device buffers and the C structs that point at them."""

        def __init__(self, tensors, step_in, step_out, keep):
            self.tensors, self.step_in, self.step_out, self._keep = tensors, step_in, step_out, keep

        @property
        def inputs(self):
            return list(self.tensors[:6])

        @property
        def outputs(self):
            return list(self.tensors[6:])

    def new_io(self) -> "DecodeModel.IO":
        """A fresh set of step inputs (x_new, g_new, q, q_idx, w, win_tok) and outputs
        (out, idx); several sets let copies of one step overlap the compute of another."""
        wl, B, dev = self.wl, self.wl.B, self.dev
        x_new = torch.zeros(self.S, B, D, dtype=torch.bfloat16, device=dev)
        g_new = torch.zeros(self.S, B, dtype=torch.float32, device=dev)
        q = torch.zeros(self.L, B, wl.H, D, dtype=torch.bfloat16, device=dev)
        q_idx = torch.zeros(self.L, B, wl.H_idx, D_IDX, dtype=torch.bfloat16, device=dev)
        w = torch.zeros(self.L, B, wl.H_idx, dtype=torch.float32, device=dev)
        win_tok = torch.zeros(self.L, B, D, dtype=torch.bfloat16, device=dev)
        out = torch.zeros(self.L, B, wl.H, D, dtype=torch.float32, device=dev)
        idx = torch.full((self.L, B, wl.K), -1, dtype=torch.int32, device=dev)
        scan = set(self.wl.table.scan_layers())
        arrays = [_ptr_array([x_new[s] for s in range(self.S)]),
                  _ptr_array([g_new[s] for s in range(self.S)]),
                  _ptr_array([q[l] for l in range(self.L)]),
                  _ptr_array([q_idx[l] if l in scan else None for l in range(self.L)]),
                  _ptr_array([w[l] if l in scan else None for l in range(self.L)]),
                  _ptr_array([win_tok[l] for l in range(self.L)])]
        outs = [_ptr_array([out[l] for l in range(self.L)]),
                _ptr_array([idx[l] if l in scan else None for l in range(self.L)])]
        step_in = csa2_step_in(*arrays)
        step_out = csa2_step_out(*outs)
        return DecodeModel.IO((x_new, g_new, q, q_idx, w, win_tok, out, idx), step_in, step_out, arrays + outs)

    # ---------------------------------------------------------------- filling
    def fill(self, chunk_tokens: int = 8192):
        """Pack the first T tokens of every source and load the windows."""
        wl, B = self.wl, self.wl.B
        T = wl.T
        for s in range(self.S):
            kx = synth.key(wl.seed, synth.TID_SRC_X, s)
            kg = synth.key(wl.seed, synth.TID_SRC_G, s)
            ch = min(chunk_tokens, max(T, 1))
            xb = torch.empty(B, ch, D, dtype=torch.bfloat16, device=self.dev)
            gb = torch.empty(B, ch, dtype=torch.float32, device=self.dev)
            for t0 in range(0, T, ch):
                n = min(ch, T - t0)
                x, g = xb[:, :n].contiguous() if n != ch else xb, gb[:, :n].contiguous() if n != ch else gb
                synth.dev_normal_bf16_rows(x, kx, t0 * D, synth.TSTRIDE * D, B, n * D, self.chan[s])
                synth.dev_normal_f32_rows(g, kg, t0, synth.TSTRIDE, B, n)
                pack_cache(self.caches[s].desc, x, g, self.W[s])
        for l in range(self.L):
            self.load_window(l, T)

    def append_turn(self, chunk_tokens: int = 8192):
        """Agent turn of the prefix-cache workload: append tokens [T, T + append)
        of every source (paged cache write) and refresh the windows to T + append."""
        wl, B = self.wl, self.wl.B
        if wl.append <= 0:
            return
        for s in range(self.S):
            kx = synth.key(wl.seed, synth.TID_SRC_X, s)
            kg = synth.key(wl.seed, synth.TID_SRC_G, s)
            for t0 in range(wl.T, wl.T + wl.append, chunk_tokens):
                n = min(chunk_tokens, wl.T + wl.append - t0)
                x = torch.empty(B, n, D, dtype=torch.bfloat16, device=self.dev)
                g = torch.empty(B, n, dtype=torch.float32, device=self.dev)
                synth.dev_normal_bf16_rows(x, kx, t0 * D, synth.TSTRIDE * D, B, n * D, self.chan[s])
                synth.dev_normal_f32_rows(g, kg, t0, synth.TSTRIDE, B, n)
                pack_cache(self.caches[s].desc, x, g, self.W[s])
        for l in range(self.L):
            self.load_window(l, wl.T + wl.append)

    def load_window(self, l: int, T: int):
        wl, B = self.wl, self.wl.B
        n = min(T, WIN)
        p0 = T - n
        k = synth.key(wl.seed, synth.TID_WIN, l)
        tmp = torch.empty(B, n, D, dtype=torch.bfloat16, device=self.dev)
        synth.dev_normal_bf16_rows(tmp, k, p0 * D, synth.TSTRIDE * D, B, n * D)
        win = self.windows[l]
        if win.fp8:
            # the library encodes: replay the tokens through the window append
            win.count.fill_(p0)
            for i in range(n):
                window_append(win.desc, tmp[:, i].contiguous())
            return
        slots = (torch.arange(p0, T, device=self.dev) % WIN)
        win.tokens[:, slots] = tmp
        win.count.fill_(T)

    def gen_step_inputs(self, st: int):
        """Seeded inputs of decode step st (token position T + st) on the device."""
        wl, B = self.wl, self.wl.B
        p = wl.T + wl.append + st
        for s in range(self.S):
            synth.dev_normal_bf16_rows(self.x_new[s], synth.key(wl.seed, synth.TID_SRC_X, s), p * D,
                                       synth.TSTRIDE * D, B, D, self.chan[s])
            synth.dev_normal_f32_rows(self.g_new[s], synth.key(wl.seed, synth.TID_SRC_G, s), p,
                                      synth.TSTRIDE, B, 1)
        for l in range(self.L):
            nq = B * wl.H * D
            synth.dev_normal_bf16(self.q[l], synth.key(wl.seed, synth.TID_Q, l), st * nq)
            ni = B * wl.H_idx * D_IDX
            synth.dev_normal_bf16(self.q_idx[l], synth.key(wl.seed, synth.TID_QIDX, l), st * ni)
            synth.dev_uniform_f32(self.w[l], synth.key(wl.seed, synth.TID_WH, l), st * B * wl.H_idx)
            synth.dev_normal_bf16_rows(self.win_tok[l], synth.key(wl.seed, synth.TID_WIN, l), p * D,
                                       synth.TSTRIDE * D, B, D)

    def step(self, stream=None, io=None):
        io = self.io if io is None else io
        layer_step(self.model, io.step_in, io.step_out, self.ws, stream)

    def status_bits(self) -> int:
        return max(c.status_bits() for c in self.caches)
