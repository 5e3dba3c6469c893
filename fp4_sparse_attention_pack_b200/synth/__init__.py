"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

Input generation only: nothing here computes a step of the CSA2 method.  The
definition (SplitMix64 counters, Irwin-Hall(12) normals, RNE to bf16) is
stated in ``synth_host.c``; ``synth_dev.cu`` implements the same definition
for the device so that large inputs can be produced in HBM directly.  Host
and device values agree bit for bit (checked by a GPU test).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(_HERE, "libcsa2_synth_host.so")
DEV_SO = os.path.join(_HERE, "libcsa2_synth_dev.so")

# tensor ids of the recipe (the ``tensor`` argument of :func:`key`)
TID_SRC_X = 1     # source tokens, sub = source; index (b * TSTRIDE + t) * 512 + c
TID_SRC_G = 2     # source gate logits, sub = source; index b * TSTRIDE + t
TID_CHAN = 3      # per-channel lognormal exponents, sub = source; 512 values
TID_W = 4         # indexer projection W[512][128], sub = source
TID_OUTLIER = 5   # outlier channel choice, sub = source
TID_Q = 6         # main query, sub = layer; index ((st * B + b) * H + h) * 512 + c
TID_QIDX = 7      # indexer query, sub = layer; index ((st * B + b) * Hi + h) * 128 + c
TID_WH = 8        # indexer head weights, sub = layer; index (st * B + b) * Hi + h
TID_WIN = 9       # SWA window tokens, sub = layer; index (b * TSTRIDE + pos) * 512 + c
TSTRIDE = 1 << 24  # token-position stride of one sequence in a token stream


def build_host(force: bool = False) -> str:
    """Compile the host generator with gcc (OpenMP) next to this file."""
    src = os.path.join(_HERE, "synth_host.c")
    if force or not os.path.exists(HOST_SO) or os.path.getmtime(HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                               src, "-o", HOST_SO])
    return HOST_SO


def build_dev(force: bool = False) -> str:
    """Compile the device generator with nvcc for sm_100a next to this file."""
    src = os.path.join(_HERE, "synth_dev.cu")
    if force or not os.path.exists(DEV_SO) or os.path.getmtime(DEV_SO) < os.path.getmtime(src):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-Xcompiler", "-fPIC", "-shared", "-fmad=false", src, "-o", DEV_SO])
    return DEV_SO


_host = None
_dev = None


def _lib():
    global _host
    if _host is None:
        _host = ctypes.CDLL(build_host())
        u64, i64 = ctypes.c_uint64, ctypes.c_int64
        vp = ctypes.c_void_p
        _host.synth_key.restype = u64
        _host.synth_key.argtypes = [u64, u64, u64]
        _host.synth_u64.restype = u64
        _host.synth_u64.argtypes = [u64, u64]
        _host.synth_normal_f32.argtypes = [u64, u64, i64, vp]
        _host.synth_normal_bf16.argtypes = [u64, u64, i64, vp, i64, vp]
        _host.synth_normal_scaled_f32.argtypes = [u64, u64, i64, ctypes.c_float, vp]
        _host.synth_uniform_f32.argtypes = [u64, u64, i64, vp]
        _host.synth_normal_bf16_rows.argtypes = [u64, u64, u64, i64, i64, vp, i64, vp]
        _host.synth_normal_f32_rows.argtypes = [u64, u64, u64, i64, i64, vp]
        _host.synth_u64_array.argtypes = [u64, u64, i64, vp]
    return _host


def _devlib():
    global _dev
    if _dev is None:
        _dev = ctypes.CDLL(build_dev())
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        _dev.synth_dev_normal_bf16.argtypes = [u64, u64, i64, vp, i64, vp, vp]
        _dev.synth_dev_normal_scaled_f32.argtypes = [u64, u64, i64, ctypes.c_float, vp, vp]
        _dev.synth_dev_uniform_f32.argtypes = [u64, u64, i64, vp, vp]
        _dev.synth_dev_normal_bf16_rows.argtypes = [u64, u64, u64, i64, i64, vp, i64, vp, vp]
        _dev.synth_dev_normal_f32_rows.argtypes = [u64, u64, u64, i64, i64, vp, vp]
    return _dev


def key(seed: int, tensor: int, sub: int = 0) -> int:
    return int(_lib().synth_key(seed, tensor, sub))


def u64(k: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint64)
    _lib().synth_u64_array(k, start, n, out.ctypes.data)
    return out


def normal_f32(k: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float32)
    _lib().synth_normal_f32(k, start, n, out.ctypes.data)
    return out


def normal_scaled_f32(k: int, start: int, n: int, scale: float) -> np.ndarray:
    out = np.empty(n, np.float32)
    _lib().synth_normal_scaled_f32(k, start, n, float(scale), out.ctypes.data)
    return out


def normal_bf16(k: int, start: int, n: int, scale: np.ndarray | None = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of normal * scale[channel]."""
    out = np.empty(n, np.uint16)
    if scale is not None:
        scale = np.ascontiguousarray(scale, np.float32)
        _lib().synth_normal_bf16(k, start, n, scale.ctypes.data, scale.size, out.ctypes.data)
    else:
        _lib().synth_normal_bf16(k, start, n, None, 1, out.ctypes.data)
    return out


def normal_bf16_rows(k: int, start: int, row_stride: int, rows: int, row_len: int,
                     scale: np.ndarray | None = None) -> np.ndarray:
    """bf16 bits [rows][row_len]: element start + r * row_stride + j."""
    out = np.empty((rows, row_len), np.uint16)
    if scale is not None:
        scale = np.ascontiguousarray(scale, np.float32)
        _lib().synth_normal_bf16_rows(k, start, row_stride, rows, row_len, scale.ctypes.data,
                                      scale.size, out.ctypes.data)
    else:
        _lib().synth_normal_bf16_rows(k, start, row_stride, rows, row_len, None, 1, out.ctypes.data)
    return out


def normal_f32_rows(k: int, start: int, row_stride: int, rows: int, row_len: int) -> np.ndarray:
    out = np.empty((rows, row_len), np.float32)
    _lib().synth_normal_f32_rows(k, start, row_stride, rows, row_len, out.ctypes.data)
    return out


def uniform_f32(k: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float32)
    _lib().synth_uniform_f32(k, start, n, out.ctypes.data)
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---- device fills (torch tensors as plumbing: pointer + stream) ----------------

def _check(rc: int):
    if rc != 0:
        raise RuntimeError(f"synthetic generator launch failed: cuda error {rc}")


def dev_normal_bf16(out, k: int, start: int, scale=None):
    import torch
    n = out.numel()
    sp = scale.data_ptr() if scale is not None else None
    nchan = scale.numel() if scale is not None else 1
    _check(_devlib().synth_dev_normal_bf16(k, start, n, sp, nchan, out.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream))


def dev_normal_bf16_rows(out, k: int, start: int, row_stride: int, rows: int, row_len: int,
                         scale=None):
    import torch
    assert out.numel() == rows * row_len
    sp = scale.data_ptr() if scale is not None else None
    nchan = scale.numel() if scale is not None else 1
    _check(_devlib().synth_dev_normal_bf16_rows(k, start, row_stride, rows, row_len, sp, nchan,
                                                out.data_ptr(),
                                                torch.cuda.current_stream().cuda_stream))


def dev_normal_f32_rows(out, k: int, start: int, row_stride: int, rows: int, row_len: int):
    import torch
    assert out.numel() == rows * row_len
    _check(_devlib().synth_dev_normal_f32_rows(k, start, row_stride, rows, row_len, out.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream))


def dev_normal_scaled_f32(out, k: int, start: int, scale: float):
    import torch
    _check(_devlib().synth_dev_normal_scaled_f32(k, start, out.numel(), float(scale), out.data_ptr(),
                                                 torch.cuda.current_stream().cuda_stream))


def dev_uniform_f32(out, k: int, start: int):
    import torch
    _check(_devlib().synth_dev_uniform_f32(k, start, out.numel(), out.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream))
