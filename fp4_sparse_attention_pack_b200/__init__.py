"""Python binding of the CSA2 C ABI (``include/csa2.h``, ``libcsa2.so``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (torch supplies device memory and
streams); calls are enqueued on torch's current stream.  Importing this
package raises if the library has not been built -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

from ._build import LIB

__all__ = ["Csa2Error", "lib", "csa2_cache", "csa2_window", "csa2_model", "csa2_step_in",
           "csa2_step_out", "pack_cache", "index_topk", "index_topk_workspace", "index_pool_workspace",
           "index_topk_pool", "index_topk_in_pool", "POOL_BLOCK", "MAX_POOL_BLOCKS", "WIN_BF16", "WIN_FP8",
           "sparse_attn",
           "sparse_attn_workspace", "window_append", "layer_step", "layer_step_workspace", "layer_step_launches", "seq_image_bytes", "cache_export",
           "cache_import",
           "SWA_ONLY", "FULL", "REINDEX", "REUSE", "DTYPE_BF16", "DTYPE_F32"]

SWA_ONLY, FULL, REINDEX, REUSE = 0, 1, 2, 3
DTYPE_BF16, DTYPE_F32 = 0, 1
POOL_BLOCK, MAX_POOL_BLOCKS = 8, 8192
WIN_BF16, WIN_FP8 = 0, 1
DEVERR_CAPACITY, DEVERR_PAGE, DEVERR_COUNT, DEVERR_TIMEOUT, DEVERR_IMAGE = 1, 2, 4, 8, 16

_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t


class Csa2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {lib().csa2_strerror(status).decode()} ({status})")
        self.status = status


class csa2_cache(ctypes.Structure):
    _fields_ = [("main_codes", _vp), ("main_scales", _vp), ("idx_codes", _vp), ("idx_scales", _vp),
                ("page_table", _vp), ("n_entries", _vp), ("pend_x", _vp), ("pend_g", _vp),
                ("pend_valid", _vp), ("status", _vp), ("batch", _i32), ("max_pages", _i32),
                ("num_pages", _i32), ("ratio", _i32)]


class csa2_window(ctypes.Structure):
    _fields_ = [("tokens", _vp), ("count", _vp), ("batch", _i32), ("dtype", _i32)]


class csa2_model(ctypes.Structure):
    _fields_ = [("n_layers", _i32), ("n_sources", _i32), ("mode", ctypes.POINTER(_i32)),
                ("src", ctypes.POINTER(_i32)), ("idx_src", ctypes.POINTER(_i32)),
                ("caches", ctypes.POINTER(csa2_cache)), ("w_idx", ctypes.POINTER(_vp)),
                ("windows", ctypes.POINTER(csa2_window)), ("batch", _i32), ("H", _i32),
                ("H_idx", _i32), ("K", _i32), ("scale", _f32), ("pool_blocks", _i32)]


class csa2_step_in(ctypes.Structure):
    _fields_ = [("x_new", ctypes.POINTER(_vp)), ("g_new", ctypes.POINTER(_vp)),
                ("q", ctypes.POINTER(_vp)), ("q_idx", ctypes.POINTER(_vp)), ("w", ctypes.POINTER(_vp)),
                ("win_tok", ctypes.POINTER(_vp))]


class csa2_step_out(ctypes.Structure):
    _fields_ = [("out", ctypes.POINTER(_vp)), ("idx", ctypes.POINTER(_vp))]


_lib = None


def lib():
    """The loaded libcsa2.so (raises if it is missing: no CPU fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError(f"{LIB} is not built; run __graft_entry__.build() first")
        L = ctypes.CDLL(LIB)
        P = ctypes.POINTER
        for name, res, args in [
            ("csa2_version", ctypes.c_int, []),
            ("csa2_strerror", ctypes.c_char_p, [ctypes.c_int]),
            ("csa2_pack_cache", ctypes.c_int, [P(csa2_cache), _vp, ctypes.c_int, _vp, _vp, ctypes.c_int, _vp]),
            ("csa2_index_topk_workspace", _sz, [ctypes.c_int] * 4),
            ("csa2_index_topk", ctypes.c_int, [P(csa2_cache), _vp, _vp, ctypes.c_int, ctypes.c_int, _vp,
                                               _vp, _vp, _sz, _vp]),
            ("csa2_index_pool_workspace", _sz, [ctypes.c_int] * 5),
            ("csa2_index_topk_pool", ctypes.c_int, [P(csa2_cache), _vp, _vp, ctypes.c_int, ctypes.c_int, _vp,
                                                    _vp, ctypes.c_int, _vp, _vp, _sz, _vp]),
            ("csa2_index_topk_in_pool", ctypes.c_int, [P(csa2_cache), _vp, _vp, ctypes.c_int, ctypes.c_int,
                                                       _vp, ctypes.c_int, _vp, _vp, _vp, _sz, _vp]),
            ("csa2_sparse_attn_workspace", _sz, [ctypes.c_int] * 3),
            ("csa2_sparse_attn", ctypes.c_int, [P(csa2_cache), _vp, ctypes.c_int, _vp, ctypes.c_int,
                                                P(csa2_window), ctypes.c_float, _vp, _vp, _sz, _vp]),
            ("csa2_window_append", ctypes.c_int, [P(csa2_window), _vp, _vp]),
            ("csa2_layer_step_workspace", _sz, [P(csa2_model)]),
            ("csa2_layer_step", ctypes.c_int, [P(csa2_model), P(csa2_step_in), P(csa2_step_out), _vp,
                                               _sz, _vp]),
            ("csa2_layer_step_launches", ctypes.c_int, [P(csa2_model), P(csa2_step_in)]),
            ("csa2_seq_image_bytes", _sz, [ctypes.c_int]),
            ("csa2_cache_export", ctypes.c_int, [P(csa2_cache), ctypes.c_int, _vp, ctypes.c_int, _vp]),
            ("csa2_cache_import", ctypes.c_int, [P(csa2_cache), ctypes.c_int, _vp, ctypes.c_int, _vp]),
        ]:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ok(rc: int, what: str):
    if rc != 0:
        raise Csa2Error(rc, what)


def pack_cache(cache: csa2_cache, x, gates, w_idx, stream=None):
    """Append x [batch][T][512] (bf16 or fp32) with gate logits [batch][T]."""
    import torch
    dt = DTYPE_F32 if x.dtype == torch.float32 else DTYPE_BF16
    T = x.shape[1]
    _ok(lib().csa2_pack_cache(ctypes.byref(cache), _ptr(x), dt, _ptr(gates), _ptr(w_idx), T,
                              _stream(stream)), "csa2_pack_cache")


def index_topk_workspace(batch: int, max_entries: int, H_idx: int, K: int) -> int:
    return int(lib().csa2_index_topk_workspace(batch, max_entries, H_idx, K))


def index_topk(cache: csa2_cache, q_idx, w, K: int, idx_out, ws, score_out=None, stream=None):
    H_idx = q_idx.shape[1]
    _ok(lib().csa2_index_topk(ctypes.byref(cache), _ptr(q_idx), _ptr(w), H_idx, K, _ptr(idx_out),
                              _ptr(score_out), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)), "csa2_index_topk")


def index_pool_workspace(batch: int, max_entries: int, H_idx: int, K: int, pool_blocks: int) -> int:
    return int(lib().csa2_index_pool_workspace(batch, max_entries, H_idx, K, pool_blocks))


def index_topk_pool(cache: csa2_cache, q_idx, w, K: int, idx_out, pool_out, ws, score_out=None,
                    stream=None):
    """Full-layer scan: Top-K into idx_out and the block pool into pool_out
    [batch][pool_blocks]."""
    H_idx = q_idx.shape[1]
    _ok(lib().csa2_index_topk_pool(ctypes.byref(cache), _ptr(q_idx), _ptr(w), H_idx, K, _ptr(idx_out),
                                   _ptr(score_out), pool_out.shape[1], _ptr(pool_out), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "csa2_index_topk_pool")


def index_topk_in_pool(cache: csa2_cache, q_idx, w, K: int, pool, idx_out, ws, score_out=None, stream=None):
    """Scan restricted to pool [batch][pool_blocks]; Top-K into idx_out."""
    H_idx = q_idx.shape[1]
    _ok(lib().csa2_index_topk_in_pool(ctypes.byref(cache), _ptr(q_idx), _ptr(w), H_idx, K, _ptr(pool),
                                      pool.shape[1], _ptr(idx_out), _ptr(score_out), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)),
        "csa2_index_topk_in_pool")


def sparse_attn_workspace(batch: int, H: int, K: int) -> int:
    return int(lib().csa2_sparse_attn_workspace(batch, H, K))


def sparse_attn(cache, q, idx, K: int, win: csa2_window, scale: float, out, ws, stream=None):
    H = q.shape[1]
    cp = ctypes.byref(cache) if cache is not None else None
    _ok(lib().csa2_sparse_attn(cp, _ptr(q), H, _ptr(idx), K, ctypes.byref(win), float(scale), _ptr(out),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
        "csa2_sparse_attn")


def selftest_wait_timeout(status, timeout_us: int, stream=None):
    """Make one bounded device wait run out (see csa2_selftest_wait_timeout):
    CSA2_DEVERR_TIMEOUT is ORed into status[0] after timeout_us microseconds."""
    f = lib().csa2_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [_vp, ctypes.c_uint, _vp]
    _ok(f(_ptr(status), int(timeout_us), _stream(stream)), "csa2_selftest_wait_timeout")


def window_append(win: csa2_window, tok, stream=None):
    _ok(lib().csa2_window_append(ctypes.byref(win), _ptr(tok), _stream(stream)), "csa2_window_append")


def layer_step_workspace(model: csa2_model) -> int:
    return int(lib().csa2_layer_step_workspace(ctypes.byref(model)))


def layer_step(model: csa2_model, step_in: csa2_step_in, step_out: csa2_step_out, ws, stream=None):
    _ok(lib().csa2_layer_step(ctypes.byref(model), ctypes.byref(step_in), ctypes.byref(step_out),
                              _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
        "csa2_layer_step")


def layer_step_launches(model: csa2_model, step_in: csa2_step_in) -> int:
    """Kernel launches one layer_step call enqueues (no work is enqueued)."""
    n = int(lib().csa2_layer_step_launches(ctypes.byref(model), ctypes.byref(step_in)))
    if n < 0:
        raise Csa2Error(n, "csa2_layer_step_launches")
    return n


def seq_image_bytes(capacity: int) -> int:
    """Bytes of a one-sequence cache image with room for `capacity` entries."""
    return int(lib().csa2_seq_image_bytes(capacity))


def cache_export(cache: csa2_cache, seq: int, image, capacity: int, stream=None):
    """Copy sequence `seq` of `cache` into `image` (a uint8 tensor the device can
    address: CUDA memory or pinned host memory) in logical entry order."""
    _ok(lib().csa2_cache_export(ctypes.byref(cache), seq, _ptr(image), capacity, _stream(stream)),
        "csa2_cache_export")


def cache_import(cache: csa2_cache, seq: int, image, capacity: int, stream=None):
    """Write an image made by cache_export into sequence `seq` of `cache`."""
    _ok(lib().csa2_cache_import(ctypes.byref(cache), seq, _ptr(image), capacity, _stream(stream)),
        "csa2_cache_import")


def index_topk_noalloc(cache: csa2_cache, q_idx, w, K: int, idx_out, score_out=None, stream=None):
    """csa2_index_topk without a workspace: for callers that cannot allocate
    device memory (a fixed memory pool, no allocation on the decode path).  The
    scratch is a fixed 8 MiB array inside the library; see include/csa2.h."""
    f = lib().csa2_index_topk_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(csa2_cache), _vp, _vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp]
    H_idx = q_idx.shape[1]
    _ok(f(ctypes.byref(cache), _ptr(q_idx), _ptr(w), H_idx, K, _ptr(idx_out), _ptr(score_out),
          _stream(stream)), "csa2_index_topk_noalloc")
