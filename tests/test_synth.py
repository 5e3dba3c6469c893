"""The seeded input generator: reproducible, counter-based, with the stated moments."""
import numpy as np

from fp4_sparse_attention_pack_b200 import synth
from fp4_sparse_attention_pack_b200 import workloads as W


def test_counter_based_slices():
    k = synth.key(3, synth.TID_SRC_X, 1)
    full = synth.normal_f32(k, 0, 10000)
    assert np.array_equal(full[1234:5678], synth.normal_f32(k, 1234, 5678 - 1234))
    assert not np.array_equal(full, synth.normal_f32(synth.key(3, synth.TID_SRC_X, 2), 0, 10000))


def test_normal_moments_and_exactness():
    z = synth.normal_f32(synth.key(0, 1, 0), 0, 2_000_000).astype(np.float64)
    assert abs(z.mean()) < 3e-3 and abs(z.var() - 1) < 5e-3
    assert np.abs(z).max() <= 6.0
    assert np.array_equal(z * 131072, np.round(z * 131072))


def test_uniform_range():
    u = synth.uniform_f32(synth.key(0, 8, 0), 0, 100000)
    assert u.min() >= 0 and u.max() < 1 and abs(u.mean() - 0.5) < 5e-3


def test_bf16_rounding_is_rne():
    k = synth.key(1, 2, 3)
    z = synth.normal_f32(k, 0, 1000)
    sc = np.linspace(0.5, 2, 512).astype(np.float32)
    b = synth.normal_bf16(k, 0, 1000, sc)
    prod = (z * sc[np.arange(1000) % 512]).astype(np.float32)
    back = synth.bf16_to_f32(b)
    # nearest bf16: error at most half a bf16 ulp
    ulp = 2.0 ** (np.floor(np.log2(np.abs(prod.astype(np.float64)) + 1e-30)) - 7)
    assert np.all(np.abs(back.astype(np.float64) - prod) <= ulp / 2 + 1e-30)


def test_workload_recipe_shapes():
    wl = W.small(W.WORKLOADS[3], B=1, T=256)
    assert W.tokens(wl, 0, 0, 0, 4).shape == (4, 512)
    assert W.w_idx(wl, 0).shape == (512, 128)
    sc = W.chan_scale(wl, 0)
    assert (sc[W.outlier_channels(wl, 0)] > 8).all() and len(W.outlier_channels(wl, 0)) == 5
    assert len(W.outlier_columns(wl, 0)) == 2
    assert W.query(wl, 0, 0).shape == (1, 64, 512)
    assert W.query_idx(wl, 0, 0).shape == (1, 64, 128)
    assert W.head_weights(wl, 0, 0).shape == (1, 64)
