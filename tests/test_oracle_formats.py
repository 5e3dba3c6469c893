"""Pins of the oracle's number formats against the format definitions, the pages'
figures and an independent library (torch's float8_e4m3fn)."""
import math

import numpy as np
import pytest
import torch


def test_e2m1_magnitudes(ref, golden):
    # OCP MX v1.0 FP4 (E2M1) value table; the pages: exactly 8 magnitudes, max 6.
    mags = [ref.e2m1_value(c) for c in range(8)]
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert len(set(mags)) == golden["e2m1_magnitudes"]["value"]
    assert max(mags) == golden["e2m1_max"]["value"]
    for c in range(8):
        v = ref.e2m1_value(c | 8)
        assert v == -mags[c] and math.copysign(1.0, v) == -1.0


def test_e4m3_decode_matches_torch(ref, golden):
    codes = torch.arange(256, dtype=torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([ref.e4m3_value(c) for c in range(256)])
    nan = np.isnan(lib_vals)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib_vals[~nan])
    assert sorted(np.flatnonzero(nan)) == [0x7F, 0xFF]
    assert ref.e4m3_value(0x7E) == golden["e4m3_max"]["value"]
    assert ref.e4m3_value(0x01) == 2.0 ** -9 and ref.e4m3_value(0x08) == 2.0 ** -6
    assert ref.e4m3_value(0x38) == 1.0
    assert golden["e4m3_max"]["value"] * golden["e2m1_max"]["value"] == golden["max_representable"]["value"]


def test_e4m3_encode_matches_torch(ref):
    # torch rounds to nearest even and turns |v| >= 464 into NaN; below that the
    # two must agree on every value, including every midpoint between codes.
    vals = np.array([ref.e4m3_value(c) for c in range(0x7F)])
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(7)
    grid = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                           rng.uniform(0, 463.9, 4000), 2.0 ** rng.uniform(-14, 8.8, 4000)])
    grid = grid.astype(np.float32)
    grid = grid[grid < 464]
    lib = torch.from_numpy(grid).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([ref.e4m3_encode(float(v)) for v in grid])
    assert np.array_equal(mine, lib)
    # saturation to the largest finite value (448), never NaN
    for v in (464.0, 500.0, 2688.0, 1e30):
        assert ref.e4m3_encode(v) == 0x7E


def test_e8m0_values(ref):
    # OCP MX v1.0 E8M0: 2^(code - 127), code 0xFF is NaN.
    assert ref.e8m0_value(127) == 1.0
    assert ref.e8m0_value(0) == 2.0 ** -127
    assert ref.e8m0_value(254) == 2.0 ** 127
    assert ref.e8m0_value(130) == 8.0
    assert math.isnan(ref.e8m0_value(255))


def test_e2m1_encode_ties_and_saturation(ref):
    # round to nearest, ties to the even code (OCP MX conversion rule)
    cases = {0.0: 0, 0.2: 0, 0.25: 0, 0.26: 1, 0.5: 1, 0.75: 2, 1.0: 2, 1.25: 2, 1.3: 3,
             1.5: 3, 1.75: 4, 2.0: 4, 2.5: 4, 2.6: 5, 3.0: 5, 3.5: 6, 4.0: 6, 5.0: 6, 5.1: 7,
             6.0: 7, 7.0: 7, 1e9: 7}
    for v, c in cases.items():
        assert ref.e2m1_encode(v) == c, v
        if v > 0:
            assert ref.e2m1_encode(-v) == c | 8, -v
    assert ref.e2m1_encode(-0.1) == 0x8  # sign kept on a negative zero


def test_e2m1_encode_is_nearest(ref):
    # brute force: no representable value is strictly closer than the chosen one
    rng = np.random.default_rng(1)
    mags = np.array([ref.e2m1_value(c) for c in range(8)])
    for v in np.concatenate([rng.uniform(-7, 7, 3000), rng.normal(0, 1, 1000)]).astype(np.float32):
        c = ref.e2m1_encode(float(v))
        got = ref.e2m1_value(c)
        best = np.min(np.abs(mags - abs(float(v))))
        assert abs(abs(got) - abs(float(v))) == best
        assert (c & 8) == (8 if v < 0 else 0)


def test_mx_shared_exponent(ref):
    # OCP MX v1.0: X = floor(log2(amax)) - 2 for FP4 (emax_elem = 2); so that
    # amax / 2^X lies in [4, 8).
    assert ref.mx_shared_exp(6.0) == 0
    assert ref.mx_shared_exp(4.0) == 0
    assert ref.mx_shared_exp(1.0) == -2
    assert ref.mx_shared_exp(0.75) == -3
    assert ref.mx_shared_exp(3.0e38) == 125
    assert ref.mx_shared_exp(1e-45) == -127  # fp32 subnormal, clamped
    rng = np.random.default_rng(3)
    for a in (2.0 ** rng.uniform(-120, 120, 2000)).astype(np.float32):
        x = ref.mx_shared_exp(float(a))
        assert 4.0 * 2.0 ** x <= float(a) < 8.0 * 2.0 ** x


def test_spec_exp_accuracy(ref):
    # the agreed fp32 exp: within 2 ulp of the fp64 exponential in the normal range
    xs = np.concatenate([np.linspace(-87, 88, 20001), np.random.default_rng(5).normal(0, 3, 5000),
                         [0.0, 1.0, -1.0, 0.5]]).astype(np.float32)
    got = ref.spec_exp(xs).astype(np.float64)
    want = np.exp(xs.astype(np.float64))
    ulp = np.spacing(want.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(got - want) / ulp) <= 2.0
    assert ref.spec_exp([0.0])[0] == 1.0
    assert ref.spec_exp([100.0])[0] == np.inf
    assert ref.spec_exp([-200.0])[0] == 0.0
