"""Pins for the oracle's number formats and its draft exponential.

E4M3 / E2M1 values follow the OCP 8-bit and 4-bit float definitions (sign,
exponent with bias 7 / 1, 3 / 1 mantissa bits, no infinities in E4M3,
largest finite 448 / 6), rounded to nearest even and saturated, as the
NVFP4 and FP8 paths of "DraftAttention2" App. C.1 require.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O

E4M3_HAND = [  # value -> code, from the format definition
    (0.0, 0x00), (-0.0, 0x80), (1.0, 0x38), (-2.0, 0xC0), (448.0, 0x7E), (480.0, 0x7E), (1e6, 0x7E),
    (-500.0, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -6, 0x08), (2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02),
    (17.0, 0x58), (19.0, 0x5A), (72.0, 0x69), (36.0, 0x61), (56.0, 0x66), (288.0, 0x79), (464.0, 0x7E),
    (0.875 * 2.0 ** -6, 0x07),
]

E2M1_HAND = [
    (0.0, 0x0), (0.5, 0x1), (1.0, 0x2), (1.5, 0x3), (2.0, 0x4), (3.0, 0x5), (4.0, 0x6), (6.0, 0x7),
    (2.5, 0x4), (5.0, 0x6), (0.25, 0x0), (0.75, 0x2), (7.0, 0x7), (1.25, 0x2), (1.75, 0x4), (3.5, 0x6),
    (-0.5, 0x9), (-6.0, 0xF), (-100.0, 0xF), (0.2, 0x0), (0.3, 0x1), (5.2, 0x7), (100.0, 0x7),
]


@pytest.mark.parametrize("x,code", E4M3_HAND)
def test_e4m3_hand_table(x, code):
    assert O.e4m3_encode(x) == code


@pytest.mark.parametrize("x,code", E2M1_HAND)
def test_e2m1_hand_table(x, code):
    assert O.e2m1_encode(x) == code


def test_e4m3_roundtrip_all_codes():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue  # NaN encodings
        v = O.e4m3_decode(c)
        assert O.e4m3_encode(v) == c or (v == 0 and O.e4m3_encode(v) in (0x00, 0x80))


def test_e2m1_roundtrip_all_codes():
    for c in range(16):
        assert O.e2m1_encode(O.e2m1_decode(c)) == c


def test_e4m3_matches_torch_cast_below_saturation():
    # torch's float8_e4m3fn cast rounds to nearest even; compare away from
    # saturation (torch maps overflow to NaN rather than saturating).
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 0.05, 1.0, 20.0, 100.0)])
    x = x[x.abs() < 440.0]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_encode(float(v)) for v in x.numpy()], np.uint8)
    assert np.array_equal(ref, got)


def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = O.e4m3_decode(c)
        if np.isnan(ref[c]):
            assert np.isnan(got)
        else:
            assert got == ref[c]


def test_e2m1_rounding_is_nearest():
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    rng = np.random.default_rng(0)
    for x in rng.uniform(0, 6, 5000).astype(np.float32):
        v = O.e2m1_decode(O.e2m1_encode(float(x)))
        assert abs(v - x) <= np.min(np.abs(grid - x)) + 1e-12


@pytest.mark.parametrize("x", [0.0, -1e-300, -1e-9, -0.5, -0.693147, -1.0, -3.7, -20.25, -100.0, -700.0,
                               -707.9, 0.3, 1.0, 10.0, 88.0])
def test_draft_exp_accuracy(x):
    # within 2 ulp of the correctly rounded exponential (math.exp is accurate to < 1 ulp)
    got = O.exp(x)
    ref = math.exp(x)
    assert abs(got - ref) <= 2 * math.ulp(ref)


def test_draft_exp_grid_and_flush():
    xs = np.linspace(-708, 0, 100001)
    got = np.array([O.exp(float(x)) for x in xs])
    ref = np.exp(xs)
    assert np.all(np.abs(got - ref) <= 3 * np.spacing(ref))
    assert O.exp(-708.5) == 0.0 and O.exp(-1000.0) == 0.0
    assert O.exp(0.0) == 1.0
