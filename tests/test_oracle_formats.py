"""Pins of the oracle's number formats (CPU only).

The oracle's codecs are checked against the published format definitions
(golden tables under tests/golden) and against torch's own bf16 and
float8_e4m3fn casts, which are independent implementations.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import formats as F


def test_e2m1_table_matches_ocp():
    for code, val in read_golden("e2m1_codes.txt"):
        got = F.e2m1_decode(np.uint8(code))
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)
        # every finite value encodes back to its own code
        assert F.e2m1_encode(np.float64(val)) == code


def test_e2m1_ties_and_saturation():
    # midpoints round to the even mantissa; beyond 6 saturates
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0,
             5.0: 4.0, 6.5: 6.0, 7.0: 6.0, 100.0: 6.0, 0.2499: 0.0, 0.2501: 0.5,
             4.99: 4.0, 5.01: 6.0}
    for v, want in cases.items():
        assert F.e2m1_round(v) == want, v
        assert F.e2m1_round(-v) == -want, v
    assert F.e2m1_encode(-0.1) == 0x8          # sign kept on underflow
    assert F.e2m1_encode(0.1) == 0x0


def test_e4m3_points_match_ocp():
    for code, val in read_golden("e4m3_points.txt"):
        got = F.e4m3_decode(np.uint8(code))
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val)


def test_e4m3_all_codes_vs_torch_and_roundtrip():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(codes)
    theirs = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(theirs)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], theirs[~nan])
    fin = codes[~nan]
    assert np.array_equal(F.e4m3_encode(ours[~nan]), fin)


def test_e4m3_rounding_vs_torch():
    g = np.random.default_rng(1)
    v = np.concatenate([
        g.uniform(-448, 448, 20000),
        g.standard_normal(20000) * 2.0 ** g.integers(-12, 8, 20000),
        # exact midpoints between neighbouring codes (ties to even)
        (F.e4m3_decode(np.arange(0, 0x7e, dtype=np.uint8)) +
         F.e4m3_decode(np.arange(1, 0x7f, dtype=np.uint8))) / 2,
    ])
    v32 = v.astype(np.float32)
    ours = F.e4m3_round(v32.astype(np.float64))
    theirs = torch.from_numpy(v32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, theirs)
    # satfinite beyond the largest finite value
    assert F.e4m3_round(1e6) == 448.0 and F.e4m3_round(-500.0) == -448.0
    assert F.e4m3_round(2.0 ** -11) == 0.0              # below half the min subnormal


def test_bf16_rounding_vs_torch():
    g = np.random.default_rng(2)
    f = np.concatenate([
        g.standard_normal(50000).astype(np.float32) * np.float32(1e3),
        # ties: low 16 bits exactly 0x8000, both parities of bit 16
        (g.integers(0x3f800000, 0x4f800000, 5000, dtype=np.uint32) & ~np.uint32(0xFFFF)
         | np.uint32(0x8000)).view(np.float32),
        np.array([1e-40, -1e-40, 3.4e38, 1e-45], dtype=np.float32),   # subnormals, overflow
    ]).astype(np.float32)
    ours = F.bf16_bits(f.astype(np.float64))
    theirs = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_int4_table():
    for code, val in read_golden("int4_range.txt"):
        assert F.int4_decode(np.uint8(code)) == val
        assert F.int4_encode(val) == code
    assert F.int4_encode(2.5) == 2 and F.int4_encode(3.5) == 4      # half to even
    assert F.int4_encode(-2.5) == (-2 & 0xF)
    assert F.int4_encode(9.0) == 7 and F.int4_encode(-9.0) == 8     # clamp


def test_nibble_packing_order():
    nib = np.array([[0x1, 0x2, 0x3, 0xF]], dtype=np.uint8)
    b = F.pack_nibbles(nib)
    assert b.tolist() == [[0x21, 0xF3]]          # even k in the low nibble
    assert np.array_equal(F.unpack_nibbles(b), nib)
