"""Pins for the oracle's E4M3 codec (OCP FP8 format definition; CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_decode_landmarks():
    # Values fixed by the format: bias 7, 3 mantissa bits, max 448, one NaN pattern.
    d = fp8.decode
    assert d(0x00) == 0.0 and math.copysign(1, d(0x80)) == -1.0
    assert d(0x01) == 2.0 ** -9          # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert d(0x08) == 2.0 ** -6          # smallest normal
    assert d(0x38) == 1.0 and d(0x39) == 1.125 and d(0x40) == 2.0
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert np.isnan(d(0x7F)) and np.isnan(d(0xFF))
    assert d(0x77) == 240.0              # E=14 M=7: 1.875 * 2^7


def test_table_against_closed_form_count():
    vals = fp8.decode(np.arange(256))
    finite = vals[~np.isnan(vals)]
    assert len(finite) == 254
    pos = np.unique(finite[finite >= 0])
    assert len(pos) == 127 and pos.max() == 448.0


def test_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    assert np.array_equal(fp8.encode(fp8.decode(codes)), codes.astype(np.uint8))


def test_ties_to_even_and_saturation():
    e = fp8.encode
    assert e(1.0625) == 0x38             # midway 1.0 / 1.125 -> even code 0x38
    assert e(1.1875) == 0x3A             # midway 1.125 / 1.25 -> even code 0x3A
    assert e(1.0625 + 1e-6) == 0x39
    assert e(2.0 ** -10) == 0x00         # midway 0 / 2^-9 -> 0
    assert e(3 * 2.0 ** -10) == 0x02     # midway 2^-9 / 2^-8 -> even code 2
    assert e(-(2.0 ** -11)) == 0x80      # negative underflow keeps the sign
    assert e(448.0) == 0x7E and e(464.0) == 0x7E and e(1e9) == 0x7E and e(-1e9) == 0xFE
    assert e(float("nan")) == 0x7F


def test_matches_torch_cast_in_range():
    # torch's float8_e4m3fn cast rounds to nearest even; it does not saturate,
    # so compare inside the finite range only.
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-3, 0.1, 1.0, 30.0, 150.0)])
    x = x[x.abs() < 448]
    # add exact midpoints between neighbouring codes
    v = fp8.decode(np.arange(127))
    mids = torch.tensor((v[:-1] + v[1:]) / 2, dtype=torch.float32)
    x = torch.cat([x, mids, -mids])
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = fp8.encode(x.numpy())
    assert np.array_equal(got, ref)
