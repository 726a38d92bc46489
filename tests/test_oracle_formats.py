"""Pins for the oracle's stored-precision decoding (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import brute, formats


def test_bf16_all_patterns_match_torch_widening():
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = formats.bf16_bits_to_f64(u)
    lib = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])


def test_e4m3_all_codes_match_torch_and_brute():
    codes = np.arange(256, dtype=np.uint8)
    ours = formats.e4m3_bits_to_f64(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    br = np.array([brute.e4m3(c) for c in codes])
    assert np.array_equal(np.isnan(br), nan)
    assert np.array_equal(br[~nan], lib[~nan])


@pytest.mark.parametrize("code,value", [
    (0x7E, 448.0),             # largest finite
    (0xFE, -448.0),
    (0x01, 2.0 ** -9),         # smallest subnormal
    (0x07, 7 * 2.0 ** -9),     # largest subnormal
    (0x08, 2.0 ** -6),         # smallest normal
    (0x38, 1.0),
    (0x3C, 1.5),
    (0xB8, -1.0),
    (0x00, 0.0),
])
def test_e4m3_spec_values(code, value):
    assert formats.e4m3_bits_to_f64(np.uint8(code)) == value


def test_e4m3_nan_codes():
    assert math.isnan(formats.e4m3_bits_to_f64(np.uint8(0x7F)))
    assert math.isnan(formats.e4m3_bits_to_f64(np.uint8(0xFF)))


def test_e4m3_rne_midpoints_via_library_cast():
    # 1 + 1/16 is the midpoint between 1 and 1.125: RNE keeps the even mantissa (1.0);
    # 1 + 3/16 lies between 1.125 and 1.25: RNE goes to the even one (1.25).
    v = torch.tensor([1.0 + 1 / 16, 1.0 + 3 / 16, 448.0, 2.0 ** -10], dtype=torch.float32)
    q = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = formats.e4m3_bits_to_f64(q)
    assert list(got) == [1.0, 1.25, 448.0, 0.0]


def test_bf16_brute_decode_agrees():
    u = np.array([0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F, 0x0000, 0x8000], dtype=np.uint16)
    assert [brute.bf16(v) for v in u] == list(formats.bf16_bits_to_f64(u))
