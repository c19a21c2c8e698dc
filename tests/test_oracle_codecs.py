"""Pins of the oracle's number formats against their definitions and against
independent library conversions (numpy float16, torch bfloat16 and
float8_e4m3fn). The FP8 cache of the method (KV cache article, section
'再往后：压 KV 的三条路线': FP8 K/V with per-channel scaling factors) is read
as OCP E4M3 'FN' with round-to-nearest-even and saturation."""
import math

import numpy as np
import pytest
import torch

ALL16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def test_f16_decode_matches_numpy_for_every_pattern(oracle_mod):
    got = oracle_mod.f16_to_double(ALL16)
    want = ALL16.view(np.float16).astype(np.float64)
    assert np.array_equal(got, want, equal_nan=True)


def test_bf16_decode_matches_torch_for_every_pattern(oracle_mod):
    got = oracle_mod.bf16_to_double(ALL16)
    want = torch.from_numpy(ALL16.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(got, want, equal_nan=True)


def test_e4m3_decode_all_codes(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    got = oracle_mod.e4m3_to_double(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(got, want, equal_nan=True)
    # landmarks of the format: largest finite, smallest normal, smallest subnormal, NaN
    assert got[0x7E] == 448.0 and got[0xFE] == -448.0
    assert got[0x08] == 2.0 ** -6
    assert got[0x01] == 2.0 ** -9
    assert math.isnan(got[0x7F]) and math.isnan(got[0xFF])
    assert np.sum(np.isnan(got)) == 2  # no infinities, two NaN codes
    # finite positive codes are strictly increasing
    pos = got[:0x7F]
    assert np.all(np.diff(pos) > 0)


def test_e4m3_round_trip_every_finite_code(oracle_mod):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle_mod.e4m3_to_double(codes).astype(np.float32)
    assert np.array_equal(oracle_mod.e4m3_from_float(vals), codes)


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    x = ALL16.view(np.float16).astype(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448.0)]
    got = oracle_mod.e4m3_from_float(x)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)


def test_e4m3_ties_round_to_even(oracle_mod):
    codes = np.arange(0, 0x7E, dtype=np.uint8)  # positive finite, below the top code
    lo = oracle_mod.e4m3_to_double(codes)
    hi = oracle_mod.e4m3_to_double(codes + 1)
    mid = ((lo + hi) / 2).astype(np.float32)  # exact: midpoints need 5 significant bits
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)
    got = oracle_mod.e4m3_from_float(mid)
    even = np.where(codes % 2 == 0, codes, codes + 1).astype(np.uint8)
    assert np.array_equal(got, even)
    # just off the midpoint, rounding goes to the nearer neighbour
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(0))
    assert np.array_equal(oracle_mod.e4m3_from_float(up), (codes + 1).astype(np.uint8))
    assert np.array_equal(oracle_mod.e4m3_from_float(dn), codes)
    # negative values mirror positive ones with the sign bit
    assert np.array_equal(oracle_mod.e4m3_from_float(-mid), even | 0x80)


@pytest.mark.parametrize("x,code", [
    (448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (480.0, 0x7E), (1e6, 0x7E),
    (float("inf"), 0x7E), (-500.0, 0xFE), (float("-inf"), 0xFE),
    (2.0 ** -10, 0x00), (3 * 2.0 ** -11, 0x01), (2.0 ** -6 - 2.0 ** -10, 0x08),
    (0.0, 0x00), (-0.0, 0x80),
])
def test_e4m3_saturation_and_subnormals(oracle_mod, x, code):
    assert int(oracle_mod.e4m3_from_float(np.array([x], np.float32))[0]) == code


def test_e4m3_nan_maps_to_nan_code(oracle_mod):
    c = int(oracle_mod.e4m3_from_float(np.array([np.nan], np.float32))[0])
    assert c & 0x7F == 0x7F
