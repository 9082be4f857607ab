"""Pins of the oracle's E4M3 and bf16 codecs against values fixed outside it:
the OCP FP8 E4M3 definition (closed-form special values, exhaustive round
trip, every rounding midpoint), brute-force nearest-code search, and
PyTorch's own float8_e4m3fn / bfloat16 casts as an independent library."""
import math
import struct

import numpy as np
import pytest
import torch

import oracle


def torch_decode_all():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def test_decode_matches_library_for_all_256_codes():
    got = oracle.e4m3_decode_table()
    ref = torch_decode_all()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    # negative zero keeps its sign
    assert math.copysign(1.0, got[0x80]) == -1.0


def test_decode_special_values_from_definition():
    d = oracle.e4m3_decode
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0       # largest finite
    assert d(0x01) == 2.0 ** -9                          # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9                      # largest subnormal
    assert d(0x08) == 2.0 ** -6                          # smallest normal
    assert d(0x38) == 1.0                                # bias 7
    assert d(0x00) == 0.0
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))   # S.1111.111


def test_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_decode_table()[codes].astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


@pytest.mark.parametrize("v", [448.0, 449.0, 463.9, 464.0, 479.0, 480.0, 1e30, 3.4e38, float("inf")])
def test_saturation(v):
    assert oracle.e4m3_encode([v])[0] == 0x7E
    assert oracle.e4m3_encode([-v])[0] == 0xFE


def _positive_grid():
    t = oracle.e4m3_decode_table()
    return [(c, t[c]) for c in range(0x00, 0x7F)]      # 0 .. 448, ascending


def test_every_midpoint_rounds_to_even_code():
    grid = _positive_grid()
    assert len(grid) == 127                             # 126 gaps
    for (c0, v0), (c1, v1) in zip(grid, grid[1:]):
        mid = (v0 + v1) / 2                              # exact in fp32 (few bits)
        assert np.float32(mid) == mid
        even = c0 if c0 % 2 == 0 else c1
        assert oracle.e4m3_encode([mid])[0] == even, (c0, c1, mid)
        assert oracle.e4m3_encode([-mid])[0] == (even | 0x80)
        below = np.nextafter(np.float32(mid), np.float32(0))
        above = np.nextafter(np.float32(mid), np.float32(1e9))
        assert oracle.e4m3_encode([below])[0] == c0
        assert oracle.e4m3_encode([above])[0] == c1


def test_small_value_cases():
    e = lambda v: int(oracle.e4m3_encode([v])[0])
    assert e(2.0 ** -10) == 0x00                         # tie between 0 and 2^-9 -> 0
    assert e(-(2.0 ** -10)) == 0x80
    assert e(1.5 * 2.0 ** -9) == 0x02                    # tie between m=1 and m=2 -> 2
    assert e(2.0 ** -11) == 0x00
    assert e(7.5 * 2.0 ** -9) == 0x08                    # tie 7*2^-9 | 2^-6 -> even 0x08
    assert e(-0.0) == 0x80
    assert e(0.0) == 0x00
    assert e(1e-45) == 0x00                              # fp32 subnormal input


def _brute_force_encode(v: float) -> int:
    """Nearest finite E4M3 value by exhaustive search; ties to the even code;
    saturating at 448."""
    t = torch_decode_all()
    sign = 0x80 if math.copysign(1.0, v) < 0 else 0
    a = abs(v)
    if a >= 448.0:
        return sign | 0x7E
    best, best_d = None, None
    for c in range(0x00, 0x7F):
        d = abs(t[c] - a)
        if best is None or d < best_d or (d == best_d and c % 2 == 0):
            best, best_d = c, d
    return sign | best


def test_encode_matches_brute_force_search():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(400) * 50,
        rng.standard_normal(300) * 0.01,
        rng.standard_normal(300) * 1e-3,
        rng.uniform(-470, 470, 200),
    ]).astype(np.float32)
    got = oracle.e4m3_encode(vals)
    for v, g in zip(vals, got):
        assert g == _brute_force_encode(float(v)), v


def test_encode_matches_library_cast_on_random_values():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) < 464.0)]
    v = np.concatenate([v, (rng.standard_normal(1_000_000) * 30).astype(np.float32)])
    v = v[np.abs(v) < 464.0]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


# ---------------------------------------------------------------- bf16

def test_bf16_rounding_matches_library_on_fp32_values():
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 2 ** 32, size=1_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_from_double(v.astype(np.float64))
    # PyTorch rounds values just below the overflow threshold to inf the same way
    assert np.array_equal(got, ref)


def test_bf16_rounding_fp64_cases():
    f = lambda v: int(oracle.bf16_from_double([v])[0])
    assert f(1.0 + 2.0 ** -8) == 0x3F80                        # tie -> even (1.0)
    assert f(1.0 + 3 * 2.0 ** -8) == 0x3F82                    # tie -> even (mantissa 2)
    assert f(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81           # just above the tie
    assert f(1.0 + 2.0 ** -8 - 2.0 ** -40) == 0x3F80           # just below the tie
    assert f(-0.0) == 0x8000
    assert f(2.0 ** -133) == 0x0001                            # smallest subnormal
    assert f(2.0 ** -134) == 0x0000                            # tie -> even 0
    assert f(1.5 * 2.0 ** -133) == 0x0002
    assert f(255.0 * 2.0 ** 120) == 0x7F7F                     # largest finite
    assert f(255.5 * 2.0 ** 120) == 0x7F80                     # tie -> even -> inf
    assert f(255.5 * 2.0 ** 120 - 2.0 ** 100) == 0x7F7F
    assert f(2.0 ** 129) == 0x7F80
    assert f(-(2.0 ** 129)) == 0xFF80
    assert f(float("inf")) == 0x7F80 and f(float("-inf")) == 0xFF80
    nan = f(float("nan"))
    assert nan & 0x7F80 == 0x7F80 and nan & 0x007F != 0                # a NaN pattern


def test_bf16_to_float_is_exact_widening():
    b = np.arange(0, 2 ** 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_float(b)
    ref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
