"""The divide-free quotient of the activation quantiser, emulated on the CPU.

The kernels compute x / s without a divide (Markstein's one-step correction,
IBM J. R&D 34(1), 1990): with r = RN(1/s),
    q0 = RN(x * r),  e = RN(q0 * s - x),  q = RN(q0 - e * r)
(the last two fused multiply-adds), and the packed form they run evaluates it
on -x with -r, giving -q, whose codes have their sign bits flipped back.
This test emulates both forms exactly in fp64 (the first FMA's exact value
fits in fp64; the second is rounded to fp32 correctly from an exact fp64 sum
and its error term) and checks, for bf16 pairs (amax, x) with |x| <= amax and
s = RN(amax / fmax) >= 2^-100, fmax the format's largest value (448 for E4M3;
6, 7.5 and 28 for the FP4 / FP6 weight formats, whose quantiser runs the same
negated form):
  * q is the IEEE quotient RN(x / s) whenever |x / s| >= 2^-11;
  * q has the IEEE quotient's sign always (below 2^-11 every format rounds
    both to a signed zero), and for E4M3 the same code;
  * the negated form gives -q bit for bit, signed zeros included.
By default a spread of amax values (every binade, random and extreme
mantissas); PTPC_FULL_QUOTIENT_SWEEP=1 runs every bf16 amax (about 90 s a format;
passes for all four).
"""
import os

import numpy as np
import pytest
import torch

F32 = np.float32
F64 = np.float64


def rn32_of_sum(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Correctly rounded fp32 of a + b for fp64 a, b whose exact sum fp64 may
    not hold: TwoSum gives hi + lo exactly; RN32(hi) is the answer unless hi
    is an fp32 midpoint that lo pushes off (then lo's sign decides)."""
    hi = a + b
    t = hi - a
    lo = (a - (hi - t)) + (b - t)
    f = hi.astype(F32)
    d = hi - f.astype(F64)
    toward = np.where(d > 0, np.inf, -np.inf).astype(F32)
    g = np.nextafter(f, toward)
    mid = (f.astype(F64) + g.astype(F64)) * 0.5
    at_mid = (d != 0) & (mid == hi) & (lo != 0)
    # at a midpoint: the exact sum lies on lo's side of it
    pick_g = at_mid & (np.sign(lo) == np.sign(g.astype(F64) - hi))
    return np.where(pick_g, g, f)


def markstein(x: np.ndarray, s: F32, r: F32) -> np.ndarray:
    q0 = (x * r).astype(F32)                                   # RN(x * r) in fp32
    e = (q0.astype(F64) * F64(s) - x.astype(F64)).astype(F32)  # exact in fp64, one rounding
    return rn32_of_sum(q0.astype(F64), -(e.astype(F64) * F64(r)))


def markstein_negated(x: np.ndarray, s: F32, r: F32) -> np.ndarray:
    nr = F32(-r)
    nq0 = (x * nr).astype(F32)
    e = (nq0.astype(F64) * F64(s) + x.astype(F64)).astype(F32)
    return rn32_of_sum(nq0.astype(F64), e.astype(F64) * F64(nr))


def e4m3_codes(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def bf16_values() -> np.ndarray:
    bits = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    v = bits.view(F32)
    return v[np.isfinite(v)]


def check_amax(amax: F32, xs_all: np.ndarray, fmax: float = 448.0):
    s = F32(amax / F32(fmax))
    if not s >= F32(2.0 ** -100):
        return
    r = F32(F32(1.0) / s)
    x = xs_all[np.abs(xs_all) <= amax]
    ieee = (x / s).astype(F32)
    q = markstein(x, s, r)
    big = np.abs(ieee) >= F32(2.0 ** -11)
    assert np.array_equal(q[big].view(np.uint32), ieee[big].view(np.uint32)), float(amax)
    assert np.array_equal(np.signbit(q), np.signbit(ieee)), float(amax)
    if fmax == 448.0:
        assert np.array_equal(e4m3_codes(q), e4m3_codes(ieee)), float(amax)
    nq = markstein_negated(x, s, r)
    assert np.array_equal(nq.view(np.uint32), (-q).view(np.uint32)), float(amax)
    if fmax == 448.0:
        assert np.array_equal(e4m3_codes(nq) ^ np.uint8(0x80), e4m3_codes(q)), float(amax)


def amax_sample(fmax: float = 448.0) -> np.ndarray:
    vals = bf16_values()
    pos = vals[(vals > 0) & (vals >= F32(fmax * 2.0 ** -100))]
    if os.environ.get("PTPC_FULL_QUOTIENT_SWEEP") == "1":
        return pos
    rng = np.random.default_rng(17)
    exps = np.unique(np.floor(np.log2(pos)).astype(int))
    picks = []
    for e in exps:
        p64 = pos.astype(F64)
        binade = pos[(p64 >= 2.0 ** e) & (p64 < 2.0 ** (e + 1))]
        picks += [binade[0], binade[-1], binade[rng.integers(len(binade))]]
    picks += [F32(448.0), F32(447.0), F32(1.0), pos[0], pos[-1]]
    return np.unique(np.array(picks, F32))


def test_rn32_of_sum_is_correctly_rounded():
    rng = np.random.default_rng(5)
    a = rng.standard_normal(200000)
    b = a * 2.0 ** -40 * rng.standard_normal(200000)
    got = rn32_of_sum(a, b)
    # exact reference through Python fractions on a subset
    from fractions import Fraction
    for i in range(0, 200000, 997):
        exact = Fraction(float(a[i])) + Fraction(float(b[i]))
        f = F32(got[i])
        lo, hi = np.nextafter(f, F32(-np.inf)), np.nextafter(f, F32(np.inf))
        d = abs(Fraction(float(f)) - exact)
        assert d <= abs(Fraction(float(lo)) - exact) and d <= abs(Fraction(float(hi)) - exact)
    # midpoints decided by the error term
    m = F64(1.0) + 2.0 ** -24                                       # fp32 midpoint of 1 and 1 + 2^-23
    assert rn32_of_sum(np.array([m]), np.array([2.0 ** -60]))[0] == F32(1.0 + 2.0 ** -23)
    assert rn32_of_sum(np.array([m]), np.array([-2.0 ** -60]))[0] == F32(1.0)
    assert rn32_of_sum(np.array([m]), np.array([0.0]))[0] == F32(1.0)      # tie to even


@pytest.mark.parametrize("fmax", [448.0, 6.0, 7.5, 28.0])
def test_divide_free_quotient_matches_ieee_division(fmax):
    xs = bf16_values()
    for amax in amax_sample(fmax):
        check_amax(F32(amax), xs, fmax)
