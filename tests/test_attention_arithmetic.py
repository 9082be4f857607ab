"""The number representations the decode-attention kernels rely on, checked
on the CPU with PyTorch's E4M3 cast (round to nearest even, the rounding of
the kernels' cvt.rn.satfinite conversions for values inside +-448).

* q as two E4M3 terms after a power-of-two scale sigma that puts the head's
  largest |q| in (224, 448]: hi = E4M3(q sigma), lo = E4M3((q sigma - hi) * 16),
  q sigma = hi + lo / 16 exactly wherever |q sigma| >= 2^-6 (E4M3's smallest
  normal), for every bf16 value; below it the error is at most 2^-14, under
  2^-20 of the head's largest element.  A value just below 2^-6 whose first
  term rounds up to the normal 2^-6 is one of the inexact ones.
* P as three E4M3 terms, P = t1 + t2 / 16 + t3 / 256: relative error at most
  2^-14 for P >= 2^-4 (the kernel's P lies below 2^8), where two terms leave
  up to 2^-9, which is why the tensor-memory kernel writes three.
"""
import numpy as np
import torch


def e4m3(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float8_e4m3fn).float()


def all_bf16_within(limit: float) -> torch.Tensor:
    v = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    return v[torch.isfinite(v) & (v.abs() <= limit)]


def test_q_as_two_e4m3_terms_is_exact_above_the_smallest_normal():
    a = all_bf16_within(448.0)
    hi = e4m3(a)
    lo = e4m3((a - hi) * 16)
    rec = hi + lo / 16
    big = a.abs() >= 2.0 ** -6
    assert torch.equal(rec[big], a[big])
    small_err = (rec[~big] - a[~big]).abs().max().item()
    assert small_err <= 2.0 ** -14
    assert small_err / 224.0 < 2.0 ** -20
    # the boundary: values just below 2^-6 round to a normal first term, inexactly
    edge = (~big) & (hi.abs() >= 2.0 ** -6) & (rec != a)
    assert edge.any()


def test_power_of_two_scale_puts_the_head_maximum_in_224_448():
    rng = np.random.default_rng(3)
    amax = np.concatenate([np.exp2(rng.uniform(-126, 127, 5000)), [2.0 ** -126, 1.0, 448.0, 449.0, 3e38]])
    amax = amax.astype(np.float32)
    # the largest power of two <= 448 / amax: the exponent bits of the quotient
    with np.errstate(over="ignore"):                   # 448 / 2^-126 overflows to inf: capped below
        q = (np.float32(448.0) / amax).astype(np.float32)
    sig = (q.view(np.uint32) & np.uint32(0x7F800000)).view(np.float32)
    sig = np.minimum(sig, np.float32(2.0 ** 126))
    top = amax.astype(np.float64) * sig
    ok = sig < np.float32(2.0 ** 126)        # not capped
    assert np.all((top[ok] > 224.0) & (top[ok] <= 448.0))


def test_p_as_three_e4m3_terms():
    g = torch.Generator().manual_seed(0)
    p = torch.exp2(torch.rand(1_000_000, generator=g) * 12 - 4)      # 2^-4 .. 2^8
    p = torch.cat([p, torch.tensor([2.0 ** -4, 1.0, 255.9, 256.0])])
    t1 = e4m3(p)
    r1 = (p - t1) * 16
    t2 = e4m3(r1)
    t3 = e4m3((r1 - t2) * 16)
    rel3 = ((t1 + t2 / 16 + t3 / 256) - p).abs() / p
    rel2 = ((t1 + t2 / 16) - p).abs() / p
    assert rel3.max().item() <= 2.0 ** -14
    assert 2.0 ** -10 < rel2.max().item() <= 2.0 ** -9
