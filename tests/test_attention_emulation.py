"""Why the tensor-memory attention kernel writes P as three E4M3 terms and
keeps its reference maximum lazily: a numpy model of its arithmetic (q as
two E4M3 terms after a power-of-two scale, scores in base 2, a reference
maximum per head that moves only when a score exceeds it by 8 and then to
`below` under the tile's maximum, a power-of-two unit over the value scales,
P written as `nterms` E4M3 terms, tiles of 128 positions; sums in fp64),
compared with the fp64 oracle under the GEMM tolerance on inputs made as the
GPU attention tests make them.

* three terms with the reference 4 below the tile's maximum (the kernel):
  within the tolerance;
* two terms with the same reference: outside it (outputs that cancel in the
  outlier channels of V);
* two terms with the reference at the tile's maximum (P <= 1): outside it;
* three terms with the reference at the tile's maximum: within it, so the
  lazy reference is there for speed (the tile maxima are needed only when a
  score moves it), not for accuracy once P has three terms.

E4M3 rounding is PyTorch's cast (round to nearest even, as the kernel's
cvt.rn.satfinite for values inside +-448).  CPU only.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic


def e4m3(x) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).double().numpy()


def make_kv(T, H, D, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((T, H, D)).astype(np.float32)
    x *= rng.lognormal(0.0, 1.0, size=(T, H, 1)).astype(np.float32)
    x[:, :, rng.choice(D, 2, replace=False)] *= 20.0          # a few outlier channels per head
    return synthetic.to_bf16_bits(x)


def make_case(lens, Hq, Hkv, D, bs):
    """Paged E4M3 caches (through the oracle's quantiser and scatter) and
    queries, seeded like the GPU attention tests."""
    seed = sum(lens) + Hq
    rng = np.random.Generator(np.random.PCG64(seed))
    B = len(lens)
    mb = max(1, max((l + bs - 1) // bs for l in lens))
    nb = B * mb + 3
    perm = rng.permutation(nb)
    tables = np.full((B, mb), -1, np.int32)
    k = 0
    for b, l in enumerate(lens):
        n = (l + bs - 1) // bs
        tables[b, :n] = perm[k:k + n]
        k += n
    slots = [tables[b, p // bs] * bs + p % bs for b, l in enumerate(lens) for p in range(l)]
    T = len(slots)
    cache = []
    for j in (1, 2):
        codes, scales = oracle.kv_quantize(make_kv(max(T, 1), Hkv, D, seed + j)[:T])
        cc = np.zeros((nb, bs, Hkv, D), np.uint8)
        cs = np.zeros((nb, bs, Hkv), np.float32)
        oracle.kv_cache_write(cc, cs, codes, scales, slots, bs)
        cache += [cc, cs]
    rng = np.random.Generator(np.random.PCG64(11))
    q = synthetic.to_bf16_bits(rng.standard_normal((B, Hq, D)).astype(np.float32) * 2.0)
    return q, cache, tables, lens, bs


def model(q_bits, cache, tables, lens, bs, scale, nterms, below, lazy=8.0):
    """The kernel's arithmetic, one chunk a sequence, fp64 sums."""
    kc, ks, vc, vs = cache
    B, Hq, D = q_bits.shape
    Hkv = kc.shape[2]
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    qf = torch.from_numpy(q_bits.astype(np.int32) << 16).view(torch.float32).double().numpy()
    out = np.zeros((B, Hq, D))
    for b, L in enumerate(lens):
        if L == 0:
            continue
        pos = np.arange(L)
        sl = tables[b, pos // bs] * bs + pos % bs
        for h in range(Hq):
            g = h // (Hq // Hkv)
            K = dec[kc.reshape(-1, Hkv, D)[sl, g]]
            V = dec[vc.reshape(-1, Hkv, D)[sl, g]]
            ksc = ks.reshape(-1, Hkv)[sl, g].astype(np.float64)
            vsc = vs.reshape(-1, Hkv)[sl, g].astype(np.float64)
            amax = np.abs(qf[b, h]).max()
            sig = 2.0 ** math.floor(math.log2(448.0 / amax))
            a = qf[b, h] * sig
            hi = e4m3(a)
            lo = e4m3((a - hi) * 16)
            s_all = (K @ hi + (K @ lo) / 16) * ksc * (scale * math.log2(math.e)) / sig
            m, l, unit, O = -np.inf, 0.0, 0.0, np.zeros(D)
            for t0 in range(0, L, 128):
                s, v = s_all[t0:t0 + 128], vsc[t0:t0 + 128]
                if v.max() > unit:                       # the value unit moves up
                    nu = 2.0 ** math.ceil(math.log2(v.max()))
                    O *= unit / nu if unit > 0 else 0.0
                    unit = nu
                if s.max() > m + lazy:                   # the reference maximum moves
                    mn = s.max() - below
                    f = 0.0 if m == -np.inf else 2.0 ** (m - mn)
                    O *= f
                    l *= f
                    m = mn
                e = 2.0 ** (s - m)
                l += e.sum()
                r = e * v / unit
                P = np.zeros_like(r)
                for i in range(nterms):
                    t = e4m3(r)
                    P += t / 16.0 ** i
                    r = (r - t) * 16
                O += P @ V[t0:t0 + 128]
            out[b, h] = O * unit / l
    return out


def worst_ratio(case, nterms, below):
    """Largest |model - oracle| / (1e-2 |oracle| + 1e-3 rms(oracle)) over the
    outputs, the model rounded to bf16 like the kernel's output."""
    q, cache, tables, lens, bs = case
    D = q.shape[2]
    scale = D ** -0.5
    kc, ks, vc, vs = cache
    ref = oracle.bf16_to_float(oracle.decode_attention_reference(q, kc, ks, vc, vs, tables, lens, bs, scale))
    got = oracle.bf16_to_float(oracle.bf16_from_double(model(q, cache, tables, lens, bs, scale, nterms, below)))
    worst = 0.0
    for b in range(len(lens)):
        r = ref[b].astype(np.float64)
        rms = float(np.sqrt(np.mean(r * r)))
        if rms == 0.0:
            continue
        ratio = np.abs(got[b] - r) / (1e-2 * np.abs(r) + 1e-3 * rms)
        assert np.isfinite(ratio).all()
        worst = max(worst, float(ratio.max()))
    return worst


@pytest.fixture(scope="module")
def cases():
    return {"ragged": make_case([1, 15, 16, 17, 100], 8, 1, 128, 16),
            "long": make_case([0, 5, 2049], 28, 4, 128, 16)}


def test_three_terms_with_the_lazy_reference_meet_the_tolerance(cases):
    for name, case in cases.items():
        assert worst_ratio(case, 3, 4.0) < 0.75, name


def test_two_terms_miss_the_tolerance(cases):
    assert worst_ratio(cases["long"], 2, 4.0) > 2.0           # the kernel's reference, P up to 2^8
    assert worst_ratio(cases["ragged"], 2, 0.0) > 2.0         # reference at the tile maximum, P <= 1


def test_three_terms_also_meet_it_with_the_reference_at_the_maximum(cases):
    for name, case in cases.items():
        assert worst_ratio(case, 3, 0.0) < 0.75, name
