"""Pins of the oracle's scaled GEMM.

Fixed outside the oracle: exact integer dot products (every E4M3 value is an
integer multiple of 2^-9), exact rational arithmetic for the epilogue with a
brute-force bf16 rounding, the hand-derived worked example, and the page's
identities: the naive two-step path equals the fused one, per-tensor scaling
is the equal-scale special case, and transposing both operands transposes the
output."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic
from golden_io import float_array, hex_array, read_sections


def int_units_table():
    """E4M3 values in integer units of 2^-9, from PyTorch's decoder."""
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    out = []
    for c in range(256):
        if np.isnan(v[c]):
            out.append(None)
        else:
            u = v[c] * 512
            assert u == int(u)
            out.append(int(u))
    return out


def random_codes(rng, shape, extreme=False):
    if extreme:
        return rng.choice(np.array([0x7E, 0xFE], np.uint8), size=shape)
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x7E      # no NaN codes
    return c


@pytest.mark.parametrize("T,Ci,Co,extreme", [(3, 5, 4, False), (7, 64, 9, False),
                                            (2, 2048, 3, True), (5, 300, 6, False)])
def test_acc_is_exact_integer_dot_product(T, Ci, Co, extreme):
    rng = np.random.default_rng(T * 1000 + Ci)
    Xq = random_codes(rng, (T, Ci), extreme)
    Wq_t = random_codes(rng, (Co, Ci), extreme)
    acc = oracle.gemm_acc64(Xq, Wq_t)
    units = int_units_table()
    for t in range(T):
        for o in range(Co):
            s = sum(units[a] * units[b] for a, b in zip(Xq[t], Wq_t[o]))
            assert Fraction(acc[t, o]) == Fraction(s, 2 ** 18)


def test_acc_exact_at_full_depth():
    Ci = 28672
    Xq = np.full((1, Ci), 0x7E, np.uint8)
    Wq_t = np.full((2, Ci), 0x7E, np.uint8)
    Wq_t[1, ::2] = 0xFE
    acc = oracle.gemm_acc64(Xq, Wq_t)
    assert acc[0, 0] == Ci * 448.0 * 448.0 and acc[0, 1] == 0.0


def brute_bf16(fr: Fraction) -> int:
    """bf16 bits of an exact rational, round-half-to-even, by bracketing."""
    if fr == 0:
        return 0
    sign = 0x8000 if fr < 0 else 0
    a = abs(fr)
    # binary search over the monotone positive finite bf16 values
    vals = lambda b: Fraction(float(oracle.bf16_to_float(np.array([b], np.uint16))[0]))
    lo, hi = 0, 0x7F7F
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if vals(mid) <= a:
            lo = mid
        else:
            hi = mid
    dl, dh = a - vals(lo), vals(hi) - a
    if dl < dh or (dl == dh and lo % 2 == 0):
        return sign | lo
    return sign | hi


def test_reference_epilogue_matches_exact_rational():
    rng = np.random.default_rng(9)
    T, Ci, Co = 4, 96, 5
    Xq = random_codes(rng, (T, Ci))
    Wq_t = random_codes(rng, (Co, Ci))
    xs = (rng.random(T) * 1e-2 + 1e-4).astype(np.float32)
    ws = (rng.random(Co) * 1e-3 + 1e-5).astype(np.float32)
    out = oracle.scaled_mm_reference(Xq, xs, Wq_t, ws)
    units = int_units_table()
    for t in range(T):
        for o in range(Co):
            s = sum(units[a] * units[b] for a, b in zip(Xq[t], Wq_t[o]))
            exact = Fraction(s, 2 ** 18) * Fraction(float(xs[t])) * Fraction(float(ws[o]))
            assert out[t, o] == brute_bf16(exact), (t, o)


def test_hand_example_gemm():
    g = read_sections("hand_example.txt")
    Xq = hex_array(g["Xq_u8"], np.uint8)
    Wq_t = hex_array(g["Wq_t_u8"], np.uint8)
    xs = float_array(g["x_scale_f32"], np.float32)[0]
    ws = float_array(g["w_scale_f32"], np.float32)[0]
    assert np.array_equal(oracle.gemm_acc64(Xq, Wq_t), float_array(g["acc_f64"], np.float64))
    expect = hex_array(g["out_bf16"], np.uint16)
    assert np.array_equal(oracle.scaled_mm_reference(Xq, xs, Wq_t, ws), expect)
    assert np.array_equal(oracle.fused_f32(Xq, xs, Wq_t, ws), expect)
    out, _, _ = oracle.linear_reference(hex_array(g["X_bf16"], np.uint16), Wq_t, ws)
    assert np.array_equal(out, expect)


def test_naive_two_step_equals_fused():
    w = synthetic.TINY
    X = synthetic.make_x(w, 0, 16, 256)
    W = synthetic.make_w(w, 0, 256, 512)
    Xq, xs = oracle.quant_act(X)
    Wq_t, ws = oracle.quant_weight(W)
    y = oracle.naive_step1_f32(Xq, Wq_t)
    naive = oracle.naive_step2_apply_scales(y, xs, ws)
    fused = oracle.fused_f32(Xq, xs, Wq_t, ws)
    assert np.array_equal(naive, fused)


def test_per_tensor_special_case():
    rng = np.random.default_rng(4)
    Xq = random_codes(rng, (6, 128))
    Wq_t = random_codes(rng, (10, 128))
    sx, sw = np.float32(0.0123), np.float32(0.000456)
    out = oracle.scaled_mm_reference(Xq, np.full(6, sx), Wq_t, np.full(10, sw))
    acc = oracle.gemm_acc64(Xq, Wq_t)
    assert np.array_equal(out, oracle.bf16_from_double(acc * (float(sx) * float(sw))))


def test_transposed_operands_give_transposed_output():
    rng = np.random.default_rng(6)
    Xq = random_codes(rng, (9, 64))
    Wq_t = random_codes(rng, (13, 64))
    xs = (rng.random(9) + 0.1).astype(np.float32)
    ws = (rng.random(13) + 0.1).astype(np.float32)
    a = oracle.scaled_mm_reference(Xq, xs, Wq_t, ws)
    b = oracle.scaled_mm_reference(Wq_t, ws, Xq, xs)
    assert np.array_equal(a, b.T)


def test_row_subset_equals_full_rows():
    rng = np.random.default_rng(8)
    Xq = random_codes(rng, (20, 64))
    Wq_t = random_codes(rng, (7, 64))
    xs = (rng.random(20) + 0.1).astype(np.float32)
    ws = (rng.random(7) + 0.1).astype(np.float32)
    rows = [0, 3, 19, 7]
    full = oracle.scaled_mm_reference(Xq, xs, Wq_t, ws)
    assert np.array_equal(oracle.scaled_mm_reference(Xq, xs, Wq_t, ws, rows), full[rows])
    full = oracle.fused_f32(Xq, xs, Wq_t, ws)
    assert np.array_equal(oracle.fused_f32(Xq, xs, Wq_t, ws, rows), full[rows])


def test_kv_cache_oracle():
    """The FP8 KV-cache oracle: per-(token, head) codes are the per-token
    quantiser's on the [T * H, D] rows (scale = amax / 448, bit-exact), the
    paged scatter puts every token at its slot, and decode attention reduces
    to textbook cases: one context token returns its dequantised V exactly
    (softmax of one score is 1), identical keys average the values, and a
    dominant score selects its value."""
    rng = np.random.Generator(np.random.PCG64(5))
    T, H, D, bs = 20, 2, 64, 4
    Kb = synthetic.to_bf16_bits(rng.standard_normal((T, H, D)).astype(np.float32))
    codes, scales = oracle.kv_quantize(Kb)
    q2, s2 = oracle.quant_act(Kb.reshape(T * H, D))
    assert np.array_equal(codes.reshape(T * H, D), q2) and np.array_equal(scales.ravel(), s2)
    amax = np.abs(oracle.bf16_to_float(Kb)).max(axis=2)
    assert np.array_equal(scales, (amax / np.float32(448.0)).astype(np.float32))
    nblk = 8
    cc = np.zeros((nblk, bs, H, D), np.uint8)
    cs = np.zeros((nblk, bs, H), np.float32)
    slots = rng.permutation(nblk * bs)[:T]
    oracle.kv_cache_write(cc, cs, codes, scales, slots, bs)
    for t in range(T):
        assert np.array_equal(cc[slots[t] // bs, slots[t] % bs], codes[t])
    dec = oracle.e4m3_decode_table()
    # one context token: the output is that token's dequantised V (p = 1)
    qb = synthetic.to_bf16_bits(rng.standard_normal((1, 4, D)).astype(np.float32))
    bt = np.array([[slots[0] // bs] + [0] * 7])
    cc1 = np.zeros_like(cc); cs1 = np.zeros_like(cs)
    cc1[slots[0] // bs, 0] = codes[0]; cs1[slots[0] // bs, 0] = scales[0]
    out = oracle.decode_attention_reference(qb, cc1, cs1, cc1, cs1, bt, [1], bs, 0.125)
    v = dec[codes[0]] * scales[0][:, None].astype(np.float64)
    for h in range(4):
        assert np.array_equal(out[0, h], oracle.bf16_from_double(v[h // 2]))
    # identical keys: the output is the mean of the values
    cc2 = np.zeros((2, bs, 1, D), np.uint8); cs2 = np.ones((2, bs, 1), np.float32)
    cc2[:, :, 0, :] = codes[0, 0]
    vc = np.zeros_like(cc2); vc[0, :, 0, :] = codes[:4, 0]; vc[1, :, 0, :] = codes[4:8, 0]
    out = oracle.decode_attention_reference(qb[:, :1], cc2, cs2, vc, cs2, np.array([[0, 1]]), [8], bs, 0.5)
    mean = dec[codes[:8, 0]].mean(axis=0)
    assert np.allclose(oracle.bf16_to_float(out[0, 0]), mean, rtol=2 ** -8, atol=1e-12)
    # a dominant score: q along one key's direction, scaled so its score
    # exceeds the others by far more than fp64's range of exp; p is then
    # (1, 0, ...) to the last bit and the output is that token's value
    kc = np.zeros((2, bs, 1, D), np.uint8); ks = np.ones((2, bs, 1), np.float32)
    kc[1, 2, 0, 0] = 0x7E                              # key at position 6: e_0 * 448
    vc3 = np.zeros_like(kc); vc3[:, :, 0, :] = codes[:8, 1].reshape(2, bs, D)
    q3 = np.zeros((1, 1, D), np.float32); q3[0, 0, 0] = 1.0
    out = oracle.decode_attention_reference(synthetic.to_bf16_bits(q3), kc, ks, vc3, cs2,
                                            np.array([[0, 1]]), [8], bs, 64.0)
    assert np.array_equal(out[0, 0], oracle.bf16_from_double(dec[codes[6, 1]]))


def test_decode_attention_oracle_matches_library_attention():
    """Decode attention against PyTorch's scaled_dot_product_attention in
    fp64 on the same dequantised keys and values, taken in token order (not
    through the block table) and with the query-head groups expanded by
    repeat_interleave.  Pins the paged gather, the query-head to KV-head map,
    the softmax scale and the reduction over ragged contexts: the oracle's
    bf16 output is the library's fp64 result rounded to nearest (within one
    bf16 unit where the two fp64 sums round to opposite sides of a tie)."""
    rng = np.random.Generator(np.random.PCG64(11))
    B, Hq, Hkv, D, bs = 3, 8, 2, 32, 4
    lens = [1, 9, 23]
    nblk = 24
    scale = 1.0 / np.sqrt(D)
    cc = {n: np.zeros((nblk, bs, Hkv, D), np.uint8) for n in "kv"}
    cs = {n: np.zeros((nblk, bs, Hkv), np.float32) for n in "kv"}
    perm = rng.permutation(nblk)
    tables = np.zeros((B, 8), np.int64)
    tokens = {}
    used = 0
    for b, L in enumerate(lens):
        nb = -(-L // bs)
        tables[b, :nb] = perm[used:used + nb]
        used += nb
        slots = tables[b, np.arange(L) // bs] * bs + np.arange(L) % bs
        for n in "kv":
            x = synthetic.to_bf16_bits((rng.standard_normal((L, Hkv, D)) * 2.0).astype(np.float32))
            c, s = oracle.kv_quantize(x)
            oracle.kv_cache_write(cc[n], cs[n], c, s, slots, bs)
            tokens[b, n] = (c, s)
    qb = synthetic.to_bf16_bits(rng.standard_normal((B, Hq, D)).astype(np.float32))
    out = oracle.decode_attention_reference(qb, cc["k"], cs["k"], cc["v"], cs["v"], tables, lens, bs, scale)
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double()
    q = torch.from_numpy(qb.astype(np.int32) << 16).view(torch.float32).double()
    for b, L in enumerate(lens):
        kv = []
        for n in "kv":
            c, s = tokens[b, n]
            x = dec[torch.from_numpy(c).long()] * torch.from_numpy(s).double()[:, :, None]   # [L, Hkv, D]
            kv.append(x.permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0))               # [Hq, L, D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[b][:, None, :], kv[0], kv[1], scale=scale)[:, 0, :].numpy()
        got = oracle.bf16_to_float(out[b]).astype(np.float64)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
        assert np.all(np.abs(got - ref) <= 0.5 * ulp + 1e-12 * np.abs(ref) + 1e-300), b
        assert np.mean(oracle.bf16_from_double(ref) == out[b]) > 0.99


def brute_f32(fr: Fraction):
    """fp32 round-half-to-even of a non-negative exact rational, by bracketing
    the monotone positive fp32 bit patterns; None where it rounds to inf
    (at or above the midpoint between the largest finite value, whose
    mantissa is odd, and 2^128)."""
    assert fr >= 0
    if fr >= Fraction(2 ** 128) - Fraction(2 ** 103):
        return None
    val = lambda b: Fraction(float(np.array([b], np.uint32).view(np.float32)[0]))
    lo, hi = 0, 0x7F7FFFFF
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if val(mid) <= fr:
            lo = mid
        else:
            hi = mid
    dl, dh = fr - val(lo), val(hi) - fr
    return val(lo) if dl < dh or (dl == dh and lo % 2 == 0) else val(hi)


def page_order_f32_bits(y, xs, ws) -> int:
    """bf16 bits of (y * xs) * ws, each product one fp32 rounding, in exact
    arithmetic with brute-force rounding (positive operands)."""
    p = brute_f32(Fraction(float(y)) * Fraction(float(xs)))
    if p is None:
        return 0x7F80
    v = brute_f32(p * Fraction(float(ws)))
    return 0x7F80 if v is None else brute_bf16(v)


def near_tie_triples(rng, n, acc=None):
    """Operands whose final product lies within an fp32 rounding of a bf16
    midpoint, so that the order and the precision of the two products decide
    the bf16 bits: y (or the given exact accumulators) and xs random, ws the
    fp32 quotient of a bf16 midpoint by fp32(y * xs)."""
    y = (rng.random(n) + 1.0).astype(np.float32) if acc is None else np.asarray(acc, np.float32)
    xs = (rng.random(n) * 0.01 + 1e-3).astype(np.float32)
    mid = (1.0 + (rng.integers(0, 128, n) + 0.5) / 128.0) * np.exp2(rng.integers(-4, 5, n))
    ws = (mid / (y.astype(np.float64) * xs)).astype(np.float32)
    return y, xs, ws


def test_fp32_epilogue_rounds_each_product_left_to_right():
    """The fp32 epilogues (naive step 2 and the fused one) take the page's
    order, (acc * token scale) * channel scale, each product one fp32
    round-to-nearest-even and the result rounded to bf16: checked against
    exact rational arithmetic with brute-force rounding, on operands where
    another order or fp64 products give other bits."""
    rng = np.random.default_rng(21)
    y, xs, ws = near_tie_triples(rng, 400)
    expect = np.array([page_order_f32_bits(*t) for t in zip(y, xs, ws)], np.uint16)
    # the cases discriminate: other orders and fp64 products differ on many
    other = np.array([brute_bf16(Fraction(float(a)) * Fraction(float(b)) * Fraction(float(c)))
                      for a, b, c in zip(y, xs, ws)], np.uint16)
    assert (other != expect).sum() >= 40
    got = oracle.naive_step2_apply_scales(np.diag(y), xs, ws)
    assert np.array_equal(np.diag(got), expect)
    # the fused epilogue: accumulators that are exact dot products of codes
    codes = rng.integers(0x38, 0x50, (400, 2)).astype(np.uint8)      # 1 .. 7.5, positive
    dec = oracle.e4m3_decode_table()
    acc = dec[codes[:, 0]] * dec[codes[:, 1]]
    a, xs, ws = near_tie_triples(rng, 400, acc)
    expect = np.array([page_order_f32_bits(*t) for t in zip(a, xs, ws)], np.uint16)
    for i in range(400):
        got = oracle.fused_f32(codes[i:i + 1, :1], xs[i:i + 1], codes[i:i + 1, 1:], ws[i:i + 1])
        assert got[0, 0] == expect[i], i


def test_fp32_epilogue_overflows_only_in_the_page_order():
    """A token scale near the top of the range: acc * token scale overflows
    fp32 (2^23.6 * 2^110) and stays inf after the channel scale (2^-100),
    while the exact product (about 2^33.6) is finite, and so is the fp64
    tolerance reference.  The token scale is reachable: amax = 448 * 2^110 is
    a finite bf16 value."""
    Ci = 64
    Xq = np.full((1, Ci), 0x7E, np.uint8)
    Wq_t = np.full((1, Ci), 0x7E, np.uint8)
    xs = np.array([2.0 ** 110], np.float32)
    ws = np.array([2.0 ** -100], np.float32)
    assert oracle.fused_f32(Xq, xs, Wq_t, ws)[0, 0] == 0x7F80
    y = oracle.naive_step1_f32(Xq, Wq_t)
    assert y[0, 0] == Ci * 448.0 * 448.0
    assert oracle.naive_step2_apply_scales(y, xs, ws)[0, 0] == 0x7F80
    exact = Fraction(Ci * 448 * 448) * 2 ** 10
    assert oracle.scaled_mm_reference(Xq, xs, Wq_t, ws)[0, 0] == brute_bf16(exact) != 0x7F80


def test_reference_epilogue_rounds_once():
    """The tolerance reference rounds the fp64 product straight to bf16: a
    value above a bf16 midpoint by less than half an fp32 unit rounds up
    (through fp32 first it would land on the midpoint and round to even)."""
    acc = np.array([[2.0 ** 12 + 2.0 ** 4 + 2.0 ** -18]])            # a multiple of 2^-18
    out = oracle.reference_epilogue(acc, np.array([2.0 ** -12], np.float32), np.array([1.0], np.float32))
    assert out[0, 0] == 0x3F81                                          # 1 + 2^-7
    assert brute_bf16(Fraction(1) + Fraction(1, 2 ** 8) + Fraction(1, 2 ** 30)) == 0x3F81
    assert brute_bf16(brute_f32(Fraction(1) + Fraction(1, 2 ** 8) + Fraction(1, 2 ** 30))) == 0x3F80


def test_decode_attention_oracle_edge_cases():
    """The positions the library leaves out: a context of 0 positions gives 0;
    positions whose block-table entry is negative, past the cache or past the
    table's width are left out, and the rest equals PyTorch's fp64 attention
    over only the positions kept (taken in token order, not through the
    table)."""
    rng = np.random.Generator(np.random.PCG64(13))
    Hq, Hkv, D, bs, nblk = 4, 2, 32, 4, 6
    scale = 0.25
    codes = {n: rng.integers(0, 0x7E, (nblk, bs, Hkv, D)).astype(np.uint8) for n in "kv"}
    scales = {n: (rng.random((nblk, bs, Hkv)) + 0.5).astype(np.float32) for n in "kv"}
    qb = synthetic.to_bf16_bits(rng.standard_normal((3, Hq, D)).astype(np.float32))
    # seq 0: no position; seq 1: blocks 2, -1 (hole), 9 (past the cache), 4; seq 2: blocks 5,
    # 1, -1, 3 and a context of 19, three positions past the table's 16 (left out)
    tables = np.array([[0, 0, 0, 0], [2, -1, 9, 4], [5, 1, -1, 3]])
    lens = [0, 15, 19]                              # seq 2: positions 16-18 lie past the table
    out = oracle.decode_attention_reference(qb, codes["k"], scales["k"], codes["v"], scales["v"],
                                            tables, lens, bs, scale)
    assert not out[0].any()
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double()
    q = torch.from_numpy(qb.astype(np.int32) << 16).view(torch.float32).double()
    kept = {1: [(2, o) for o in range(4)] + [(4, o) for o in range(3)],      # positions 0-3 and 12-14
            2: [(5, o) for o in range(4)] + [(1, o) for o in range(4)] + [(3, o) for o in range(4)]}
    for b, slots in kept.items():
        kv = []
        for n in "kv":
            x = torch.stack([dec[torch.from_numpy(codes[n][blk, o]).long()] *
                             torch.from_numpy(scales[n][blk, o]).double()[:, None] for blk, o in slots])
            kv.append(x.permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0))
        ref = torch.nn.functional.scaled_dot_product_attention(q[b][:, None, :], kv[0], kv[1], scale=scale)[:, 0, :]
        got = oracle.bf16_to_float(out[b]).astype(np.float64)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref.numpy()), 1e-30))) - 7)
        assert np.all(np.abs(got - ref.numpy()) <= 0.5 * ulp + 1e-12 * np.abs(ref.numpy())), b
