"""Pins of the oracle's sub-byte weight formats (FP4 E2M1, FP6 E2M3 / E3M2),
their per-output-channel quantiser, the packing of codes into memory and the
exact GEMM reference with such weights, against values fixed independently
of the oracle's code: the OCP Microscaling (MX) v1.0 element-format
definitions (value tables and extremes), PyTorch's float8_e4m3fn cast (every
sub-byte value lies on the E4M3 grid), the oracle's already pinned E4M3
codec and PTPC quantiser (the generic code with E4M3 parameters must equal
them), brute-force nearest-value search, Python integer bit strings and exact
integer dot products.  Runs without a GPU."""
import numpy as np
import pytest
import torch

import oracle
import synthetic

SUB = ("e2m1", "e2m3", "e3m2")
BITS = {"e2m1": 4, "e2m3": 6, "e3m2": 6}
MBITS = {"e2m1": 1, "e2m3": 3, "e3m2": 2}


def test_e2m1_values_match_the_ocp_table():
    # OCP MX v1.0, FP4 E2M1: the eight magnitudes
    t = oracle.fmt_decode_table("e2m1")
    assert t[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert (t[8:] == -t[:8]).all() and np.signbit(t[8])


@pytest.mark.parametrize("fmt,mx,min_normal,min_sub,nvals", [
    ("e2m1", 6.0, 1.0, 0.5, 8), ("e2m3", 7.5, 1.0, 0.125, 32), ("e3m2", 28.0, 0.25, 0.0625, 32)])
def test_extremes_match_the_ocp_definitions(fmt, mx, min_normal, min_sub, nvals):
    t = oracle.fmt_decode_table(fmt)
    pos = t[: len(t) // 2]
    assert len(pos) == nvals and oracle.fmt_max(fmt) == mx
    assert pos.max() == mx and pos[1] == min_sub
    assert pos[1 << MBITS[fmt]] == min_normal          # first code with exponent field 1
    assert (np.diff(pos) > 0).all()                    # codes ordered by value
    assert not np.isnan(t).any()                       # no NaN and no infinity codes
    assert (t[len(t) // 2:] == -pos).all()


@pytest.mark.parametrize("fmt", SUB)
def test_every_value_lies_on_the_e4m3_grid(fmt):
    """Each sub-byte value is exactly an E4M3 value: PyTorch's float8 cast and
    the oracle's pinned E4M3 codec both reproduce it."""
    t = oracle.fmt_decode_table(fmt)
    via_torch = torch.from_numpy(t).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(via_torch, t)
    codes = oracle.e4m3_encode(t.astype(np.float32))
    assert np.array_equal(np.array([oracle.e4m3_decode(c) for c in codes]), t)


@pytest.mark.parametrize("fmt", SUB)
def test_encode_roundtrip(fmt):
    n = 1 << BITS[fmt]
    t = oracle.fmt_decode_table(fmt)
    assert np.array_equal(oracle.fmt_encode(t.astype(np.float32), fmt), np.arange(n, dtype=np.uint8))


def test_generic_encoder_with_e4m3_parameters_equals_the_pinned_e4m3_encoder():
    rng = np.random.Generator(np.random.PCG64(11))
    v = np.concatenate([
        (rng.standard_normal(2_000_000) * np.exp(rng.uniform(-14, 7, 2_000_000))).astype(np.float32),
        np.float32([0.0, -0.0, 448.0, 449.0, 464.0, 480.0, -1e30, 2.0 ** -10, 2.0 ** -9 * 1.5])])
    t = oracle.e4m3_decode_table()[:127]
    mids = ((t[1:] + t[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, -mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    assert np.array_equal(oracle.fmt_encode(v, "e4m3"), oracle.e4m3_encode(v))


def brute_force_codes(v, fmt):
    """Nearest value by exhaustive search, ties to the even code, saturation at
    the format's maximum, sign kept."""
    t = oracle.fmt_decode_table(fmt)
    half = len(t) // 2
    pos = t[:half]
    out = np.empty(len(v), dtype=np.uint8)
    for i, x in enumerate(np.asarray(v, dtype=np.float64)):
        a = min(abs(x), pos[-1])
        d = np.abs(pos - a)
        cand = np.flatnonzero(d == d.min())
        c = cand[0] if len(cand) == 1 else [k for k in cand if k % 2 == 0][0]
        out[i] = c | (half if np.signbit(x) else 0)
    return out


@pytest.mark.parametrize("fmt", SUB)
def test_encode_against_brute_force(fmt):
    t = oracle.fmt_decode_table(fmt)
    pos = t[: len(t) // 2]
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.Generator(np.random.PCG64(3))
    v = np.concatenate([
        rng.uniform(-2 * pos[-1], 2 * pos[-1], 4000),
        rng.standard_normal(2000) * pos[1],
        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), pos, -pos, [0.0, -0.0, 1e30, -1e30],
        [pos[1] / 2, pos[1] / 4, -pos[1] / 2]]).astype(np.float32)
    assert np.array_equal(oracle.fmt_encode(v, fmt), brute_force_codes(v, fmt))


def test_generic_quantiser_with_e4m3_equals_the_ptpc_weight_quantiser():
    W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, 256, 96)
    W = synthetic.with_edge_rows(W.T.copy()).T.copy()         # edge columns
    codes, ws = oracle.quant_weight_fmt(W, "e4m3")
    rq, rws = oracle.quant_weight(W)
    assert np.array_equal(codes, rq) and np.array_equal(ws.view(np.uint32), rws.view(np.uint32))


@pytest.mark.parametrize("fmt", SUB)
def test_quantiser_invariants(fmt):
    Ci, Co = 384, 80
    W = synthetic.random_bf16((Ci, Co), seed=21, scale=0.02)
    W[:, 3] = 0x0000                      # all +0 column
    W[:, 4] = 0x8000                      # all -0 column
    codes, ws = oracle.quant_weight_fmt(W, fmt)
    half = 1 << (BITS[fmt] - 1)
    maxcode = half - 1
    wf = oracle.bf16_to_float(W).astype(np.float64)
    # zero columns: scale 1, every code +0
    assert ws[3] == 1.0 and ws[4] == 1.0 and not codes[3].any() and not codes[4].any()
    live = [o for o in range(Co) if o not in (3, 4)]
    for o in live:
        amax = np.abs(wf[:, o]).max()
        assert ws[o] == np.float32(np.float32(amax) / np.float32(oracle.fmt_max(fmt)))
        k = int(np.abs(wf[:, o]).argmax())
        assert (codes[o, k] & (half - 1)) == maxcode          # the amax element gets the largest code
    # negation flips only the sign bit; 2^k scaling leaves codes, scales x 2^k
    cneg, wsn = oracle.quant_weight_fmt(W ^ np.uint16(0x8000), fmt)
    assert np.array_equal(cneg[live] ^ np.uint8(half), codes[live]) and np.array_equal(wsn, ws)
    W4 = synthetic.to_bf16_bits(wf.astype(np.float32) * np.float32(4.0))
    c4, ws4 = oracle.quant_weight_fmt(W4, fmt)
    assert np.array_equal(c4, codes) and np.array_equal(ws4[live], ws[live] * 4)
    # error bound: |w - dec(code) * s| <= half a grid step at dec's magnitude, times s
    dec = oracle.fmt_decode_table(fmt)[codes].T * ws
    t = oracle.fmt_decode_table(fmt)[:half]
    step = np.max(np.diff(t))
    assert (np.abs(wf - dec) <= 0.5 * step * ws + 1e-12).all()


@pytest.mark.parametrize("fmt", SUB)
def test_packing_against_python_bit_strings(fmt):
    rng = np.random.Generator(np.random.PCG64(9))
    codes = rng.integers(0, 1 << BITS[fmt], size=(5, 64)).astype(np.uint8)
    packed = oracle.pack_fmt(codes, fmt)
    b = BITS[fmt]
    assert packed.shape == (5, 64 * b // 8)
    for r in range(5):
        value = sum(int(c) << (b * k) for k, c in enumerate(codes[r]))
        assert bytes(packed[r]) == value.to_bytes(64 * b // 8, "little")
    if fmt == "e2m1":   # two codes a byte, the even position in the low nibble
        assert np.array_equal(packed, codes[:, 0::2] | (codes[:, 1::2] << 4))


def test_fp6_packing_hand_example():
    """Codes 0, 1, ..., 15: bit string 000000 100000 010000 110000 ... read
    little-endian; the first three bytes are 0x40, 0x20, 0x0C by hand."""
    packed = oracle.pack_fmt(np.arange(16, dtype=np.uint8)[None, :], "e3m2")[0]
    assert packed[:3].tolist() == [0x40, 0x20, 0x0C]
    assert len(packed) == 12


@pytest.mark.parametrize("fmt", SUB)
def test_gemm_exact_against_integer_dot_products(fmt):
    T, Ci, Co = 5, 256, 48
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.TINY, 0, T, Ci))
    W = synthetic.random_bf16((Ci, Co), seed=4, scale=0.03)
    Xq, xs = oracle.quant_act(X)
    codes, ws = oracle.quant_weight_fmt(W, fmt)
    acc = oracle.gemm_acc64_fmt(Xq, codes, fmt)
    ea = np.rint(oracle.e4m3_decode_table()[:127] * 512).astype(np.int64)       # units of 2^-9
    eb = np.rint(oracle.fmt_decode_table(fmt) * 16).astype(np.int64)           # units of 2^-4
    assert np.array_equal(ea / 512, oracle.e4m3_decode_table()[:127])
    assert np.array_equal(eb / 16, oracle.fmt_decode_table(fmt))
    ia = np.where(Xq & 0x80, -ea[Xq & 0x7F], ea[Xq & 0x7F])
    for t in range(T):
        for o in range(Co):
            exact = sum(int(ia[t, k]) * int(eb[codes[o, k]]) for k in range(Ci))
            assert acc[t, o] * 8192 == exact
    # the E4M3 special case of the generic GEMM is the pinned PTPC GEMM
    rq, _ = oracle.quant_weight(W)
    assert np.array_equal(oracle.gemm_acc64_fmt(Xq, rq, "e4m3"), oracle.gemm_acc64(Xq, rq))


def test_generic_reference_with_e4m3_equals_the_ptpc_reference():
    """The format-generic fused entry with E4M3 weights is the pinned PTPC
    one: the same bf16 outputs over all tokens and over a subset of rows (the
    token scales then follow the chosen rows)."""
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.TINY, 0, 12, 256))
    W = synthetic.random_bf16((256, 40), seed=6, scale=0.05)
    codes, ws = oracle.quant_weight_fmt(W, "e4m3")
    rows = [11, 0, 5, 7]
    for r in (None, rows):
        got, gq, gs = oracle.linear_reference_fmt(X, codes, ws, "e4m3", r)
        want, wq, wsc = oracle.linear_reference(X, codes, ws, r)
        assert np.array_equal(got, want) and np.array_equal(gq, wq) and np.array_equal(gs, wsc)


@pytest.mark.parametrize("fmt", SUB)
def test_reference_row_subset_equals_full_rows(fmt):
    """A subset of token rows of the sub-byte reference equals those rows of
    the full result (the token scales follow the rows)."""
    rng = np.random.default_rng(12)
    X = synthetic.make_x(synthetic.TINY, 0, 16, 256)
    Xq, xs = oracle.quant_act(X)
    xs = xs * (rng.random(16) + 0.5).astype(np.float32)         # distinct token scales
    codes, ws = oracle.quant_weight_fmt(synthetic.random_bf16((256, 24), seed=7, scale=0.05), fmt)
    rows = [15, 2, 9]
    full = oracle.scaled_mm_reference_fmt(Xq, xs, codes, ws, fmt)
    assert np.array_equal(oracle.scaled_mm_reference_fmt(Xq, xs, codes, ws, fmt, rows), full[rows])
