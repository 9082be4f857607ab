"""Pins of the oracle's quantisers.

Fixed outside the oracle: the hand-derived worked example, an independent
restatement through numpy's fp32 division and PyTorch's float8 cast, and the
invariants the method implies (the amax element maps to +-448, negation flips
only the sign bit, power-of-two rescaling leaves codes unchanged, the error
bound of round-to-nearest, per-tensor scaling as the equal-scale special case,
and the weight quantiser being the activation quantiser of W transposed)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from golden_io import float_array, hex_array, read_sections


def restated_quant_rows(X_bits):
    """Independent restatement: numpy fp32 division and PyTorch's float8 cast."""
    x = oracle.bf16_to_float(X_bits)
    amax = np.abs(x).max(axis=1)
    s = np.where(amax == 0, np.float32(1.0), amax / np.float32(448.0)).astype(np.float32)
    q = (x / s[:, None]).astype(np.float32)
    codes = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    codes[amax == 0] = 0
    return codes, s


@pytest.fixture(scope="module")
def x_mix():
    X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, 64, 4096)
    return synthetic.with_edge_rows(X)


def test_hand_example_codes_and_scales():
    g = read_sections("hand_example.txt")
    Xq, xs = oracle.quant_act(hex_array(g["X_bf16"], np.uint16))
    assert np.array_equal(Xq, hex_array(g["Xq_u8"], np.uint8))
    assert np.array_equal(xs, float_array(g["x_scale_f32"], np.float32)[0])
    Wq_t, ws = oracle.quant_weight(hex_array(g["W_bf16"], np.uint16))
    assert np.array_equal(Wq_t, hex_array(g["Wq_t_u8"], np.uint8))
    assert np.array_equal(ws, float_array(g["w_scale_f32"], np.float32)[0])


def test_quant_act_matches_restatement(x_mix):
    Xq, xs = oracle.quant_act(x_mix)
    rq, rs = restated_quant_rows(x_mix)
    assert np.array_equal(xs, rs)
    assert np.array_equal(Xq, rq)


@pytest.mark.parametrize("w", [synthetic.TINY, synthetic.LLAMA70B_PREFILL])
def test_quant_act_matches_restatement_other_distributions(w):
    X = synthetic.make_x(w, 0, 32, 1024)
    Xq, xs = oracle.quant_act(X)
    rq, rs = restated_quant_rows(X)
    assert np.array_equal(xs, rs) and np.array_equal(Xq, rq)


def test_amax_element_maps_to_448(x_mix):
    Xq, xs = oracle.quant_act(x_mix)
    x = oracle.bf16_to_float(x_mix)
    amax = np.abs(x).max(axis=1)
    for t in range(x.shape[0]):
        if amax[t] == 0:
            assert xs[t] == 1.0 and (Xq[t] == 0).all()
            continue
        k = int(np.argmax(np.abs(x[t])))
        assert Xq[t, k] & 0x7F == 0x7E


def test_negation_flips_only_sign_bit(x_mix):
    Xq, xs = oracle.quant_act(x_mix)
    Nq, ns = oracle.quant_act(x_mix ^ np.uint16(0x8000))
    assert np.array_equal(xs, ns)
    nonzero = np.abs(oracle.bf16_to_float(x_mix)).max(axis=1) > 0
    assert np.array_equal(Nq[nonzero], Xq[nonzero] ^ 0x80)


@pytest.mark.parametrize("k", [-20, -3, 1, 5, 20])
def test_power_of_two_rescaling(k):
    X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 1, 16, 512)
    x = oracle.bf16_to_float(X)
    y = (x * np.float32(2.0 ** k)).astype(np.float32)
    Y = (y.view(np.uint32) >> 16).astype(np.uint16)        # exact: bf16 scaled by 2^k
    assert np.array_equal(oracle.bf16_to_float(Y), y)
    Xq, xs = oracle.quant_act(X)
    Yq, ys = oracle.quant_act(Y)
    assert np.array_equal(Xq, Yq)
    assert np.array_equal(ys, (xs * np.float32(2.0 ** k)).astype(np.float32))


def test_rounding_error_bound(x_mix):
    Xq, xs = oracle.quant_act(x_mix)
    dec = oracle.e4m3_decode_table()[Xq]
    x = oracle.bf16_to_float(x_mix).astype(np.float64)
    q = x / xs[:, None].astype(np.float64)                   # exact quotient (fp64 close enough)
    half_gap = np.where(np.abs(dec) >= 2.0 ** -6, np.abs(dec) * 2.0 ** -4, 2.0 ** -10)
    err = np.abs(q - dec)
    bound = half_gap * (1 + 2.0 ** -20) + np.abs(q) * 2.0 ** -23
    zero_rows = np.abs(x).max(axis=1) == 0
    assert (err[~zero_rows] <= bound[~zero_rows]).all()


def test_zero_row_rule():
    X = np.zeros((3, 64), np.uint16)
    X[1] = 0x8000
    Xq, xs = oracle.quant_act(X)
    assert (xs == 1.0).all() and (Xq == 0).all()


def test_per_tensor_is_equal_scale_special_case():
    rng = np.random.default_rng(2)
    X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, 32, 256)
    x = oracle.bf16_to_float(X)
    big = np.abs(x).max() * 2
    Xp = X.copy()
    # plant the same amax (+-big) in every row
    bits = (np.float32(big).view(np.uint32) >> 16).astype(np.uint16)
    cols = rng.integers(0, 256, 32)
    Xp[np.arange(32), cols] = bits | (rng.integers(0, 2, 32).astype(np.uint16) << 15)
    Xq, xs = oracle.quant_act(Xp)
    Pq, ps = oracle.quant_per_tensor(Xp)
    assert (xs == np.float32(ps)).all()
    assert np.array_equal(Xq, Pq)


def test_per_tensor_is_the_one_token_case():
    """Per-tensor quantisation is per-token quantisation of the whole tensor
    read as one token: same codes, and the scale is the tensor's largest
    magnitude / 448.  The largest magnitude is planted in the last element,
    then in the first, so a maximum over part of the tensor fails."""
    X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 3, 24, 256)
    for where in (-1, 0):
        Xp = X.copy().ravel()
        big = np.abs(oracle.bf16_to_float(X)).max() * 4
        Xp[where] = (np.float32(-big).view(np.uint32) >> 16).astype(np.uint16)
        Xp = Xp.reshape(X.shape)
        q, s = oracle.quant_per_tensor(Xp)
        q1, s1 = oracle.quant_act(Xp.reshape(1, -1))
        assert s == s1[0] == np.float32(np.abs(oracle.bf16_to_float(Xp)).max()) / np.float32(448.0)
        assert np.array_equal(q.ravel(), q1[0])
        Wq_t, sw = oracle.quant_weight_per_tensor(Xp)
        assert sw == s and np.array_equal(Wq_t, q.T)


def test_weight_quant_is_activation_quant_of_transpose():
    W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, 384, 96)
    Wq_t, ws = oracle.quant_weight(W)
    Aq, as_ = oracle.quant_act(np.ascontiguousarray(W.T))
    assert Wq_t.shape == (96, 384)
    assert np.array_equal(Wq_t, Aq) and np.array_equal(ws, as_)


def test_weight_per_tensor_matches_flat_per_tensor():
    W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, 128, 64)
    Wq_t, s = oracle.quant_weight_per_tensor(W)
    q, s2 = oracle.quant_per_tensor(W)
    assert s == s2 and np.array_equal(Wq_t, q.T)


def test_quantize_value_single_element():
    assert oracle.quantize_value(3.5, 3.5 / 448, 3.5) == 0x7E
    assert oracle.quantize_value(-0.0, 1.0, 1.0) == 0x80
    assert oracle.quantize_value(-0.0, 1.0, 0.0) == 0x00
    assert oracle.scale_from_amax(0.0) == 1.0
    assert oracle.scale_from_amax(448.0) == 1.0


def test_row_split_quantisation_equals_whole_rows():
    """Tensor-parallel split of the input channels: the maximum of the slices'
    row maxima is the row maximum (checked against numpy), and quantising each
    slice with it reproduces the whole-row codes and scales of quant_act."""
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.LLAMA70B_PREFILL, 0, 40, 1024))
    Xq, xs = oracle.quant_act(X)
    full_amax = np.abs(oracle.bf16_to_float(X)).max(axis=1)
    assert np.array_equal(oracle.row_amax(X), full_amax)
    for parts in (2, 4, 8):
        w = 1024 // parts
        slices = [X[:, r * w:(r + 1) * w] for r in range(parts)]
        amax = np.max(np.stack([oracle.row_amax(s) for s in slices]), axis=0)
        assert np.array_equal(amax, full_amax)
        got = [oracle.quant_act_amax(s, amax) for s in slices]
        assert np.array_equal(np.concatenate([g[0] for g in got], axis=1), Xq)
        for g in got:
            assert np.array_equal(g[1].view(np.uint32), xs.view(np.uint32))
