"""GPU parity of the sub-byte weight path against the oracle: FP4 (E2M1) and
FP6 (E2M3, E3M2) per-output-channel weights with per-token FP8 activations.

The weight quantiser must give the oracle's scales and packed bytes bit for
bit (over the whole bf16 domain, and on ragged shapes with zero columns);
the scaled GEMM, whose tensor cores read the packed codes directly, must be
within |gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref) of the oracle's exact fp64
reference on the decode shapes (every K split) and on prefill shapes (both
tile widths of the CTA-pair kernel)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from helpers import assert_gemm_close, from_dev_bf16, to_dev_bf16
from test_gpu_quant import _domain_chunks

pytestmark = pytest.mark.gpu

FMTS = ("e2m1", "e2m3", "e3m2")


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


def oracle_weights(W_bits, fmt):
    codes, ws = oracle.quant_weight_fmt(W_bits, fmt)
    return codes, oracle.pack_fmt(codes, fmt), ws


def assert_weight_fmt_parity(ptpc, W_bits, fmt):
    Wq, ws = ptpc.quantize_weights_fmt(to_dev_bf16(W_bits), fmt)
    _, rp, rs = oracle_weights(W_bits, fmt)
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), rs.view(np.uint32)), f"{fmt}: scales differ"
    g = Wq.cpu().numpy()
    if not np.array_equal(g, rp):
        bad = np.argwhere(g != rp)[0]
        raise AssertionError(f"{fmt}: packed codes differ at {tuple(bad)}: gpu {g[tuple(bad)]:#x} "
                             f"oracle {rp[tuple(bad)]:#x}")
    return Wq, ws


@pytest.mark.parametrize("fmt", FMTS)
def test_weight_fmt_exhaustive_bf16_domain(ptpc, fmt):
    """Every (column amax, element) pair of bf16 values, columns = amax."""
    for X in _domain_chunks():
        assert_weight_fmt_parity(ptpc, np.ascontiguousarray(X.T), fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("Ci,Co", [(128, 16), (256, 512), (384, 4112), (4096, 6144), (8192, 48)])
def test_weight_fmt_shapes(ptpc, fmt, Ci, Co):
    W = synthetic.random_bf16((Ci, Co), seed=Ci + Co + 7, scale=0.02)
    W[:, 0] = 0                      # zero column
    W[:, min(3, Co - 1)] = 0x8000    # -0 column
    W[5 % Ci, min(5, Co - 1)] = 0x8000
    assert_weight_fmt_parity(ptpc, W, fmt)


def test_weight_fmt_e4m3_is_the_ptpc_quantiser(ptpc):
    W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, 512, 384)
    a, sa = ptpc.quantize_weights_fmt(to_dev_bf16(W), "e4m3")
    b, sb = ptpc.quantize_weights(to_dev_bf16(W))
    assert torch.equal(a, b) and torch.equal(sa, sb)


def run_fmt(ptpc, X, W, fmt, rows=None, check_linear=True):
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    Wq, ws = ptpc.quantize_weights_fmt(Wd, fmt)
    Xq, xs = ptpc.quantize_activations(Xd)
    out = ptpc.scaled_mm_fmt(Xq, xs, Wq, ws, fmt)
    codes, rp, rws = oracle_weights(W, fmt)
    rXq, rxs = oracle.quant_act(X)
    assert np.array_equal(Wq.cpu().numpy(), rp) and np.array_equal(Xq.cpu().numpy(), rXq)
    ref = oracle.scaled_mm_reference_fmt(rXq, rxs, codes, rws, fmt, rows)
    g = from_dev_bf16(out)
    if check_linear:
        lin = ptpc.linear_fmt(Xd, Wq, ws, fmt)
        assert torch.equal(lin.view(torch.int16), out.view(torch.int16)), "linear_fmt != quantize + scaled_mm_fmt"
    return (g if rows is None else g[rows]), ref


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("T", [1, 8, 32, 128])
@pytest.mark.parametrize("layer", [0, 1])
def test_gemm_fmt_decode_70b(ptpc, fmt, T, layer):
    """The 70B decode layers (8192 -> 28672 whole tiles, 28672 -> 8192 with K
    split over a cluster) with sub-byte weights."""
    w = synthetic.DECODE_70B
    L = w.layers[layer]
    X = synthetic.make_x(w, layer, T, L.Ci)
    W = synthetic.make_w(w, layer, L.Ci, L.Co)
    g, r = run_fmt(ptpc, X, W, fmt)
    assert_gemm_close(g, r, f"{fmt} decode {L.name} T={T}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("T,Ci,Co", [(1, 128, 16), (7, 256, 272), (77, 384, 528), (200, 1024, 1040),
                                     (300, 640 + 128, 1040), (1000, 1024, 768), (3001, 512, 2064),
                                     (2048, 4096, 6144)])
def test_gemm_fmt_ragged(ptpc, fmt, T, Ci, Co):
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.LLAMA70B_PREFILL, 0, T, Ci), huge_bits=0x7180)
    W = synthetic.random_bf16((Ci, Co), seed=T + Ci + Co, scale=0.02)
    W[:, 1] = 0
    g, r = run_fmt(ptpc, X, W, fmt)
    assert_gemm_close(g, r, f"{fmt} T={T} {Ci}->{Co}")


@pytest.mark.parametrize("fmt", FMTS)
def test_gemm_fmt_forced_plans(ptpc, fmt, monkeypatch):
    """Every plan (both prefill tile widths, the decode kernel with and
    without a K split) with sub-byte weights."""
    names = ("PTPC_FORCE_KSPLIT", "PTPC_FORCE_PAIR_BN", "PTPC_FORCE_KERNEL")
    X = synthetic.make_x(synthetic.DECODE_70B, 0, 256, 1024)
    W = synthetic.random_bf16((1024, 2064), seed=17, scale=0.02)
    cases = [({"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_PAIR_BN": "128"}, 100),
             ({"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_PAIR_BN": "256"}, 7),
             ({"PTPC_FORCE_KERNEL": "decode"}, 256),
             ({"PTPC_FORCE_KERNEL": "decode", "PTPC_FORCE_KSPLIT": "1"}, 64),
             ({"PTPC_FORCE_KSPLIT": "2"}, 13)]
    try:
        for env, t in cases:
            for k in names:
                monkeypatch.delenv(k, raising=False)
            for k, v in env.items():
                monkeypatch.setenv(k, v)
            ptpc.reload_tuning_overrides()
            g, r = run_fmt(ptpc, X[:t].copy(), W, fmt, check_linear=False)
            assert_gemm_close(g, r, f"{fmt} forced {env} T={t}")
    finally:
        for k in names:
            monkeypatch.delenv(k, raising=False)
        ptpc.reload_tuning_overrides()


@pytest.mark.parametrize("fmt", FMTS)
def test_gemm_fmt_70b_prefill_sampled(ptpc, fmt):
    """Full 70B down-proj at T = 2048 (pair kernel, 256-wide tiles), sampled rows."""
    w = synthetic.LLAMA70B_PREFILL
    L = w.layers[1]
    X = synthetic.make_x(w, 1, 2048, L.Ci)
    W = synthetic.make_w(w, 1, L.Ci, L.Co)
    rows = np.unique(np.concatenate([[0, 2047], np.arange(127, 2048, 128), np.arange(128, 2048, 128),
                                     np.random.Generator(np.random.PCG64(1)).choice(2048, 64, replace=False)]))
    g, r = run_fmt(ptpc, X, W, fmt, rows=rows, check_linear=False)
    assert_gemm_close(g, r, f"{fmt} 70B down T=2048 sampled")
