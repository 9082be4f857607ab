"""GPU parity of the quantisers against the oracle: codes and scales must be
bit-identical (per-token activations, per-channel weights, per-tensor)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from helpers import from_dev_bf16, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


def gpu_quant_act(ptpc, X_bits):
    Xq, xs = ptpc.quantize_activations(to_dev_bf16(X_bits))
    return Xq.cpu().numpy(), xs.cpu().numpy()


def assert_act_parity(ptpc, X_bits):
    gq, gs = gpu_quant_act(ptpc, X_bits)
    rq, rs = oracle.quant_act(X_bits)
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32)), "scales differ"
    if not np.array_equal(gq, rq):
        bad = np.argwhere(gq != rq)[0]
        raise AssertionError(f"codes differ at {tuple(bad)}: gpu {gq[tuple(bad)]:#x} oracle {rq[tuple(bad)]:#x}")


def assert_weight_parity(ptpc, W_bits):
    Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W_bits))
    rq, rs = oracle.quant_weight(W_bits)
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), rs.view(np.uint32)), "scales differ"
    assert np.array_equal(Wq_t.cpu().numpy(), rq), "codes differ"


def test_tiny_workload(ptpc):
    w = synthetic.TINY
    assert_act_parity(ptpc, synthetic.make_x(w, 0, 16, 256))
    assert_weight_parity(ptpc, synthetic.make_w(w, 0, 256, 512))


# every (T, Ci) pair up to 30 M elements (the two larger ones, T = 3001 with
# 14336 or 28672 columns, are within the full-size cases' range)
RAGGED_ACT = [(T, Ci) for T in (1, 2, 7, 77, 1000, 3001) for Ci in (16, 256, 4096, 4112, 8192, 14336, 28672)
              if T * Ci <= 30_000_000]


@pytest.mark.parametrize("T,Ci", RAGGED_ACT)
def test_act_ragged_shapes(ptpc, T, Ci):
    X = synthetic.make_x(synthetic.LLAMA70B_PREFILL, 0, T, Ci)
    assert_act_parity(ptpc, synthetic.with_edge_rows(X))


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_act_llama8b_prefill_full(ptpc, layer):
    w = synthetic.LLAMA8B_PREFILL
    L = w.layers[layer]
    assert_act_parity(ptpc, synthetic.make_x(w, layer, 2048, L.Ci))


def test_act_llama70b_prefill_full(ptpc):
    w = synthetic.LLAMA70B_PREFILL
    assert_act_parity(ptpc, synthetic.make_x(w, 1, 8192, 28672))


def test_signed_zero_in_nonzero_groups(ptpc):
    """-0.0 keeps its sign (code 0x80) in rows/columns with a normal scale."""
    X = synthetic.random_bf16((64, 512), seed=5)
    X[:, ::7] = 0x8000
    X[:, 3::7] = 0x0000
    assert_act_parity(ptpc, X)
    assert_weight_parity(ptpc, X)


def test_act_long_rows_two_pass_kernel(ptpc):
    # rows longer than the register-resident kernel holds (Ci > 131072)
    X = synthetic.random_bf16((3, 131072 + 4096), seed=21, scale=3.0)
    assert_act_parity(ptpc, synthetic.with_edge_rows(X))


def _domain_chunks(rows_per_chunk=2048):
    """Rows of every positive finite bf16 amax (0x0001..0x7F7F); row r holds
    every bf16 x with |x| <= amax_r (the others replaced by +-amax_r).  The
    last chunk is padded with its last amax to a multiple of 16 rows."""
    amax = np.arange(1, 0x7F80, dtype=np.uint32).astype(np.uint16)
    allb = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    mag = allb & np.uint16(0x7FFF)
    sign = allb & np.uint16(0x8000)
    for i in range(0, amax.size, rows_per_chunk):
        chunk = amax[i:i + rows_per_chunk]
        pad = (-chunk.size) % 16
        if pad:
            chunk = np.concatenate([chunk, np.full(pad, chunk[-1], np.uint16)])
        keep = mag[None, :] <= chunk[:, None]
        yield np.where(keep, allb[None, :], sign[None, :] | chunk[:, None]).astype(np.uint16)


def test_act_exhaustive_bf16_domain(ptpc):
    """Every (row amax, element) pair of bf16 values: 32640 rows x 65536."""
    for X in _domain_chunks():
        assert_act_parity(ptpc, X)


def test_weight_exhaustive_bf16_domain(ptpc):
    """Same domain through the weight quantiser (columns = amax values)."""
    for X in _domain_chunks():
        assert_weight_parity(ptpc, np.ascontiguousarray(X.T))


@pytest.mark.parametrize("Ci,Co", [(16, 16), (256, 512), (384, 4112), (4096, 6144), (4112, 48)])
def test_weight_shapes(ptpc, Ci, Co):
    W = synthetic.random_bf16((Ci, Co), seed=Ci + Co, scale=0.02)
    W[:, 0] = 0                      # zero column
    W[:, min(3, Co - 1)] = 0x8000    # -0 column
    assert_weight_parity(ptpc, W)


def test_weight_llama8b_full(ptpc):
    w = synthetic.LLAMA8B_PREFILL
    for layer, L in enumerate(w.layers):
        assert_weight_parity(ptpc, synthetic.make_w(w, layer, L.Ci, L.Co))


def test_per_tensor(ptpc):
    X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, 77, 4096)
    Xq, xs = ptpc.quantize_activations_per_tensor(to_dev_bf16(X))
    rq, rs = oracle.quant_per_tensor(X)
    assert np.array_equal(Xq.cpu().numpy(), rq)
    assert (xs.cpu().numpy() == np.float32(rs)).all()
    W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, 512, 384)
    Wq_t, ws = ptpc.quantize_weights_per_tensor(to_dev_bf16(W))
    wq, wsc = oracle.quant_weight_per_tensor(W)
    assert np.array_equal(Wq_t.cpu().numpy(), wq)
    assert (ws.cpu().numpy() == np.float32(wsc)).all()


def test_per_tensor_weights_long_columns(ptpc):
    """Per-tensor weight scale on long columns (Ci = 28672, the 70B down-proj
    input width) and a narrow output (Co = 64)."""
    W = synthetic.make_w(synthetic.DECODE_70B, 1, 28672, 64)
    Wq_t, ws = ptpc.quantize_weights_per_tensor(to_dev_bf16(W))
    wq, wsc = oracle.quant_weight_per_tensor(W)
    assert np.array_equal(Wq_t.cpu().numpy(), wq)
    assert (ws.cpu().numpy() == np.float32(wsc)).all()


def test_codes_do_not_depend_on_stream_or_repeat(ptpc):
    X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 1, 333, 4096)
    Xd = to_dev_bf16(X)
    a = ptpc.quantize_activations(Xd)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = ptpc.quantize_activations(Xd)
    s.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("T,Ci,extra", [(7, 4096, 64), (300, 8192, 2048), (1000, 256, 8), (2048, 28672, 28672)])
def test_act_row_pitch(ptpc, T, Ci, extra):
    """X given as a column slice of a wider tensor (row pitch ldx = Ci + extra)."""
    full = synthetic.make_x(synthetic.LLAMA70B_PREFILL, 1, T, Ci + extra)
    view = to_dev_bf16(full)[:, :Ci]
    assert view.stride(0) == Ci + extra
    gq, gs = ptpc.quantize_activations(view)
    rq, rs = oracle.quant_act(np.ascontiguousarray(full[:, :Ci]))
    assert np.array_equal(gs.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(gq.cpu().numpy(), rq)
    pq, ps = ptpc.quantize_activations_per_tensor(view)
    oq, osc = oracle.quant_per_tensor(np.ascontiguousarray(full[:, :Ci]))
    assert np.array_equal(pq.cpu().numpy(), oq) and (ps.cpu().numpy() == np.float32(osc)).all()
