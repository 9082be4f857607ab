"""ptpc_scaled_mm_static_scratch: the scaled GEMM for callers that cannot
allocate device memory when they call it (an engine whose device memory is
partitioned once at start-up, or an integration that only passes its input
and output buffers).  Its scratch is the library's own static device array,
so the caller passes no workspace.

Checked through the C ABI against ptpc_scaled_mm (which takes a caller
workspace) on two calls in a row, on decode shapes (K split over a cluster
and whole tiles) and a prefill shape: the two entry points run the same plan,
so the outputs agree within the GEMM tolerance and, in fact, bit for bit.
The calls allocate nothing (PyTorch's and the driver's free-memory counters
do not move across them), one of them runs on a side stream, the status
reader reports no timeout after each, and one case is compared with the
oracle directly.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthetic
from helpers import assert_gemm_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


def _abi_call(ptpc, Xq, xs, Wq_t, ws, out, stream=None):
    T, Ci = Xq.shape
    Co = Wq_t.shape[0]
    P = ctypes.c_void_p
    st = (stream or torch.cuda.current_stream()).cuda_stream
    return ptpc.lib.ptpc_scaled_mm_static_scratch(
        P(Xq.data_ptr()), P(xs.data_ptr()), P(Wq_t.data_ptr()), P(ws.data_ptr()), T, Ci, Co, P(out.data_ptr()),
        P(st))


def _status(ptpc, stream=None):
    st = (stream or torch.cuda.current_stream()).cuda_stream
    return ptpc.lib.ptpc_static_scratch_status(ctypes.c_void_p(st))


@pytest.mark.parametrize("T,layer", [(8, 1), (32, 1), (128, 1), (1, 0), (128, 0), (300, 0)])
def test_static_scratch_matches_workspace_entry_point(ptpc, T, layer):
    w = synthetic.DECODE_70B
    L = w.layers[layer]
    Ci, Co = L.Ci, L.Co
    if T > 128:  # a prefill-sized case; keep the weight small
        Co = 4096
    X = synthetic.make_x(w, layer, T, Ci)
    W = synthetic.make_w(w, layer, Ci, Co)
    Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W))
    Xq, xs = ptpc.quantize_activations(to_dev_bf16(X))
    ref = ptpc.scaled_mm(Xq, xs, Wq_t, ws)
    ref_bits = from_dev_bf16(ref)
    side = torch.cuda.Stream()
    outs = [torch.full((T, Co), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    # one call first: the library looks up the array's address and the
    # driver loads the kernels' module on first use
    assert _abi_call(ptpc, Xq, xs, Wq_t, ws, outs[2]) == ptpc.OK
    assert _status(ptpc) == ptpc.OK
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for i in range(2):
        stream = side if i == 1 else None
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream())
        assert _abi_call(ptpc, Xq, xs, Wq_t, ws, outs[i], stream) == ptpc.OK
        assert _status(ptpc, stream) == ptpc.OK
        torch.cuda.synchronize()
        got = from_dev_bf16(outs[i])
        assert_gemm_close(got, ref_bits, f"static scratch T={T} {Ci}->{Co} call {i}")
        assert np.array_equal(got, ref_bits)
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0
    if T == 300:  # one case straight against the oracle's fp64 reference
        rXq, rxs = oracle.quant_act(X)
        rWq, rws = oracle.quant_weight(W)
        assert_gemm_close(from_dev_bf16(outs[1]), oracle.scaled_mm_reference(rXq, rxs, rWq, rws),
                          "static scratch vs oracle")
