"""Two fused linear layers issued from one host thread on two CUDA streams,
with the binding's default workspaces: each stream gets its own workspace, so
the quantised activations one call keeps there are never overwritten by the
other call running at the same time.  Both results are checked against the
oracle (codes bit-exact through the quantiser, outputs within the GEMM
tolerance)."""
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


def test_linear_on_two_streams_from_one_thread(ptpc):
    w = synthetic.LLAMA8B_PREFILL
    cases = []
    for layer, T in ((0, 1024), (1, 1536)):
        L = w.layers[layer]
        X = synthetic.make_x(w, layer, T, L.Ci)
        W = synthetic.make_w(w, layer, L.Ci, 2048)
        Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W))
        cases.append((X, W, to_dev_bf16(X), Wq_t, ws))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [None, None]
    for rep in range(3):
        for i, (X, W, Xd, Wq_t, ws) in enumerate(cases):
            streams[i].wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(streams[i]):
                outs[i] = ptpc.linear(Xd, Wq_t, ws)
        torch.cuda.synchronize()
        for i, (X, W, Xd, Wq_t, ws) in enumerate(cases):
            rWq, rws = oracle.quant_weight(W)
            assert np.array_equal(Wq_t.cpu().numpy(), rWq)
            ref, _, _ = oracle.linear_reference(X, rWq, rws)
            assert_gemm_close(from_dev_bf16(outs[i]), ref, f"stream {i} rep {rep}")
    # the two streams used two different default workspaces
    keys = [k for k in ptpc._ws_cache if k[1] in (streams[0].cuda_stream, streams[1].cuda_stream)]
    assert len(keys) == 2
