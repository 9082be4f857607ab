"""The C-ABI calls only enqueue work on the caller's stream (no host
synchronisation, no allocation), so a whole PTPC-FP8 layer chain can be
captured into a CUDA graph and replayed; the replay must give the same bits
as the eager calls."""
import pytest
import torch

import synthetic
from helpers import to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


@pytest.mark.parametrize("T", [1, 77, 2048])
def test_linear_chain_replays_from_a_cuda_graph(ptpc, T):
    w = synthetic.LLAMA8B_PREFILL
    layers = []
    for i, L in enumerate(w.layers):
        Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(synthetic.make_w(w, i, L.Ci, L.Co)))
        X = to_dev_bf16(synthetic.make_x(w, i, T, L.Ci))
        out = torch.empty((T, L.Co), dtype=torch.bfloat16, device="cuda")
        wsp = ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, L.Ci, L.Co), "cuda")
        layers.append((X, Wq_t, ws, out, wsp))

    def step():
        for X, Wq_t, ws, out, wsp in layers:
            ptpc.linear(X, Wq_t, ws, out=out, ws=wsp)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside capture (one-time per-device set-up)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager = [out.clone() for _, _, _, out, _ in layers]
    for _, _, _, out, _ in layers:
        out.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for e, (_, _, _, out, wsp) in zip(eager, layers):
        assert torch.equal(e.view(torch.int16), out.view(torch.int16))
        assert ptpc.device_status(wsp) == ptpc.OK
