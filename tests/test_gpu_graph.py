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


@pytest.mark.parametrize("lens,Hq", [([500, 1, 300, 17], 64),   # one 512-position chunk: the kernel writes out
                                     ([5000, 700], 128)])        # several chunks and the combine kernel
def test_decode_attention_replays_from_a_cuda_graph(ptpc, lens, Hq):
    """A decode step's cache append and attention (one chunk a context, the
    kernel writing the output; or several chunks and the combine kernel;
    groups of 8 and of 16 query heads) captured into a CUDA graph: the replay
    gives the eager calls' bits."""
    import numpy as np
    B, Hkv, D, bs = len(lens), 8, 128, 16
    max_blocks = max((l + bs - 1) // bs for l in lens) + 1
    nb = B * max_blocks
    rng = np.random.Generator(np.random.PCG64(sum(lens)))
    tables = torch.from_numpy(rng.permutation(nb).astype(np.int32).reshape(B, max_blocks)).cuda()
    kc = torch.randint(0, 0x7E, (nb, bs, Hkv, D), dtype=torch.uint8, device="cuda")
    vc = torch.randint(0, 0x7E, (nb, bs, Hkv, D), dtype=torch.uint8, device="cuda")
    ksc = torch.rand((nb, bs, Hkv), device="cuda") * 0.01
    vsc = torch.rand((nb, bs, Hkv), device="cuda") * 0.01
    q = torch.randn((B, Hq, D), device="cuda").to(torch.bfloat16)
    Kn = torch.randn((B, Hkv, D), device="cuda").to(torch.bfloat16)
    # the new token of each sequence goes to its next position
    slots = torch.tensor([int(tables[b, lens[b] // bs]) * bs + lens[b] % bs for b in range(B)],
                         dtype=torch.int64, device="cuda")
    ctx = torch.tensor([l + 1 for l in lens], dtype=torch.int32, device="cuda")
    max_ctx = max(lens) + 1
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    wsp = ptpc.Workspace(int(ptpc.lib.ptpc_decode_attention_workspace_size(B, Hq, D, max_ctx)), "cuda")
    state = [t.clone() for t in (kc, vc, ksc, vsc)]

    def step():
        ptpc.kv_cache_append(Kn, Kn, slots, kc, vc, ksc, vsc)
        ptpc.decode_attention(q, kc, vc, ksc, vsc, tables, ctx, max_ctx, D ** -0.5, out=out, ws=wsp)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside capture (one-time per-device set-up)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager = out.clone()
    for t, t0 in zip((kc, vc, ksc, vsc), state):
        t.copy_(t0)
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    assert ptpc.device_status(wsp) == 0
