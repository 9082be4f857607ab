"""Stray-write checks: every output buffer (and the workspace) is placed
inside a larger allocation whose guard bytes before and after must come back
unchanged, over shapes that exercise every tail path (ragged rows and
columns, both prefill tile widths, the decode kernel with and without a K
split, the long-row quantiser, the naive path, decode attention on both of
its kernels)."""
import ctypes

import numpy as np
import pytest
import torch

import synthetic
from helpers import to_dev_bf16

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side; keeps 256-byte alignment
PATTERN = 0xA5


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


class Guarded:
    """nbytes of device memory between two guard regions filled with PATTERN."""

    def __init__(self, nbytes: int):
        self.nbytes = nbytes
        self.buf = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")

    def view(self, dtype, shape):
        return self.buf[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr() + GUARD)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.buf[:GUARD]
        tail = self.buf[GUARD + self.nbytes:]
        assert bool((head == PATTERN).all()), f"{what}: write before the buffer"
        assert bool((tail == PATTERN).all()), f"{what}: write past the end of the buffer"


@pytest.mark.parametrize("T,Ci", [(1, 16), (77, 4112), (1000, 256), (3, 65552)])
def test_activation_quantiser_stays_in_bounds(ptpc, T, Ci):
    X = to_dev_bf16(synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, T, Ci))
    q, s = Guarded(T * Ci), Guarded(T * 4)
    ptpc.quantize_activations(X, q.view(torch.uint8, (T, Ci)), s.view(torch.float32, (T,)))
    q.check(f"Xq {T}x{Ci}")
    s.check(f"x_scale {T}x{Ci}")


@pytest.mark.parametrize("Ci,Co", [(16, 16), (384, 4112), (4112, 48), (4096, 6144)])
def test_weight_quantiser_stays_in_bounds(ptpc, Ci, Co):
    W = to_dev_bf16(synthetic.random_bf16((Ci, Co), seed=Ci + 3 * Co, scale=0.02))
    q, s = Guarded(Co * Ci), Guarded(Co * 4)
    need = ptpc.workspace_size(ptpc.OP_QUANTIZE_WEIGHTS, 0, Ci, Co)
    ws = Guarded(need)
    ws.view(torch.uint8, (need,)).zero_()
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream().cuda_stream)
    assert ptpc.lib.ptpc_quantize_weights(P(W.data_ptr()), Ci, Co, q.ptr(), s.ptr(), ws.ptr(), need, st) == ptpc.OK
    q.check(f"Wq_t {Ci}x{Co}")
    s.check(f"w_scale {Ci}x{Co}")
    ws.check(f"weight workspace {Ci}x{Co}")


@pytest.mark.parametrize("T,Ci,Co", [
    (1, 4096, 2048), (13, 2048, 4096), (128, 1024, 8192), (200, 4112, 8192), (77, 384, 528),
    (300, 640, 1040), (512, 8192, 10240), (2048, 4096, 6144), (1000, 1024, 2064),
    (1, 1024, 28672), (64, 512, 20512),      # decode, a second partial round of tiles
])
def test_gemm_and_linear_stay_in_bounds(ptpc, T, Ci, Co):
    X = to_dev_bf16(synthetic.make_x(synthetic.DECODE_70B, 0, T, Ci))
    Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(synthetic.random_bf16((Ci, Co), seed=T + Ci, scale=0.02)))
    Xq, xs = ptpc.quantize_activations(X)
    out = Guarded(T * Co * 2)
    need = ptpc.workspace_size(ptpc.OP_LINEAR, T, Ci, Co)
    wsg = Guarded(need)
    wsg.view(torch.uint8, (need,)).zero_()
    ws_obj = ptpc.Workspace(0, "cuda")
    ws_obj.buf = wsg.view(torch.uint8, (need,))
    ptpc.scaled_mm(Xq, xs, Wq_t, ws, out=out.view(torch.bfloat16, (T, Co)), ws=ws_obj)
    out.check(f"scaled_mm out {T}x{Ci}x{Co}")
    wsg.check(f"scaled_mm workspace {T}x{Ci}x{Co}")
    ptpc.linear(X, Wq_t, ws, out=out.view(torch.bfloat16, (T, Co)), ws=ws_obj)
    out.check(f"linear out {T}x{Ci}x{Co}")
    wsg.check(f"linear workspace {T}x{Ci}x{Co}")
    assert ptpc.device_status(ws_obj) == ptpc.OK


@pytest.mark.parametrize("T,Ci,Co", [(7, 1024, 2048), (300, 512, 1040)])
def test_naive_path_stays_in_bounds(ptpc, T, Ci, Co):
    X = to_dev_bf16(synthetic.make_x(synthetic.DECODE_70B, 1, T, Ci))
    Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(synthetic.random_bf16((Ci, Co), seed=11, scale=0.02)))
    Xq, xs = ptpc.quantize_activations(X)
    y, out = Guarded(T * Co * 4), Guarded(T * Co * 2)
    ptpc.unscaled_mm_f32(Xq, Wq_t, out=y.view(torch.float32, (T, Co)))
    y.check(f"naive step 1 {T}x{Ci}x{Co}")
    ptpc.apply_scales(y.view(torch.float32, (T, Co)), xs, ws, out=out.view(torch.bfloat16, (T, Co)))
    out.check(f"naive step 2 {T}x{Ci}x{Co}")
    assert np.isfinite(out.view(torch.bfloat16, (T, Co)).float().cpu().numpy()).all()


@pytest.mark.parametrize("T,Ci,Co,env", [
    (33, 256, 1040, {"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_SWAP": "1"}),   # swapped, one ragged token tile
    (300, 2048, 28672, {"PTPC_FORCE_SPLIT_TAIL": "1"}),                        # swapped with a split tail
    (600, 512, 2064, {"PTPC_FORCE_SWAP": "1"}),
])
def test_swapped_gemm_stays_in_bounds(ptpc, monkeypatch, T, Ci, Co, env):
    for k in ("PTPC_FORCE_SWAP", "PTPC_FORCE_KERNEL", "PTPC_FORCE_SPLIT_TAIL"):
        monkeypatch.delenv(k, raising=False)
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    ptpc.reload_tuning_overrides()
    try:
        assert ptpc.gemm_swap_tokens(T, Ci, Co) > 0
        X = to_dev_bf16(synthetic.make_x(synthetic.DECODE_70B, 0, T, Ci))
        Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(synthetic.random_bf16((Ci, Co), seed=T + Co, scale=0.02)))
        Xq, xs = ptpc.quantize_activations(X)
        need = ptpc.workspace_size(ptpc.OP_LINEAR, T, Ci, Co)
        wsg = Guarded(need)
        wsg.view(torch.uint8, (need,)).zero_()
        ws_obj = ptpc.Workspace(0, "cuda")
        ws_obj.buf = wsg.view(torch.uint8, (need,))
        out = Guarded(T * Co * 2)
        ptpc.scaled_mm(Xq, xs, Wq_t, ws, out=out.view(torch.bfloat16, (T, Co)), ws=ws_obj)
        out.check(f"swapped scaled_mm out {T}x{Ci}x{Co}")
        wsg.check(f"swapped scaled_mm workspace {T}x{Ci}x{Co}")
        y = Guarded(T * Co * 4)
        ptpc.unscaled_mm_f32(Xq, Wq_t, out=y.view(torch.float32, (T, Co)))
        y.check(f"swapped fp32 GEMM out {T}x{Ci}x{Co}")
        assert ptpc.device_status(ws_obj) == ptpc.OK
    finally:
        for k in env:
            monkeypatch.delenv(k, raising=False)
        ptpc.reload_tuning_overrides()


@pytest.mark.parametrize("kernel,chunk", [("tc", "auto"), ("tc", "1024"), ("mma", "auto")])
@pytest.mark.parametrize("lens,Hq,Hkv,D,bs", [
    ([1, 300, 4096, 0, 77], 64, 8, 128, 16),     # one chunk a context: the kernel writes the output itself
    ([5000, 130], 24, 3, 128, 8),                # several chunks: partial results and the combine kernel
    ([40, 600], 32, 2, 64, 16),                  # the warp-level kernel's shape
])
def test_decode_attention_stays_in_bounds(ptpc, monkeypatch, kernel, chunk, lens, Hq, Hkv, D, bs):
    """Decode attention's output and workspace (status word, partial results)
    stay inside their buffers on both kernels, with the output written by the
    attention kernel itself (one chunk a context) and by the combine kernel."""
    monkeypatch.setenv("PTPC_FORCE_ATTN_KERNEL", kernel)
    if chunk != "auto":
        monkeypatch.setenv("PTPC_FORCE_ATTN_CHUNK", chunk)
    ptpc.reload_tuning_overrides()
    try:
        B = len(lens)
        max_blocks = max(1, max((l + bs - 1) // bs for l in lens))
        nb = B * max_blocks + 1
        rng = np.random.Generator(np.random.PCG64(sum(lens) + Hq))
        tables = torch.from_numpy(rng.permutation(nb)[:B * max_blocks].astype(np.int32).reshape(B, max_blocks)).cuda()
        kc = torch.randint(0, 0x7E, (nb, bs, Hkv, D), dtype=torch.uint8, device="cuda")
        vc = torch.randint(0, 0x7E, (nb, bs, Hkv, D), dtype=torch.uint8, device="cuda")
        ksc = torch.rand((nb, bs, Hkv), device="cuda") * 0.01
        vsc = torch.rand((nb, bs, Hkv), device="cuda") * 0.01
        q = torch.randn((B, Hq, D), device="cuda").to(torch.bfloat16)
        max_ctx = max(lens)
        out = Guarded(B * Hq * D * 2)
        need = int(ptpc.lib.ptpc_decode_attention_workspace_size(B, Hq, D, max_ctx))
        ws = Guarded(need)
        ws.view(torch.uint8, (need,)).zero_()
        lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
        P = ctypes.c_void_p
        st = P(torch.cuda.current_stream().cuda_stream)
        r = ptpc.lib.ptpc_decode_attention(P(q.data_ptr()), P(kc.data_ptr()), P(vc.data_ptr()), P(ksc.data_ptr()),
                                           P(vsc.data_ptr()), P(tables.data_ptr()), P(lens_d.data_ptr()), B, Hq, Hkv,
                                           D, bs, nb, max_blocks, max_ctx, ctypes.c_float(D ** -0.5), out.ptr(),
                                           ws.ptr(), need, st)
        assert r == ptpc.OK
        out.check(f"attention out {kernel} {lens}")
        ws.check(f"attention workspace {kernel} {lens}")
        assert ptpc.lib.ptpc_get_device_status(ws.ptr(), st) == ptpc.OK
    finally:
        monkeypatch.delenv("PTPC_FORCE_ATTN_KERNEL", raising=False)
        monkeypatch.delenv("PTPC_FORCE_ATTN_CHUNK", raising=False)
        ptpc.reload_tuning_overrides()
