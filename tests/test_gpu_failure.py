"""Failure detection on the GPU without a GPU fault: a kernel's bounded wait
runs out on a barrier that nothing arrives at, the timeout reaches the host
through the workspace's status word, and the context stays usable."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


def test_bounded_wait_runs_out_and_is_reported(ptpc):
    ws = ptpc.Workspace(256, "cuda")
    assert ptpc.device_status(ws) == ptpc.OK
    ptpc.selftest_wait_timeout(ws)
    assert ptpc.device_status(ws) == ptpc.ERR_DEVICE_TIMEOUT
    assert ptpc.device_status(ws) == ptpc.OK          # read and cleared
    # the context still works: a small scaled GEMM with its own status word
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    Xq = torch.randint(0, 0x7E, (32, 256), dtype=torch.uint8, device="cuda", generator=g)
    Wq = torch.randint(0, 0x7E, (512, 256), dtype=torch.uint8, device="cuda", generator=g)
    xs = torch.ones(32, device="cuda")
    w = torch.ones(512, device="cuda")
    out = ptpc.scaled_mm(Xq, xs, Wq, w, ws=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert ptpc.device_status(ws) == ptpc.OK
