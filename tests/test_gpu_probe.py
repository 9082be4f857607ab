"""The measurement-only clock probe: it records while other kernels run on
the GPU (it shares an SM with them) and reports a plausible SM clock."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


def test_clock_probe_runs_alongside_a_gemm(ptpc):
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    T, Ci, Co = 2048, 4096, 8192
    Xq = torch.randint(0, 0x7E, (T, Ci), dtype=torch.uint8, device=dev, generator=g)
    Wq = torch.randint(0, 0x7E, (Co, Ci), dtype=torch.uint8, device=dev, generator=g)
    xs = torch.full((T,), 1e-3, device=dev)
    ws = torch.full((Co,), 1e-3, device=dev)
    out = torch.empty((T, Co), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    probe = ptpc.ClockProbe(dev)
    probe.start(0.05)
    for _ in range(200):
        ptpc.scaled_mm(Xq, xs, Wq, ws, out=out)
    mhz = probe.mhz()
    n = int(probe.count.item())
    assert n >= 10, n
    assert mhz is not None and 100.0 < mhz < 3000.0, mhz
    rec = probe.records[:n].cpu()
    assert bool((rec[1:, 0] > rec[:-1, 0]).all()) and bool((rec[1:, 1] > rec[:-1, 1]).all())
