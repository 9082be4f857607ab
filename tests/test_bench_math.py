"""The measurement arithmetic bench.py reports (runs without a GPU): the
algorithmic FLOP and byte counts of the path's launches, the whole-job
throughput, and the workloads' shapes against the stated configurations."""
import importlib.util
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_llama8b_step_flops(bench):
    layers = bench.workload_layers(bench.WORKLOADS["llama8b_prefill"], 2048)
    assert [(n, T, Ci, Co) for _, n, T, Ci, Co in layers] == [
        ("qkv", 2048, 4096, 6144), ("gate_up", 2048, 4096, 28672), ("down", 2048, 14336, 4096)]
    # 2 * T * (4096*6144 + 4096*28672 + 14336*4096)
    assert bench.layer_flops(layers) == 2 * 2048 * (4096 * 6144 + 4096 * 28672 + 14336 * 4096)
    assert bench.layer_flops(layers) == 824633720832


def test_decode_and_70b_shapes(bench):
    dec = bench.workload_layers(bench.WORKLOADS["decode70b"], 1)
    assert [(Ci, Co) for *_, Ci, Co in dec] == [(8192, 28672), (28672, 8192)]
    pre = bench.workload_layers(bench.WORKLOADS["llama70b_prefill"], 8192)
    assert [(T, Ci, Co) for _, _, T, Ci, Co in pre] == [(8192, 8192, 57344), (8192, 28672, 8192)]
    chain = bench.WORKLOADS["chain70b"]
    assert [(L.Ci, L.Co) for L in chain.layers] == [(8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192)]
    assert sorted(chain.tokens) == sorted([1 << k for k in range(15)] + [77, 1000, 3001])


def test_algorithmic_bytes(bench):
    # decode T=1 up-proj: the weight dominates (235 MB of codes)
    b = bench.gemm_bytes(1, 8192, 28672)
    assert b == 8192 + 8192 * 28672 + 2 * 28672 + 4 * (1 + 28672)
    assert 234_900_000 < b < 235_100_000
    # quantiser: 2 B read + 1 B written per element, 4 B per row scale
    assert bench.quant_bytes(2048, 4096) == 3 * 2048 * 4096 + 4 * 2048


def test_whole_job_throughput(bench):
    # 1e12 FLOP per rank per step, 4 ranks, 10 steps in 20 ms (slowest rank) -> 2000 TFLOP/s
    assert bench.whole_job_tflops(1e12, 4, 10, 20.0) == pytest.approx(2000.0)
    assert bench.whole_job_tflops(1e12, 1, 10, 20.0) == pytest.approx(500.0)


def test_roofline_bound_by_arithmetic_intensity(bench):
    """Prefill GEMMs sit far right of the ridge point (tensor bound), decode far
    left (HBM bound): the intensity the bench compares with the ridge."""
    peaks = {"hbm_gbs": 6516.1, "bf16_tflops": 1683.5}
    ridge = 2.0 * peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)   # FLOP per byte, ~517
    pre = [(2048, 4096, 6144), (2048, 4096, 28672), (2048, 14336, 4096)]
    dec = [(1, 8192, 28672), (128, 28672, 8192)]
    intensity = lambda shapes: (sum(2.0 * T * Ci * Co for T, Ci, Co in shapes)
                                / sum(bench.gemm_bytes(T, Ci, Co) for T, Ci, Co in shapes))
    assert intensity(pre) > ridge
    assert intensity(dec) < ridge


def test_cpu_sample_rows(bench):
    """The CPU-oracle row sample: first/last rows, both rows at every 128-row
    tile boundary, then a seeded draw; all rows when the sample covers T."""
    r = bench.sample_rows(8192, 512, seed=3)
    assert len(r) == 512 and len(set(r.tolist())) == 512
    assert r[0] == 0 and r[-1] == 8191 and (np.diff(r) > 0).all()
    for b in range(128, 8192, 128):
        assert b - 1 in r and b in r
    assert np.array_equal(r, bench.sample_rows(8192, 512, seed=3))
    assert np.array_equal(bench.sample_rows(100, 512), np.arange(100))
    assert np.array_equal(bench.sample_rows(300, 0), np.arange(300))
    small = bench.sample_rows(8192, 64)
    assert len(small) == 64 and small[0] == 0 and small[-1] == 8191


def test_chain_roofline(bench):
    """The chain's roofline time is the slower of its FLOPs at the FP8 peak and
    its algorithmic bytes at HBM bandwidth: bytes decide at T = 1, FLOPs at
    T = 8192."""
    import synthetic
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1650.0}
    layers = synthetic.CHAIN_70B.layers
    w_bytes = sum(L.Ci * L.Co for L in layers)
    t1 = bench.chain_roofline_ms(1, layers, peaks)
    assert t1 == pytest.approx(sum(bench.quant_bytes(1, L.Ci) + bench.gemm_bytes(1, L.Ci, L.Co) for L in layers)
                               / 6500e9 * 1e3)
    assert t1 > w_bytes / 6500e9 * 1e3
    t8k = bench.chain_roofline_ms(8192, layers, peaks)
    assert t8k == pytest.approx(sum(2.0 * 8192 * L.Ci * L.Co for L in layers) / 3300e12 * 1e3)
