"""GPU parity of the scaled GEMM, the fused entry and the comparison paths.

Outputs are compared with the oracle's fp64-accumulated reference rounded to
bf16, element by element, within |gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref).
The GPU quantises its own inputs; the test also checks those codes are the
oracle's, so both sides work from the same operands."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from helpers import assert_gemm_close, from_dev_bf16, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

# bf16 bits of 2^100: a row of this magnitude has x_scale ~ 2^91, and every
# accumulator times x_scale stays far inside the fp32 range.
BIG_BF16 = 0x7180


@pytest.fixture(scope="module")
def ptpc():
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


def run_pair(ptpc, X, W, rows=None, check_linear=True):
    """GPU: quantize_weights, quantize_activations, scaled_mm (and linear).
    Oracle: the same three steps.  Returns (gpu_out, ref_out) bf16 bits."""
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    Wq_t, ws = ptpc.quantize_weights(Wd)
    Xq, xs = ptpc.quantize_activations(Xd)
    out = ptpc.scaled_mm(Xq, xs, Wq_t, ws)
    rWq, rws = oracle.quant_weight(W)
    rXq, rxs = oracle.quant_act(X)
    assert np.array_equal(Wq_t.cpu().numpy(), rWq) and np.array_equal(Xq.cpu().numpy(), rXq)
    ref = oracle.scaled_mm_reference(rXq, rxs, rWq, rws, rows)
    g = from_dev_bf16(out)
    if check_linear:
        lin = ptpc.linear(Xd, Wq_t, ws)
        assert torch.equal(lin.view(torch.int16), out.view(torch.int16)), "linear != quantize + scaled_mm"
    return (g if rows is None else g[rows]), ref


def test_tiny_workload(ptpc):
    w = synthetic.TINY
    g, r = run_pair(ptpc, synthetic.make_x(w, 0, 16, 256), synthetic.make_w(w, 0, 256, 512))
    assert_gemm_close(g, r, "tiny")


@pytest.mark.parametrize("T,Ci,Co", [
    (1, 16, 16), (2, 32, 48), (7, 128, 256), (77, 384, 528), (129, 256, 272), (300, 640, 1040),
    (1000, 1024, 768), (3001, 512, 2064), (128, 4112, 256), (257, 128, 4096),
])
def test_ragged_shapes(ptpc, T, Ci, Co):
    # the large-magnitude edge row stays where acc * x_scale fits in fp32
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.LLAMA70B_PREFILL, 0, T, Ci), huge_bits=BIG_BF16)
    W = synthetic.random_bf16((Ci, Co), seed=T + Ci + Co, scale=0.02)
    g, r = run_pair(ptpc, X, W)
    assert_gemm_close(g, r, f"{T}x{Ci}x{Co}")


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_llama8b_prefill_full(ptpc, layer):
    w = synthetic.LLAMA8B_PREFILL
    L = w.layers[layer]
    g, r = run_pair(ptpc, synthetic.make_x(w, layer, 2048, L.Ci), synthetic.make_w(w, layer, L.Ci, L.Co))
    assert_gemm_close(g, r, L.name)


@pytest.mark.parametrize("T", [1, 8, 32, 128, 192])
@pytest.mark.parametrize("layer", [0, 1])
def test_decode_full(ptpc, T, layer):
    w = synthetic.DECODE_70B
    L = w.layers[layer]
    g, r = run_pair(ptpc, synthetic.make_x(w, layer, T, L.Ci), synthetic.make_w(w, layer, L.Ci, L.Co))
    assert_gemm_close(g, r, f"decode {L.name} T={T}")


# Decode shapes whose tile counts (Co / 128) select each K split on a 148-SM
# B200: 16 tiles -> 8 CTAs per tile (or 4, when fewer than 16 clusters of 8
# fit at once), 32 -> 4, 64 -> 2, 80 -> whole tiles; 8 tiles -> 8.  Ci 4112
# leaves a partial last K-block and uneven shares; Co 2064 a partial last
# tile.
@pytest.mark.parametrize("Ci,Co,splits", [
    (4096, 1024, (8,)), (4096, 2048, (4, 8)), (4112, 2064, (4, 8)), (2048, 4096, (4,)), (1024, 8192, (2,)),
    (4112, 8192, (2,)), (1024, 10240, (1,)),
])
@pytest.mark.parametrize("T", [1, 13, 77, 128, 160, 192, 256])
def test_decode_cluster_split(ptpc, monkeypatch, T, Ci, Co, splits):
    # above T = 192 the plan takes the pair kernel: the decode kernel's largest
    # token count (256) is reached through the override
    if T > 192:
        monkeypatch.setenv("PTPC_FORCE_KERNEL", "decode")
    ptpc.reload_tuning_overrides()
    try:
        got_split = ptpc.gemm_ksplit(T, Ci, Co)
        assert got_split in splits, f"{T}x{Ci}x{Co}: K split {got_split}, expected one of {splits}"
        X = synthetic.with_edge_rows(synthetic.make_x(synthetic.DECODE_70B, 0, T, Ci), huge_bits=BIG_BF16)
        W = synthetic.random_bf16((Ci, Co), seed=T * 7 + Ci + Co, scale=0.02)
        g, r = run_pair(ptpc, X, W)
        assert_gemm_close(g, r, f"decode {T}x{Ci}x{Co} split {got_split}")
    finally:
        monkeypatch.delenv("PTPC_FORCE_KERNEL", raising=False)
        ptpc.reload_tuning_overrides()


@pytest.mark.parametrize("T,Ci,Co,fmt", [(1, 1024, 28672, "e4m3"), (77, 512, 20512, "e4m3"),
                                         (1, 1024, 28672, "e2m1"), (32, 1024, 20480, "e3m2")])
def test_decode_two_rounds_of_tiles(ptpc, T, Ci, Co, fmt):
    """Decode shapes with more 128-channel tiles than SMs (a second, partial
    round of tiles): parity on every channel, including the last, partial
    tile, for FP8 and sub-byte weights."""
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.DECODE_70B, 0, T, Ci), huge_bits=BIG_BF16)
    W = synthetic.random_bf16((Ci, Co), seed=T + Co, scale=0.02)
    Wq, ws = ptpc.quantize_weights_fmt(to_dev_bf16(W), fmt)
    Xq, xs = ptpc.quantize_activations(to_dev_bf16(X))
    out = from_dev_bf16(ptpc.scaled_mm_fmt(Xq, xs, Wq, ws, fmt))
    rXq, rxs = oracle.quant_act(X)
    if fmt == "e4m3":
        ref = oracle.scaled_mm_reference(rXq, rxs, *oracle.quant_weight(W))
    else:
        codes, rws = oracle.quant_weight_fmt(W, fmt)
        ref = oracle.scaled_mm_reference_fmt(rXq, rxs, codes, rws, fmt)
    assert_gemm_close(out, ref, f"decode, two rounds of tiles {fmt} {T}x{Ci}x{Co}")


def test_decode_split_matches_naive_step1(ptpc):
    """The K-split path's fp32 output (naive step 1) is what the fused path
    scales: applying the scales to it gives the fused output bit for bit."""
    T, Ci, Co = 32, 2048, 4096
    assert ptpc.gemm_ksplit(T, Ci, Co) > 1
    X = synthetic.make_x(synthetic.DECODE_70B, 1, T, Ci)
    W = synthetic.random_bf16((Ci, Co), seed=5, scale=0.02)
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    Wq_t, ws = ptpc.quantize_weights(Wd)
    Xq, xs = ptpc.quantize_activations(Xd)
    y = ptpc.unscaled_mm_f32(Xq, Wq_t)
    naive = ptpc.apply_scales(y, xs, ws)
    fused = ptpc.scaled_mm(Xq, xs, Wq_t, ws)
    assert torch.equal(naive.view(torch.int16), fused.view(torch.int16))


def sample_rows(T, n=256, seed=0):
    """About n output rows spread over all of T: the first and last rows, both
    sides of evenly spaced 128-row tile boundaries (up to n / 4 boundaries),
    and random rows for the rest."""
    rng = np.random.default_rng(seed)
    rows = {0, T - 1}
    bounds = np.arange(128, T, 128)
    if bounds.size:
        pick = bounds[np.unique(np.linspace(0, bounds.size - 1, min(bounds.size, max(1, n // 4))).astype(np.int64))]
        for b in pick.tolist():
            rows |= {b - 1, b}
    extra = max(0, n - len(rows))
    rows |= set(rng.choice(T, size=min(T, extra), replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("layer", [0, 1])
def test_llama70b_prefill_sampled(ptpc, layer):
    w = synthetic.LLAMA70B_PREFILL
    L = w.layers[layer]
    rows = sample_rows(8192, 192, seed=layer)
    g, r = run_pair(ptpc, synthetic.make_x(w, layer, 8192, L.Ci), synthetic.make_w(w, layer, L.Ci, L.Co),
                    rows=rows, check_linear=False)
    assert_gemm_close(g, r, f"70B {L.name}")


@pytest.mark.parametrize("T", [77, 1000, 3001])
def test_chain_ragged_sampled(ptpc, T):
    w = synthetic.CHAIN_70B
    L = w.layers[0]
    rows = sample_rows(T, 128, seed=T)
    g, r = run_pair(ptpc, synthetic.make_x(w, 0, T, L.Ci), synthetic.make_w(w, 0, L.Ci, L.Co), rows=rows)
    assert_gemm_close(g, r, f"chain qkv T={T}")


@pytest.mark.parametrize("layer", [2, 3])
def test_chain_largest_T_sampled(ptpc, layer):
    """The chain's largest size (T = 16384) on its two largest layers, gate+up
    8192 -> 57344 and down 28672 -> 8192: codes bit-exact everywhere, outputs
    checked on sampled rows (both sides of every 128-row boundary included)."""
    w = synthetic.CHAIN_70B
    L = w.layers[layer]
    T = 16384
    rows = sample_rows(T, 128, seed=layer)
    g, r = run_pair(ptpc, synthetic.make_x(w, layer, T, L.Ci), synthetic.make_w(w, layer, L.Ci, L.Co), rows=rows,
                    check_linear=False)
    assert_gemm_close(g, r, f"chain {L.name} T={T}")


def test_tuning_overrides(ptpc, monkeypatch):
    """PTPC_FORCE_KSPLIT / PTPC_FORCE_PAIR_BN / PTPC_FORCE_KERNEL change the
    plan (where feasible) and every forced plan still matches the oracle.  The
    library reads them once, so every change is followed by a reload."""
    names = ("PTPC_FORCE_KSPLIT", "PTPC_FORCE_PAIR_BN", "PTPC_FORCE_KERNEL", "PTPC_FORCE_SWAP")

    def setenv(env):
        for k in names:
            monkeypatch.delenv(k, raising=False)
        for k, v in env.items():
            monkeypatch.setenv(k, v)
        ptpc.reload_tuning_overrides()

    T, Ci, Co = 32, 2048, 4096                 # 32 channel tiles: K split over 4 by default
    try:
        setenv({})
        assert ptpc.gemm_ksplit(T, Ci, Co) == 4
        monkeypatch.setenv("PTPC_FORCE_KSPLIT", "2")
        assert ptpc.gemm_ksplit(T, Ci, Co) == 4    # not re-read until a reload
        setenv({"PTPC_FORCE_KSPLIT": "2"})
        assert ptpc.gemm_ksplit(T, Ci, Co) == 2
        setenv({"PTPC_FORCE_KSPLIT": "8"})         # 32 x 8 CTAs do not fit in one wave: ignored
        assert ptpc.gemm_ksplit(T, Ci, Co) == 4
        setenv({"PTPC_FORCE_KSPLIT": "1"})
        assert ptpc.gemm_ksplit(T, Ci, Co) == 1
        X = synthetic.with_edge_rows(synthetic.make_x(synthetic.DECODE_70B, 0, 256, 1024), huge_bits=BIG_BF16)
        W = synthetic.random_bf16((1024, 2064), seed=17, scale=0.02)
        cases = [({"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_PAIR_BN": "128", "PTPC_FORCE_SWAP": "0"}, 100),
                 ({"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_PAIR_BN": "256", "PTPC_FORCE_SWAP": "0"}, 7),
                 ({"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_SWAP": "1"}, 7),
                 ({"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_SWAP": "1"}, 256),
                 ({"PTPC_FORCE_KERNEL": "decode"}, 256),
                 ({"PTPC_FORCE_KERNEL": "decode", "PTPC_FORCE_KSPLIT": "1"}, 64),
                 ({"PTPC_FORCE_KSPLIT": "2"}, 13)]
        for env, t in cases:
            setenv(env)
            g, r = run_pair(ptpc, X[:t].copy(), W)
            assert_gemm_close(g, r, f"forced {env} T={t}")
    finally:
        setenv({})
    assert ptpc.gemm_ksplit(T, Ci, Co) == 4


def test_tensor_map_cache(ptpc):
    """Repeated GEMM calls on the same buffers take their tensor maps from the
    library's host-side cache; another buffer of the same shape is a miss and
    still computes its own result."""
    T, Ci, Co = 64, 1024, 2048
    X = synthetic.make_x(synthetic.DECODE_70B, 0, T, Ci)
    W = synthetic.random_bf16((Ci, Co), seed=5, scale=0.02)
    Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W))
    Xq, xs = ptpc.quantize_activations(to_dev_bf16(X))
    out = ptpc.scaled_mm(Xq, xs, Wq_t, ws)
    h0, m0 = ptpc.map_cache_stats()
    for _ in range(5):
        ptpc.scaled_mm(Xq, xs, Wq_t, ws, out=out)
    h1, m1 = ptpc.map_cache_stats()
    assert m1 == m0 and h1 - h0 >= 10, (h0, m0, h1, m1)
    # same shape, other buffers (the second weight is the first one negated)
    Wq2, ws2 = ptpc.quantize_weights(to_dev_bf16(W ^ np.uint16(0x8000)))
    out2 = ptpc.scaled_mm(Xq, xs, Wq2, ws2)
    h2, m2 = ptpc.map_cache_stats()
    assert m2 > m1
    torch.cuda.synchronize()
    a = from_dev_bf16(out).astype(np.uint16)
    b = from_dev_bf16(out2).astype(np.uint16)
    nz = (a & 0x7FFF) != 0
    assert np.array_equal(a[nz] ^ np.uint16(0x8000), b[nz])


def test_naive_two_step_equals_fused(ptpc):
    """The page's naive path (GEMM -> fp32 intermediate -> scale) gives the
    same bits as the fused epilogue: same accumulator, same two products."""
    for T, Ci, Co in [(300, 1024, 768), (2048, 4096, 6144), (8, 8192, 1024)]:
        X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, T, Ci)
        W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, Ci, Co)
        Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W))
        Xq, xs = ptpc.quantize_activations(to_dev_bf16(X))
        fused = ptpc.scaled_mm(Xq, xs, Wq_t, ws)
        y = ptpc.unscaled_mm_f32(Xq, Wq_t)
        naive = ptpc.apply_scales(y, xs, ws)
        assert torch.equal(fused.view(torch.int16), naive.view(torch.int16)), (T, Ci, Co)
        # the intermediate itself is the dot product up to fp32 accumulation
        acc = oracle.gemm_acc64(Xq.cpu().numpy(), Wq_t.cpu().numpy())
        yy = y.cpu().numpy().astype(np.float64)
        rms = np.sqrt(np.mean(acc * acc))
        assert (np.abs(yy - acc) <= 1e-2 * np.abs(acc) + 1e-3 * rms).all()


def test_per_tensor_path(ptpc):
    X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, 300, 1024)
    W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, 1024, 768)
    Xq, xs = ptpc.quantize_activations_per_tensor(to_dev_bf16(X))
    Wq_t, ws = ptpc.quantize_weights_per_tensor(to_dev_bf16(W))
    out = from_dev_bf16(ptpc.scaled_mm(Xq, xs, Wq_t, ws))
    rXq, sx = oracle.quant_per_tensor(X)
    rWq, sw = oracle.quant_weight_per_tensor(W)
    ref = oracle.scaled_mm_reference(rXq, np.full(300, sx, np.float32), rWq, np.full(768, sw, np.float32))
    assert_gemm_close(out, ref, "per-tensor")


def test_extreme_codes_full_depth(ptpc):
    """All-448 operands at K = 28672: the largest dot products of the format."""
    T, Ci, Co = 130, 28672, 272
    rng = np.random.default_rng(1)
    Xq = np.full((T, Ci), 0x7E, np.uint8)
    Xq[1::2] = rng.choice(np.array([0x7E, 0xFE], np.uint8), size=(T // 2, Ci))
    Wq_t = np.full((Co, Ci), 0x7E, np.uint8)
    xs = np.full(T, 2.0 ** -12, np.float32)
    ws = np.full(Co, 2.0 ** -14, np.float32)
    out = ptpc.scaled_mm(to_dev(Xq), to_dev(xs), to_dev(Wq_t), to_dev(ws))
    ref = oracle.scaled_mm_reference(Xq, xs, Wq_t, ws)
    assert_gemm_close(from_dev_bf16(out), ref, "extreme")


def test_deterministic_and_status_clean(ptpc):
    for T, Ci, Co in [(1, 28672, 8192), (2048, 4096, 6144)]:
        X = synthetic.make_x(synthetic.DECODE_70B, 1, T, Ci)
        W = synthetic.make_w(synthetic.DECODE_70B, 1, Ci, Co)
        Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W))
        Xd = to_dev_bf16(X)
        wsp = ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, Ci, Co), "cuda")
        a = ptpc.linear(Xd, Wq_t, ws, ws=wsp)
        b = ptpc.linear(Xd, Wq_t, ws, ws=wsp)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert ptpc.device_status(wsp) == ptpc.OK


def test_empty_input_is_noop(ptpc):
    Wq_t = torch.zeros((64, 128), dtype=torch.uint8, device="cuda")
    ws = torch.ones(64, dtype=torch.float32, device="cuda")
    out = ptpc.linear(torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda"), Wq_t, ws)
    assert out.shape == (0, 64)


def test_workspace_shared_across_entry_points(ptpc):
    """Every entry point leaves the workspace's control words zero, so one
    workspace can serve the weight quantiser, the per-tensor quantiser and a
    decode GEMM with K split over a cluster in turn."""
    T, Ci, Co = 1, 28672, 8192
    need = max(ptpc.workspace_size(ptpc.OP_LINEAR, T, Ci, Co),
               ptpc.workspace_size(ptpc.OP_QUANTIZE_WEIGHTS, 0, Ci, Co),
               ptpc.workspace_size(ptpc.OP_BENCH_PER_TENSOR, T, Ci, 0))
    wsp = ptpc.Workspace(need, "cuda")
    W = synthetic.make_w(synthetic.DECODE_70B, 1, Ci, Co)
    X = synthetic.make_x(synthetic.DECODE_70B, 1, T, Ci)
    Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W), ws=wsp)
    ptpc.quantize_activations_per_tensor(to_dev_bf16(X), ws=wsp)
    torch.cuda.synchronize()
    assert int(wsp.buf[4:].count_nonzero()) == 0 or int(wsp.buf[256:].count_nonzero()) == 0
    out = from_dev_bf16(ptpc.linear(to_dev_bf16(X), Wq_t, ws, ws=wsp))
    rWq, rws = oracle.quant_weight(W)
    rXq, rxs = oracle.quant_act(X)
    assert_gemm_close(out, oracle.scaled_mm_reference(rXq, rxs, rWq, rws), "shared workspace")
    assert ptpc.device_status(wsp) == ptpc.OK


def test_linear_on_column_slice(ptpc):
    """The fused entry reads a layer input that is a column slice of the
    previous layer's output (row pitch > Ci) without a copy."""
    T, Ci, Co, wide = 300, 1024, 768, 1536
    Xw = synthetic.make_x(synthetic.LLAMA70B_PREFILL, 0, T, wide)
    W = synthetic.make_w(synthetic.LLAMA70B_PREFILL, 0, Ci, Co)
    Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W))
    out = ptpc.linear(to_dev_bf16(Xw)[:, :Ci], Wq_t, ws)
    X = np.ascontiguousarray(Xw[:, :Ci])
    ref, _, _ = oracle.linear_reference(X, *oracle.quant_weight(W))
    assert_gemm_close(from_dev_bf16(out), ref, "column slice")
    dense = ptpc.linear(to_dev_bf16(X), Wq_t, ws)
    assert torch.equal(dense.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("T,Ci,Co,fmt,forced", [
    (2048, 16384, 8192, "e4m3", False),                   # long K: split by the automatic plan
    (256, 8192, 57344, "e4m3", True), (300, 2048, 28672, "e4m3", True),
    (512, 4096, 10240, "e4m3", True), (1000, 1024, 5120, "e4m3", True),
    (300, 2048, 28672, "e2m1", True), (512, 4096, 10240, "e3m2", True)])
def test_split_tail(ptpc, monkeypatch, T, Ci, Co, fmt, forced):
    """Prefill shapes whose last wave of tiles is split along K over the GPU
    (partials through the workspace, distributed fixed-order reduction):
    parity with the oracle, agreement with the whole-tile plan, repeated
    calls on one workspace (its counters back at zero after each), no
    timeout in the status word.  Short-K shapes take the split only when
    PTPC_FORCE_SPLIT_TAIL=1 asks for it."""
    if forced:
        monkeypatch.setenv("PTPC_FORCE_SPLIT_TAIL", "1")
    ptpc.reload_tuning_overrides()
    try:
        _split_tail_case(ptpc, monkeypatch, T, Ci, Co, fmt)
    finally:
        monkeypatch.delenv("PTPC_FORCE_SPLIT_TAIL", raising=False)
        ptpc.reload_tuning_overrides()


def _split_tail_case(ptpc, monkeypatch, T, Ci, Co, fmt):
    assert ptpc.gemm_tail_split(T, Ci, Co) >= 2, "shape does not exercise the split tail"
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.CHAIN_70B, 2, T, Ci), huge_bits=BIG_BF16)
    W = synthetic.make_w(synthetic.CHAIN_70B, 2, Ci, Co)
    Xd = to_dev_bf16(X)
    Wq, ws_ = ptpc.quantize_weights_fmt(to_dev_bf16(W), fmt)
    Xq, xs = ptpc.quantize_activations(Xd)
    wsp = ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, Ci, Co), "cuda")
    outs = [ptpc.scaled_mm_fmt(Xq, xs, Wq, ws_, fmt, ws=wsp) for _ in range(3)]
    lin = ptpc.linear_fmt(Xd, Wq, ws_, fmt, ws=wsp)
    assert ptpc.device_status(wsp) == ptpc.OK
    assert int(wsp.buf[256:256 + 1024].count_nonzero()) == 0          # counters left at zero
    for o in outs[1:] + [lin]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))   # deterministic
    rXq, rxs = oracle.quant_act(X)
    rows = np.unique(np.concatenate([np.arange(0, T, 7), [T - 1]]))
    if fmt == "e4m3":
        rWq, rws = oracle.quant_weight(W)
        ref = oracle.scaled_mm_reference(rXq, rxs, rWq, rws, rows)
    else:
        codes, rws = oracle.quant_weight_fmt(W, fmt)
        ref = oracle.scaled_mm_reference_fmt(rXq, rxs, codes, rws, fmt, rows)
    assert_gemm_close(from_dev_bf16(outs[0])[rows], ref, f"split tail {fmt} T={T} {Ci}->{Co}")
    # the whole-tile plan of the same shape agrees within the tolerance
    try:
        monkeypatch.setenv("PTPC_FORCE_SPLIT_TAIL", "0")
        ptpc.reload_tuning_overrides()
        assert ptpc.gemm_tail_split(T, Ci, Co) == 0
        whole = ptpc.scaled_mm_fmt(Xq, xs, Wq, ws_, fmt, ws=wsp)
    finally:
        monkeypatch.delenv("PTPC_FORCE_SPLIT_TAIL")
        ptpc.reload_tuning_overrides()
    assert_gemm_close(from_dev_bf16(outs[0]), from_dev_bf16(whole), "split tail vs whole tiles")


def test_split_tail_needs_the_workspace(ptpc):
    """With only the status word of workspace the same shape runs whole
    tiles; short K and a mostly full last wave are not split."""
    assert ptpc.gemm_tail_split(2048, 16384, 8192) >= 2
    assert ptpc.gemm_tail_split(2048, 16384, 8192, ws_bytes=256) == 0
    assert ptpc.gemm_tail_split(256, 8192, 57344) == 0        # K = 8192: not worth it
    assert ptpc.gemm_tail_split(8192, 8192, 57344) == 0       # last wave mostly full: no split


def _set_tuning(ptpc, monkeypatch, env):
    for k in ("PTPC_FORCE_SWAP", "PTPC_FORCE_SPLIT_TAIL", "PTPC_FORCE_KERNEL"):
        monkeypatch.delenv(k, raising=False)
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    ptpc.reload_tuning_overrides()


@pytest.mark.parametrize("T,Ci,Co,fmt,env,nt", [
    (300, 8192, 10240, "e4m3", {}, 160),                          # 70B QKV at T = 300: chosen by the plan
    (300, 1024, 1040, "e4m3", {"PTPC_FORCE_SWAP": "1"}, 160),     # channels end inside a 32-wide store box
    (200, 512, 2064, "e4m3", {"PTPC_FORCE_SWAP": "1"}, 224),      # one token tile, 24 padded tokens
    (33, 256, 1040, "e4m3", {"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_SWAP": "1"}, 64),
    (600, 2048, 4096, "e4m3", {"PTPC_FORCE_SWAP": "1"}, 224),     # three token tiles
    (400, 1024, 2064, "e2m3", {"PTPC_FORCE_SWAP": "1"}, 224),     # FP6 weights as the M operand
    (300, 2048, 4096, "e2m1", {"PTPC_FORCE_SWAP": "1"}, 160),     # FP4 weights as the M operand
])
def test_swapped_operand_tiles(ptpc, monkeypatch, T, Ci, Co, fmt, env, nt):
    """The prefill kernel with the weights as the 256-row MMA operand and the
    tokens as the tile's columns (transposed epilogue): parity with the
    oracle on every row, the same output from linear, agreement with the
    unswapped plan, deterministic, no timeout."""
    try:
        _set_tuning(ptpc, monkeypatch, env)
        assert ptpc.gemm_swap_tokens(T, Ci, Co) == nt
        X = synthetic.with_edge_rows(synthetic.make_x(synthetic.CHAIN_70B, 0, T, Ci), huge_bits=BIG_BF16)
        W = synthetic.make_w(synthetic.CHAIN_70B, 0, Ci, Co)
        Xd = to_dev_bf16(X)
        Wq, ws_ = ptpc.quantize_weights_fmt(to_dev_bf16(W), fmt)
        Xq, xs = ptpc.quantize_activations(Xd)
        wsp = ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, Ci, Co), "cuda")
        a = ptpc.scaled_mm_fmt(Xq, xs, Wq, ws_, fmt, ws=wsp)
        b = ptpc.scaled_mm_fmt(Xq, xs, Wq, ws_, fmt, ws=wsp)
        lin = ptpc.linear_fmt(Xd, Wq, ws_, fmt, ws=wsp)
        assert ptpc.device_status(wsp) == ptpc.OK
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert torch.equal(a.view(torch.int16), lin.view(torch.int16))
        rXq, rxs = oracle.quant_act(X)
        assert np.array_equal(Xq.cpu().numpy(), rXq)
        if fmt == "e4m3":
            rWq, rws = oracle.quant_weight(W)
            ref = oracle.scaled_mm_reference(rXq, rxs, rWq, rws)
        else:
            codes, rws = oracle.quant_weight_fmt(W, fmt)
            ref = oracle.scaled_mm_reference_fmt(rXq, rxs, codes, rws, fmt)
        assert_gemm_close(from_dev_bf16(a), ref, f"swapped {fmt} T={T} {Ci}->{Co}")
        _set_tuning(ptpc, monkeypatch, {"PTPC_FORCE_SWAP": "0"})
        assert ptpc.gemm_swap_tokens(T, Ci, Co) == 0
        plain = ptpc.scaled_mm_fmt(Xq, xs, Wq, ws_, fmt, ws=wsp)
        assert_gemm_close(from_dev_bf16(a), from_dev_bf16(plain), "swapped vs unswapped")
    finally:
        _set_tuning(ptpc, monkeypatch, {})


@pytest.mark.parametrize("T,Ci,Co", [(300, 1024, 768), (77, 512, 1040)])
def test_swapped_naive_path(ptpc, monkeypatch, T, Ci, Co):
    """The fp32-output GEMM (the naive path's first step) with swapped
    operands: its accumulator is the oracle's dot product up to fp32
    accumulation, and scaling it afterwards gives the fused bits."""
    try:
        _set_tuning(ptpc, monkeypatch, {"PTPC_FORCE_KERNEL": "pair", "PTPC_FORCE_SWAP": "1"})
        X = synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, T, Ci)
        W = synthetic.make_w(synthetic.LLAMA8B_PREFILL, 0, Ci, Co)
        Wq_t, ws = ptpc.quantize_weights(to_dev_bf16(W))
        Xq, xs = ptpc.quantize_activations(to_dev_bf16(X))
        fused = ptpc.scaled_mm(Xq, xs, Wq_t, ws)
        y = ptpc.unscaled_mm_f32(Xq, Wq_t)
        naive = ptpc.apply_scales(y, xs, ws)
        assert torch.equal(fused.view(torch.int16), naive.view(torch.int16))
        acc = oracle.gemm_acc64(Xq.cpu().numpy(), Wq_t.cpu().numpy())
        yy = y.cpu().numpy().astype(np.float64)
        rms = np.sqrt(np.mean(acc * acc))
        assert (np.abs(yy - acc) <= 1e-2 * np.abs(acc) + 1e-3 * rms).all()
    finally:
        _set_tuning(ptpc, monkeypatch, {})


@pytest.mark.parametrize("split", ["0", "1"])
def test_swapped_70b_gate_up(ptpc, monkeypatch, split):
    """The 70B gate+up layer at T = 300 takes swapped tiles (with and
    without a split last wave); sampled rows against the oracle."""
    T, Ci, Co = 300, 8192, 57344
    try:
        _set_tuning(ptpc, monkeypatch, {"PTPC_FORCE_SPLIT_TAIL": split})
        assert ptpc.gemm_swap_tokens(T, Ci, Co) == 160
        assert (ptpc.gemm_tail_split(T, Ci, Co) >= 2) == (split == "1")
        rows = np.unique(np.concatenate([np.arange(0, T, 5), [T - 1]]))
        w = synthetic.CHAIN_70B
        g, r = run_pair(ptpc, synthetic.make_x(w, 2, T, Ci), synthetic.make_w(w, 2, Ci, Co), rows=rows)
        assert_gemm_close(g, r, f"70B gate_up T=300 swapped, split tail {split}")
    finally:
        _set_tuning(ptpc, monkeypatch, {})
