"""The CUDA side of the tensor-parallel layers on one GPU, with the ranks
emulated in one process (the collectives done by torch on the device):
the row-maximum kernel and the quantiser with given maxima against the
oracle (bit-exact, on column slices of a wider activation, as a rank holds
them), and the column- and row-parallel layers against the unsplit oracle
(codes and scales bit-exact, outputs within the GEMM tolerance)."""
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


@pytest.mark.parametrize("T,Ci,parts", [(1, 256, 2), (37, 4096, 2), (300, 8192, 4), (2048, 28672, 2),
                                        (5, 262144, 2)])
def test_row_split_quantisation(ptpc, T, Ci, parts):
    X = synthetic.with_edge_rows(synthetic.make_x(synthetic.LLAMA70B_PREFILL, 1, T, 28672)[:, :Ci]
                                 if Ci <= 28672 else synthetic.random_bf16((T, Ci), seed=2, scale=3.0))
    Xd = to_dev_bf16(X)
    w = Ci // parts
    slices = [Xd[:, r * w:(r + 1) * w] for r in range(parts)]       # column slices, row pitch Ci
    amax_r = [ptpc.row_amax(s) for s in slices]
    for r in range(parts):
        assert np.array_equal(amax_r[r].cpu().numpy(), oracle.row_amax(X[:, r * w:(r + 1) * w]))
    amax = torch.stack(amax_r).amax(dim=0)
    rXq, rxs = oracle.quant_act(X)
    for r in range(parts):
        Xq, xs = ptpc.quantize_activations_amax(slices[r], amax)
        assert np.array_equal(Xq.cpu().numpy(), rXq[:, r * w:(r + 1) * w]), r
        assert np.array_equal(xs.cpu().numpy().view(np.uint32), rxs.view(np.uint32)), r


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("T", [1, 128, 1000])
def test_parallel_layers_emulated(ptpc, world, T):
    from fp8_quantized_gemm_ptpc_b200.tp import ColumnParallelLinear, RowParallelLinear
    w = synthetic.LLAMA70B_PREFILL
    Ci, Co = 4096, 2064
    X = synthetic.with_edge_rows(synthetic.make_x(w, 0, T, Ci), huge_bits=0x7180)
    W = synthetic.random_bf16((Ci, Co), seed=T + world, scale=0.015)
    rWq, rws = oracle.quant_weight(W)
    ref, _, _ = oracle.linear_reference(X, rWq, rws)
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    # column-parallel: every rank's columns of the unsplit output
    cols = [ColumnParallelLinear(Wd, r, world) for r in range(world)]
    got = np.concatenate([from_dev_bf16(c.forward(Xd)) for c in cols], axis=1)
    assert_gemm_close(got, ref, f"column-parallel x{world} T={T}")
    # row-parallel: the three phases per rank, the reductions by torch
    rows = [RowParallelLinear(Wd, r, world) for r in range(world)]
    X_r = [Xd[:, l.k0:l.k1] for l in rows]
    amax = torch.stack([l.slice_amax(x) for l, x in zip(rows, X_r)]).amax(dim=0)
    parts = [l.partial(x, amax) for l, x in zip(rows, X_r)]
    acc = torch.stack([p[0] for p in parts]).sum(dim=0)
    for p in parts[1:]:
        assert torch.equal(p[1], parts[0][1])                      # same token scales on every rank
    out = rows[0].finish(acc, parts[0][1])
    assert_gemm_close(from_dev_bf16(out), ref, f"row-parallel x{world} T={T}")
