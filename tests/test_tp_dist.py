"""Tensor-parallel PTPC-FP8 linear layers (fp8_quantized_gemm_ptpc_b200.tp)
run as world-size-2 and -4 gloo ranks on CPU, with the oracle's arithmetic
plugged in for the kernels: the partitioning and the collectives must give
exactly the unsplit oracle results.  Column-parallel: each rank's output
columns, and the gathered output, equal the unsplit layer's.  Row-parallel:
the combined slice maxima give the unsplit scales and codes, and the summed
fp64 partial accumulators (exact) give the unsplit output bit for bit."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    """The oracle's arithmetic on CPU tensors, in place of the CUDA kernels."""

    def __init__(self):
        import oracle
        self.o = oracle

    def quantize_weights(self, W):
        q, s = self.o.quant_weight(_bits(W))
        return torch.from_numpy(q), torch.from_numpy(s)

    def linear(self, X, Wq_t, w_scale):
        out, _, _ = self.o.linear_reference(_bits(X), Wq_t.numpy(), w_scale.numpy())
        return _bf16(out)

    def row_amax(self, X):
        return torch.from_numpy(self.o.row_amax(_bits(X)))

    def quantize_activations_amax(self, X, amax):
        q, s = self.o.quant_act_amax(_bits(X), amax.numpy())
        return torch.from_numpy(q), torch.from_numpy(s)

    def unscaled_mm(self, Xq, Wq_t):
        return torch.from_numpy(self.o.gemm_acc64(Xq.numpy(), Wq_t.numpy()))   # exact fp64

    def apply_scales(self, acc, x_scale, w_scale):
        return _bf16(self.o.reference_epilogue(acc.numpy(), x_scale.numpy(), w_scale.numpy()))

    def slice_k(self, Wq_t, k0, k1):
        return Wq_t[:, k0:k1].contiguous()


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    import oracle
    import synthetic
    from fp8_quantized_gemm_ptpc_b200.tp import ColumnParallelLinear, RowParallelLinear
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w = synthetic.LLAMA70B_PREFILL
        T, Ci, Co = 37, 512, 272
        X = synthetic.with_edge_rows(synthetic.make_x(w, 0, T, Ci))
        W = synthetic.random_bf16((Ci, Co), seed=3, scale=0.015)
        Wq, ws = oracle.quant_weight(W)
        ref, rXq, rxs = oracle.linear_reference(X, Wq, ws)
        ops = OracleOps()
        res = {}
        col = ColumnParallelLinear(_bf16(W), rank, world, ops)
        mine = _bits(col.forward(_bf16(X)))
        res["col_own"] = bool(np.array_equal(mine, ref[:, col.o0:col.o1]))
        res["col_gather"] = bool(np.array_equal(_bits(col.forward(_bf16(X), gather=True)), ref))
        row = RowParallelLinear(_bf16(W), rank, world, ops)
        X_r = np.ascontiguousarray(X[:, row.k0:row.k1])
        amax = row.slice_amax(_bf16(X_r))
        dist.all_reduce(amax, op=dist.ReduceOp.MAX)
        q, s = ops.quantize_activations_amax(_bf16(X_r), amax)
        res["row_codes"] = bool(np.array_equal(q.numpy(), rXq[:, row.k0:row.k1]))
        res["row_scales"] = bool(np.array_equal(s.numpy().view(np.uint32), rxs.view(np.uint32)))
        res["row_out"] = bool(np.array_equal(_bits(row.forward(_bf16(X_r))), ref))
        res["k_range"] = (row.k0, row.k1)
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_tensor_parallel_layers_equal_the_unsplit_oracle(world):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    spans = []
    for r in range(world):
        res = out[r]
        for k in ("col_own", "col_gather", "row_codes", "row_scales", "row_out"):
            assert res[k], (r, k)
        spans.append(res["k_range"])
    assert spans[0][0] == 0 and spans[-1][1] == 512
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))


def test_shard_range():
    sys.path.insert(0, ROOT)
    from fp8_quantized_gemm_ptpc_b200.tp import shard_range
    assert [shard_range(8192, r, 2) for r in range(2)] == [(0, 4096), (4096, 8192)]
    assert [shard_range(272, r, 4) for r in range(4)] == [(0, 80), (80, 144), (144, 208), (208, 272)]
    assert shard_range(256, 3, 4, align=128) == (256, 256)      # no share left
    with pytest.raises(ValueError):
        shard_range(100, 0, 2)
