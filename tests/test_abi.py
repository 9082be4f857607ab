"""The C-ABI library loads, exports every symbol include/ptpc.h declares, and
rejects bad arguments before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ptpc():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_ptpc_build", os.path.join(ROOT, "fp8_quantized_gemm_ptpc_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
    import fp8_quantized_gemm_ptpc_b200 as p
    return p


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "ptpc.h")).read()
    return sorted(set(re.findall(r"PTPC_API[^;(]*?\b(ptpc_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ["ptpc_quantize_activations", "ptpc_quantize_weights", "ptpc_scaled_mm", "ptpc_linear",
              "ptpc_workspace_size", "ptpc_get_device_status", "ptpc_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(ptpc):
    lib = ctypes.CDLL(ptpc.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert set(declared_symbols()) == set(ptpc.SIGNATURES)


def test_status_strings(ptpc):
    assert ptpc.status_string(0) == "PTPC_OK"
    assert ptpc.status_string(ptpc.ERR_DEVICE_TIMEOUT) == "PTPC_ERR_DEVICE_TIMEOUT"
    assert ptpc.status_string(999) == "PTPC_ERR_UNKNOWN"


def test_workspace_sizes(ptpc):
    ws = ptpc.workspace_size
    assert ws(ptpc.OP_SCALED_MM, 2048, 4096, 6144) % 256 == 0
    assert ws(ptpc.OP_SCALED_MM, 2048, 4096, 6144) >= 256
    assert ws(ptpc.OP_LINEAR, 2048, 4096, 6144) >= ws(ptpc.OP_SCALED_MM, 2048, 4096, 6144) + 2048 * 4096
    assert ws(ptpc.OP_QUANTIZE_WEIGHTS, 0, 4096, 6144) >= 256 + 4 * 6145
    assert ws(ptpc.OP_SCALED_MM, 16, 100, 64) == 0          # Ci not a multiple of 16
    assert ws(ptpc.OP_SCALED_MM, -1, 128, 64) == 0
    assert ws(99, 16, 128, 64) == 0
    # decode-sized T: the device status word only; prefill-sized T: room for
    # the split tail (74 CTA pairs x a 256 x 256 fp32 partial + counters)
    assert ws(ptpc.OP_SCALED_MM, 1, 28672, 8192) == 256
    assert ws(ptpc.OP_SCALED_MM, 192, 8192, 57344) == 256
    big = 256 + 1024 + 74 * 256 * 256 * 4
    assert ws(ptpc.OP_SCALED_MM, 8192, 28672, 8192) == big
    assert ws(ptpc.OP_SCALED_MM, 300, 768, 1040) == 256           # K too short to split
    assert ws(ptpc.OP_LINEAR, 8192, 28672, 8192) == big + 8192 * 28672 + 8192 * 4
    assert ws(ptpc.OP_BENCH_UNSCALED_MM, 8192, 28672, 8192) == 256


def test_ksplit_query_rejects_bad_shapes(ptpc):
    assert ptpc.gemm_ksplit(16, 100, 64) == 0     # Ci not a multiple of 16
    assert ptpc.gemm_ksplit(16, 128, 60) == 0     # Co not a multiple of 16
    assert ptpc.gemm_ksplit(-1, 128, 64) == 0
    assert ptpc.gemm_ksplit(0, 128, 64) == 0      # nothing to run


FAKE = 0x10000  # 16-byte aligned, never dereferenced: checks fail before any access


def call(ptpc, name, *args):
    return getattr(ptpc.lib, name)(*args)


def test_argument_checks_without_gpu(ptpc):
    P = ctypes.c_void_p
    q = lambda *a: call(ptpc, "ptpc_quantize_activations", *a)
    assert q(P(FAKE), 16, 100, 100, P(FAKE), P(FAKE), None) == ptpc.ERR_UNSUPPORTED_SHAPE
    assert q(P(FAKE), -1, 128, 128, P(FAKE), P(FAKE), None) == ptpc.ERR_INVALID_ARG
    assert q(None, 16, 128, 128, P(FAKE), P(FAKE), None) == ptpc.ERR_INVALID_ARG
    assert q(P(FAKE + 8), 16, 128, 128, P(FAKE), P(FAKE), None) == ptpc.ERR_MISALIGNED
    assert q(P(FAKE), 16, 128, 100, P(FAKE), P(FAKE), None) == ptpc.ERR_INVALID_ARG   # ldx < Ci
    assert q(P(FAKE), 16, 128, 132, P(FAKE), P(FAKE), None) == ptpc.ERR_MISALIGNED    # 16-byte rows
    assert q(None, 0, 128, 128, None, None, None) == ptpc.OK     # T == 0: no-op
    mm = lambda *a: call(ptpc, "ptpc_scaled_mm", *a)
    need = ptpc.workspace_size(ptpc.OP_SCALED_MM, 16, 128, 64)
    assert mm(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 16, 128, 64, P(FAKE), P(FAKE), need - 1, None) == \
        ptpc.ERR_WORKSPACE_TOO_SMALL
    assert mm(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 16, 128, 60, P(FAKE), P(FAKE), need, None) == \
        ptpc.ERR_UNSUPPORTED_SHAPE
    assert mm(P(FAKE), P(FAKE), P(FAKE), P(FAKE + 4), 16, 128, 64, P(FAKE), P(FAKE), need, None) == \
        ptpc.ERR_MISALIGNED
    assert mm(P(FAKE), None, P(FAKE), P(FAKE), 16, 128, 64, P(FAKE), P(FAKE), need, None) == \
        ptpc.ERR_INVALID_ARG
    lin = lambda *a: call(ptpc, "ptpc_linear", *a)
    need = ptpc.workspace_size(ptpc.OP_LINEAR, 16, 128, 64)
    assert lin(P(FAKE), 128, P(FAKE), P(FAKE), 16, 128, 64, P(FAKE), P(FAKE), need - 256, None) == \
        ptpc.ERR_WORKSPACE_TOO_SMALL
    assert lin(P(FAKE), 64, P(FAKE), P(FAKE), 16, 128, 64, P(FAKE), P(FAKE), need, None) == ptpc.ERR_INVALID_ARG
    assert lin(None, 128, None, None, 0, 128, 64, None, None, 0, None) == ptpc.OK
    qw = lambda *a: call(ptpc, "ptpc_quantize_weights", *a)
    need = ptpc.workspace_size(ptpc.OP_QUANTIZE_WEIGHTS, 0, 128, 64)
    assert qw(P(FAKE), 128, 64, P(FAKE), P(FAKE), P(FAKE), need - 1, None) == ptpc.ERR_WORKSPACE_TOO_SMALL
    assert qw(P(FAKE), 128, 0, P(FAKE), P(FAKE), P(FAKE), need, None) == ptpc.ERR_UNSUPPORTED_SHAPE
    assert call(ptpc, "ptpc_get_device_status", None, None) == ptpc.ERR_INVALID_ARG
    assert call(ptpc, "ptpc_bench_apply_scales", P(FAKE), P(FAKE), P(FAKE), -3, 64, P(FAKE), None) == \
        ptpc.ERR_INVALID_ARG
    probe = lambda *a: call(ptpc, "ptpc_bench_clock_probe", *a)
    assert probe(P(FAKE), 1, 1000000, 1000000, P(FAKE), None) == ptpc.ERR_INVALID_ARG      # < 2 records
    assert probe(P(FAKE), 64, 10, 1000000, P(FAKE), None) == ptpc.ERR_INVALID_ARG          # period < 1 us
    assert probe(P(FAKE), 64, 1000000, 121 * 10**9, P(FAKE), None) == ptpc.ERR_INVALID_ARG  # > 120 s
    assert probe(P(FAKE + 4), 64, 1000000, 1000000, P(FAKE), None) == ptpc.ERR_MISALIGNED
    assert probe(None, 64, 1000000, 1000000, P(FAKE), None) == ptpc.ERR_INVALID_ARG
    assert call(ptpc, "ptpc_selftest_wait_timeout", None, None) == ptpc.ERR_INVALID_ARG
    assert call(ptpc, "ptpc_selftest_wait_timeout", P(FAKE + 16), None) == ptpc.ERR_MISALIGNED


def test_binding_rejects_cpu_tensors(ptpc):
    import torch
    with pytest.raises(TypeError):
        ptpc.quantize_activations(torch.zeros(4, 16, dtype=torch.bfloat16))


def test_weight_format_argument_checks(ptpc):
    P = ctypes.c_void_p
    wb = lambda *a: call(ptpc, "ptpc_weight_bytes", *a)
    assert wb(0, 4096, 6144) == 4096 * 6144
    assert wb(1, 4096, 6144) == 4096 * 6144 // 2
    assert wb(2, 4096, 6144) == 4096 * 6144 * 3 // 4
    assert wb(3, 8192, 16) == 8192 * 16 * 3 // 4
    assert wb(1, 4112, 16) == 0          # sub-byte rows need Ci % 128 == 0
    assert wb(4, 4096, 16) == 0          # unknown format
    need = ptpc.workspace_size(ptpc.OP_QUANTIZE_WEIGHTS, 0, 256, 64)
    qw = lambda *a: call(ptpc, "ptpc_quantize_weights_fmt", *a)
    assert qw(P(FAKE), 256, 64, 7, P(FAKE), P(FAKE), P(FAKE), need, None) == ptpc.ERR_INVALID_ARG
    assert qw(P(FAKE), 144, 64, 1, P(FAKE), P(FAKE), P(FAKE), need, None) == ptpc.ERR_UNSUPPORTED_SHAPE
    assert qw(P(FAKE), 256, 64, 2, P(FAKE + 16), P(FAKE), P(FAKE), need, None) == ptpc.ERR_MISALIGNED
    assert qw(P(FAKE), 256, 64, 3, P(FAKE), P(FAKE), P(FAKE), need - 1, None) == ptpc.ERR_WORKSPACE_TOO_SMALL
    mm = lambda *a: call(ptpc, "ptpc_scaled_mm_fmt", *a)
    need = ptpc.workspace_size(ptpc.OP_SCALED_MM, 16, 256, 64)
    assert mm(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 9, 16, 256, 64, P(FAKE), P(FAKE), need, None) == \
        ptpc.ERR_INVALID_ARG
    assert mm(P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1, 16, 272, 64, P(FAKE), P(FAKE), need, None) == \
        ptpc.ERR_UNSUPPORTED_SHAPE
    assert mm(P(FAKE), P(FAKE), P(FAKE + 16), P(FAKE), 2, 16, 256, 64, P(FAKE), P(FAKE), need, None) == \
        ptpc.ERR_MISALIGNED
    assert mm(None, None, None, None, 1, 0, 256, 64, None, None, 0, None) == ptpc.OK
    lin = lambda *a: call(ptpc, "ptpc_linear_fmt", *a)
    need = ptpc.workspace_size(ptpc.OP_LINEAR, 16, 256, 64)
    assert lin(P(FAKE), 256, P(FAKE), P(FAKE), 3, 16, 256, 64, P(FAKE), P(FAKE), need - 256, None) == \
        ptpc.ERR_WORKSPACE_TOO_SMALL
    assert lin(P(FAKE), 256, P(FAKE + 16), P(FAKE), 1, 16, 256, 64, P(FAKE), P(FAKE), need, None) == \
        ptpc.ERR_MISALIGNED


def test_kv_cache_argument_checks(ptpc):
    P = ctypes.c_void_p
    ap = lambda *a: call(ptpc, "ptpc_kv_cache_append", *a)
    args = [P(FAKE), P(FAKE), P(FAKE), 4, 8, 128, 16, 10, P(FAKE), P(FAKE), P(FAKE), P(FAKE), None]
    bad = list(args); bad[5] = 96
    assert ap(*bad) == ptpc.ERR_UNSUPPORTED_SHAPE          # head size 64 or 128
    bad = list(args); bad[3] = -1
    assert ap(*bad) == ptpc.ERR_INVALID_ARG
    bad = list(args); bad[2] = P(FAKE + 4)
    assert ap(*bad) == ptpc.ERR_MISALIGNED                 # int64 slots
    bad = list(args); bad[3] = 0
    assert ap(*bad) == ptpc.OK
    wsz = lambda *a: call(ptpc, "ptpc_decode_attention_workspace_size", *a)
    assert wsz(32, 64, 128, 4096) == 256 + 32 * 64 * 8 * (2 + 128) * 4   # status word, then the chunks
    assert wsz(32, 64, 96, 4096) == 0
    at = lambda *a: call(ptpc, "ptpc_decode_attention", *a)
    need = wsz(2, 16, 128, 100)
    base = [P(FAKE)] * 7 + [2, 16, 8, 128, 16, 10, 7, 100, ctypes.c_float(0.1), P(FAKE), P(FAKE), need, None]
    bad = list(base); bad[8] = 12
    assert at(*bad) == ptpc.ERR_UNSUPPORTED_SHAPE           # Hq not a multiple of Hkv
    bad = list(base); bad[8] = 256; bad[9] = 8
    assert at(*bad) == ptpc.ERR_UNSUPPORTED_SHAPE           # group of 32 query heads
    bad = list(base); bad[12] = 2 ** 27
    assert at(*bad) == ptpc.ERR_UNSUPPORTED_SHAPE           # 2^31 cache slots
    bad = list(base); bad[-2] = need - 1
    assert at(*bad) == ptpc.ERR_WORKSPACE_TOO_SMALL
    bad = list(base); bad[7] = 0
    assert at(*bad) == ptpc.OK


def test_tensor_map_cache_logic(ptpc):
    """The host-side tensor-map cache (hits, misses for another pointer or
    shape, emptying at capacity, failed encodes) on a private instance with a
    stand-in encoder: no GPU needed."""
    assert call(ptpc, "ptpc_bench_map_cache_selftest") == ptpc.OK


def test_decode_attention_kernel_choice(ptpc, monkeypatch):
    """Which decode-attention kernel a shape runs: the tensor-memory kernel
    for the shapes it takes (D = 128, blocks of a multiple of 8; groups up to
    16), the warp-level kernel otherwise or when forced, 0 for invalid
    arguments.  Host logic only."""
    k = lambda *a: call(ptpc, "ptpc_decode_attention_kernel", *a)
    try:
        monkeypatch.delenv("PTPC_FORCE_ATTN_KERNEL", raising=False)
        ptpc.reload_tuning_overrides()
        assert k(64, 8, 128, 16) == 2 and k(64, 8, 64, 16) == 1 and k(128, 8, 128, 16) == 2
        monkeypatch.setenv("PTPC_FORCE_ATTN_KERNEL", "tc")
        ptpc.reload_tuning_overrides()
        assert k(64, 8, 128, 16) == 2 and k(8, 8, 128, 8) == 2 and k(24, 3, 128, 48) == 2
        assert k(64, 8, 64, 16) == 1                # D = 64
        assert k(128, 8, 128, 16) == 2 and k(96, 8, 128, 16) == 2   # groups of 16 and 12
        assert k(64, 8, 128, 12) == 1               # block of 12 positions
        assert k(12, 8, 128, 16) == 0 and k(64, 0, 128, 16) == 0 and k(64, 8, 96, 16) == 0
        assert k(64, 8, 128, 0) == 0
        monkeypatch.setenv("PTPC_FORCE_ATTN_KERNEL", "mma")
        ptpc.reload_tuning_overrides()
        assert k(64, 8, 128, 16) == 1
    finally:
        monkeypatch.delenv("PTPC_FORCE_ATTN_KERNEL", raising=False)
        ptpc.reload_tuning_overrides()


def test_binding_remembers_workspace_sizes_until_overrides_reload(ptpc):
    """The binding remembers ptpc_workspace_size per (op, shape, device) and
    forgets it when the tuning overrides are re-read (a forced plan may need
    another size).  Host logic only."""
    import torch
    dev = torch.device("cuda", 0)
    for op, T, Ci, Co in ((ptpc.OP_LINEAR, 1, 8192, 8192), (ptpc.OP_LINEAR, 8192, 8192, 57344),
                          (ptpc.OP_SCALED_MM, 300, 8192, 10240)):
        assert ptpc._ws_need(op, T, Ci, Co, dev) == ptpc.workspace_size(op, T, Ci, Co)
    assert len(ptpc._size_cache) >= 3
    ptpc.reload_tuning_overrides()
    assert len(ptpc._size_cache) == 0


def test_release_default_workspaces(ptpc, monkeypatch):
    """The cached default workspaces are dropped per device or all at once
    (host logic: the cache is filled with placeholders, no device memory)."""
    import torch
    cache = {(torch.device("cuda", 0), 11): object(), (torch.device("cuda", 0), 12): object(),
             (torch.device("cuda", 1), 11): object()}
    monkeypatch.setattr(ptpc, "_ws_cache", dict(cache))
    assert ptpc.release_default_workspaces("cuda:1") == 1
    assert set(ptpc._ws_cache) == {(torch.device("cuda", 0), 11), (torch.device("cuda", 0), 12)}
    assert ptpc.release_default_workspaces("cuda:3") == 0
    assert ptpc.release_default_workspaces() == 2
    assert ptpc._ws_cache == {}


def test_binding_fails_loudly_without_the_library(tmp_path):
    """The package refuses to import when libptpc.so has not been built: no
    fallback path exists.  (A copy of the binding in a folder with no _lib.)"""
    import shutil
    import subprocess
    import sys
    src = os.path.join(ROOT, "fp8_quantized_gemm_ptpc_b200", "__init__.py")
    pkg = tmp_path / "fp8_quantized_gemm_ptpc_b200"
    pkg.mkdir()
    shutil.copy(src, pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import fp8_quantized_gemm_ptpc_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "is missing" in r.stderr
