"""Register and local-memory budget of the hot kernels, from the compiler's
own resource report (nvcc -Xptxas -v, sm_100a), checked on the CPU.

The GEMM kernels, the tensor-memory attention kernel, the exact-split
activation quantiser that the prefill step runs, the sub-byte weight
quantiser and the KV-cache append must not spill registers to local memory,
and the attention kernel must fit two CTAs of 192 threads on an SM
(__launch_bounds__(192, 2): at most 168 registers a thread).
"""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "fp8_quantized_gemm_ptpc_b200", "csrc")

HOT = ("ptpc_gemm_pair_kernel", "ptpc_gemm_decode_kernel", "decode_attn_tc_kernel", "quant_act_exact_kernel",
       "quant_weight_sub_kernel", "kv_append_kernel")


def nvcc_flags():
    """The library's own compile flags (its build script, loaded by path)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("_ptpc_build_flags",
                                                  os.path.join(ROOT, "fp8_quantized_gemm_ptpc_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    return [f for f in build.NVCC_FLAGS if f not in ("-Xcompiler", "-fPIC") and not f.startswith("-fvisibility")]


@pytest.fixture(scope="module")
def reports(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    out = tmp_path_factory.mktemp("ptxas")
    flags = nvcc_flags()
    procs = {}
    for src in ("gemm.cu", "attention_tc.cu", "quant.cu"):
        cmd = [nvcc] + flags + ["-Xptxas", "-v", "-c", os.path.join(CSRC, src), "-o", str(out / (src + ".o"))]
        procs[src] = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    text = {}
    for src, p in procs.items():
        log, _ = p.communicate(timeout=900)
        assert p.returncode == 0, log[-2000:]
        text[src] = log
    return "\n".join(text.values())


def entries(log):
    """(mangled name, registers, spill store bytes, spill load bytes) per entry function."""
    res = []
    for block in re.split(r"ptxas info\s*: Compiling entry function ", log)[1:]:
        name = re.match(r"'([^']+)'", block).group(1)
        spill = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", block)
        regs = re.search(r"Used (\d+) registers", block)
        res.append((name, int(regs.group(1)) if regs else None, int(spill.group(1)), int(spill.group(2))))
    return res


def test_hot_kernels_do_not_spill(reports):
    found = {h: 0 for h in HOT}
    bad = []
    for name, regs, st, ld in entries(reports):
        for h in HOT:
            if h in name:
                found[h] += 1
                if st or ld:
                    bad.append(f"{name}: {st} B spill stores, {ld} B spill loads")
    assert all(found.values()), found
    assert not bad, "\n".join(bad)


def test_attention_kernel_fits_two_ctas_an_sm(reports):
    regs = [r for name, r, _, _ in entries(reports) if "decode_attn_tc_kernel" in name]
    assert regs and max(regs) <= 168, regs
