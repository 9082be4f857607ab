"""Seeded synthetic inputs for the PTPC-FP8 linear layers.

This module is shared by the tests, the benchmark and the smoke check.  It
only draws random numbers and lays them out as bf16 tensors; it holds none of
the method's arithmetic (no amax, no scale, no FP8 code, no GEMM), so the
oracle and the CUDA path can both be fed from it without sharing any step of
the computation.

Shapes follow the Llama-3.1-8B / 70B linear layers named in the workloads, and
the activations carry the structure that "PTPC-FP8: boosting vLLM performance
on AMD ROCm" (section "The outlier problem") describes: outliers sit in a few
fixed channels for every token, magnitudes vary strongly inside a token, and
weights are comparatively uniform.  No dataset or trained weight is used.

Seed recipe: ``seed = 1000 * workload + 10 * layer + {0: X, 1: W, 2: outlier
channel list}``; the tiny workload uses seed 0 for X and 1 for W.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Layer:
    name: str
    Ci: int
    Co: int


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    layers: tuple
    tokens: tuple          # token counts T this workload is run at
    x_kind: str            # "normal50" | "student_t" | "lognormal"
    w_sigma: float


# Workloads, numbered as the benchmark names them.
TINY = Workload(0, "tiny 16x256->512", (Layer("tiny", 256, 512),), (16,), "normal50", 0.02)
LLAMA8B_PREFILL = Workload(
    1, "Llama-3.1-8B prefill T=2048",
    (Layer("qkv", 4096, 6144), Layer("gate_up", 4096, 28672), Layer("down", 14336, 4096)),
    (2048,), "student_t", 0.02)
DECODE_70B = Workload(
    2, "70B decode T in {1,8,32,128}",
    (Layer("up", 8192, 28672), Layer("down", 28672, 8192)),
    (1, 8, 32, 128), "student_t", 0.02)
LLAMA70B_PREFILL = Workload(
    3, "Llama-3.1-70B prefill T=8192",
    (Layer("gate_up", 8192, 57344), Layer("down", 28672, 8192)),
    (8192,), "lognormal", 0.015)
CHAIN_70B = Workload(
    4, "70B 4-linear chain, ragged T",
    (Layer("qkv", 8192, 10240), Layer("o", 8192, 8192),
     Layer("gate_up", 8192, 57344), Layer("down", 28672, 8192)),
    tuple(sorted({2 ** i for i in range(15)} | {77, 1000, 3001})), "lognormal", 0.015)

WORKLOADS = (TINY, LLAMA8B_PREFILL, DECODE_70B, LLAMA70B_PREFILL, CHAIN_70B)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (PyTorch's cast) and return the bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _seed(w: Workload, layer: int, what: int) -> int:
    if w.index == 0:
        return what  # tiny workload: X seed 0, W seed 1
    return 1000 * w.index + 10 * layer + what


def outlier_channels(w: Workload, layer: int, Ci: int) -> np.ndarray:
    """Fixed outlier channels of one layer's input (same for every token)."""
    if w.x_kind == "normal50":
        return np.array([3, 77, 140, 201], dtype=np.int64)
    n = 8 if w.x_kind == "student_t" else 16
    rng = np.random.Generator(np.random.PCG64(_seed(w, layer, 2)))
    return np.sort(rng.choice(Ci, size=n, replace=False))


def make_x_f32(w: Workload, layer: int, T: int, Ci: int) -> np.ndarray:
    """fp32 activations before the bf16 cast."""
    rng = np.random.Generator(np.random.PCG64(_seed(w, layer, 0)))
    ch = outlier_channels(w, layer, Ci)
    if w.x_kind == "normal50":
        x = rng.standard_normal((T, Ci), dtype=np.float32)
        x[:, ch] *= 50.0
    elif w.x_kind == "student_t":
        x = (0.5 * rng.standard_t(3.0, size=(T, Ci))).astype(np.float32)
        x[:, ch] *= 30.0
    elif w.x_kind == "lognormal":
        x = rng.standard_normal((T, Ci), dtype=np.float32)
        x *= rng.lognormal(0.0, 1.0, size=(T, 1)).astype(np.float32)
        x[:, ch] *= 100.0
    else:
        raise ValueError(w.x_kind)
    return x


def make_x(w: Workload, layer: int, T: int, Ci: int) -> np.ndarray:
    """bf16 bit patterns [T, Ci] of one layer's input."""
    return to_bf16_bits(make_x_f32(w, layer, T, Ci))


def make_w(w: Workload, layer: int, Ci: int, Co: int) -> np.ndarray:
    """bf16 bit patterns [Ci, Co] of one layer's weight, N(0, sigma)."""
    rng = np.random.Generator(np.random.PCG64(_seed(w, layer, 1)))
    return to_bf16_bits(rng.standard_normal((Ci, Co), dtype=np.float32) * np.float32(w.w_sigma))


def random_bf16(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale) bf16 tensor for edge-case tests."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(scale))


def with_edge_rows(X_bits: np.ndarray, seed: int = 7, huge_bits: int = 0x7F7F) -> np.ndarray:
    """Copy of X with edge-case rows planted (when T is large enough):
    row 0 all +0, row 1 all -0, row 2 only bf16 subnormals,
    row 3 a single nonzero element, row 4 mixed +-0 and tiny normals,
    row 5 values of magnitude ``huge_bits`` (default: the bf16 maximum)."""
    X = np.array(X_bits, dtype=np.uint16, copy=True)
    T, Ci = X.shape
    rng = np.random.Generator(np.random.PCG64(seed))
    plans = []
    plans.append(lambda: np.zeros(Ci, np.uint16))                                   # +0 row
    plans.append(lambda: np.full(Ci, 0x8000, np.uint16))                            # -0 row
    plans.append(lambda: (rng.integers(1, 0x80, Ci).astype(np.uint16)
                          | (rng.integers(0, 2, Ci).astype(np.uint16) << 15)))      # subnormals
    def single():
        r = np.zeros(Ci, np.uint16)
        r[rng.integers(0, Ci)] = 0xC1A0                                             # -20.0
        return r
    plans.append(single)
    def mixed_tiny():
        r = rng.integers(0x0080, 0x0400, Ci).astype(np.uint16)                      # tiny normals
        r[rng.random(Ci) < 0.3] = 0x8000
        r[rng.random(Ci) < 0.3] = 0x0000
        r |= (rng.integers(0, 2, Ci).astype(np.uint16) << 15)
        return r
    plans.append(mixed_tiny)
    plans.append(lambda: (np.full(Ci, huge_bits, np.uint16)
                          | (rng.integers(0, 2, Ci).astype(np.uint16) << 15)))      # bf16 max
    for i, plan in enumerate(plans):
        if i < T:
            X[i] = plan()
    return X
