"""Shared test helpers: tolerance check and tensor conversions."""
import numpy as np
import torch

import oracle

# GEMM tolerance: |gpu - ref| <= REL * |ref| + ABS_RMS * rms(ref), per element,
# against the fp64-accumulated reference rounded to bf16.
REL = 1e-2
ABS_RMS = 1e-3


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_float(bits).astype(np.float64)


def assert_gemm_close(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str = ""):
    g = bf16_bits_to_float(gpu_bits)
    r = bf16_bits_to_float(ref_bits)
    assert g.shape == r.shape
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    err = np.abs(g - r)
    bound = REL * np.abs(r) + ABS_RMS * rms
    bad = ~(err <= bound)   # NaN or inf on either side counts as a mismatch
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu {g[tuple(i)]} ref {r[tuple(i)]} bound {bound[tuple(i)]}")
    return float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)
