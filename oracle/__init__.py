"""PTPC-FP8 oracle (test infrastructure only).

Plain CPU definitions of every step on the PTPC-FP8 hot path, used to check the
CUDA library.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package; the product path never does, and
this package imports nothing from the product.

Source: "PTPC-FP8: boosting vLLM performance on AMD ROCm" (vLLM blog), sections
"What is PTPC-FP8", "Per-Token Activation + Per-Channel Weight Quantization"
(tensor shapes X: T x Ci, W: Ci x Co, scale vectors Delta_X[T x 1] and
Delta_W[1 x Co]) and "The challenge: two-step vs fused" (the naive path: an
unscaled FP8 GEMM into an intermediate, then a rescale by the token scales and
then the channel scales; the fused path: the GEMM given both scale vectors).

The element-wise steps (E4M3 codec, bf16 rounding, quantisers, fp32
epilogues) are plain C in ``ptpc_oracle.c``; the dot products use a library
fp64 matrix product, which is exact here (see :func:`gemm_acc64`).

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
values fixed independently of this code (the OCP E4M3 definition, PyTorch's
own float8/bfloat16 casts, exact integer dot products, hand-derived golden
fixtures and invariants of the method).  No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ptpc_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

# Every finite E4M3 magnitude is an integer multiple of 2^-9 below 2^18 units,
# so a product of two is an integer multiple of 2^-18 below 2^36 units and a
# sum of K such products stays below 2^(36 + log2 K) units.  For K <= 2^17 that
# is below 2^53: every partial sum is exact in fp64, whatever the order.
MAX_EXACT_K = 1 << 17


def build(force: bool = False) -> str:
    """Compile ptpc_oracle.c into _build/liboracle.so (gcc, no FMA contraction)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-std=c11", _SRC, "-o", _LIB_PATH + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_e4m3_decode.restype = ctypes.c_double
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_scale_from_amax.restype = ctypes.c_float
            lib.oracle_scale_from_amax.argtypes = [ctypes.c_float]
            lib.oracle_quantize_value.restype = ctypes.c_uint8
            lib.oracle_quantize_value.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_float]
            lib.oracle_bf16_from_double.restype = ctypes.c_uint16
            lib.oracle_bf16_from_double.argtypes = [ctypes.c_double]
            lib.oracle_fmt_decode.restype = ctypes.c_double
            lib.oracle_fmt_decode.argtypes = [ctypes.c_uint8, ctypes.c_int]
            lib.oracle_fmt_encode.restype = ctypes.c_uint8
            lib.oracle_fmt_encode.argtypes = [ctypes.c_float, ctypes.c_int]
            lib.oracle_fmt_max.restype = ctypes.c_double
            lib.oracle_fmt_max.argtypes = [ctypes.c_int]
            lib.oracle_packed_row_bytes.restype = ctypes.c_int64
            lib.oracle_packed_row_bytes.argtypes = [ctypes.c_int64, ctypes.c_int]
            for name, args in {
                "oracle_quant_act": [P, I64, I64, P, P],
                "oracle_quant_weight": [P, I64, I64, P, P],
                "oracle_quant_per_tensor": [P, I64, P, P],
                "oracle_quant_weight_per_tensor": [P, I64, I64, P, P],
                "oracle_apply_scales_f32": [P, I64, I64, P, P, P],
                "oracle_fused_epilogue_f32": [P, I64, I64, P, P, P],
                "oracle_reference_epilogue_f64": [P, I64, I64, P, P, P],
                "oracle_e4m3_encode_array": [P, I64, P],
                "oracle_bf16_from_double_array": [P, I64, P],
                "oracle_quant_weight_fmt": [P, I64, I64, ctypes.c_int, P, P],
                "oracle_pack_fmt": [P, I64, I64, ctypes.c_int, P],
                "oracle_fmt_encode_array": [P, I64, ctypes.c_int, P],
                "oracle_row_amax": [P, I64, I64, P],
                "oracle_quant_act_amax": [P, I64, I64, P, P, P],
            }.items():
                fn = getattr(lib, name)
                fn.restype = None
                fn.argtypes = args
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


# --------------------------------------------------------------------------
# Codec
# --------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    """Value of one OCP E4M3 code (NaN for 0x7F / 0xFF)."""
    return float(_load().oracle_e4m3_decode(int(code)))


def e4m3_decode_table() -> np.ndarray:
    """fp64 value of each of the 256 E4M3 codes."""
    lib = _load()
    return np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(v) -> np.ndarray:
    """Saturating round-half-to-even E4M3 codes of fp32 values."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.empty(a.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(a), a.size, _ptr(out))
    return out


def bf16_from_double(v) -> np.ndarray:
    """bf16 bit patterns (uint16) of fp64 values, round-half-to-even."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_bf16_from_double_array(_ptr(a), a.size, _ptr(out))
    return out


def bf16_to_float(bits) -> np.ndarray:
    """Exact fp32 values of bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def scale_from_amax(amax: float) -> float:
    return float(_load().oracle_scale_from_amax(float(amax)))


def quantize_value(x: float, s: float, amax: float) -> int:
    return int(_load().oracle_quantize_value(float(x), float(s), float(amax)))


# --------------------------------------------------------------------------
# Quantisers
# --------------------------------------------------------------------------

def quant_act(X_bits: np.ndarray):
    """Per-token quantisation of X (T x Ci bf16 bits) -> (Xq [T,Ci] u8, x_scale [T] f32)."""
    X = np.ascontiguousarray(X_bits, dtype=np.uint16)
    T, Ci = X.shape
    Xq = np.empty((T, Ci), dtype=np.uint8)
    xs = np.empty((T,), dtype=np.float32)
    _load().oracle_quant_act(_ptr(X), T, Ci, _ptr(Xq), _ptr(xs))
    return Xq, xs


def quant_weight(W_bits: np.ndarray):
    """Per-output-channel quantisation of W (Ci x Co bf16 bits)
    -> (Wq_t [Co,Ci] u8, w_scale [Co] f32)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    Ci, Co = W.shape
    Wq_t = np.empty((Co, Ci), dtype=np.uint8)
    ws = np.empty((Co,), dtype=np.float32)
    _load().oracle_quant_weight(_ptr(W), Ci, Co, _ptr(Wq_t), _ptr(ws))
    return Wq_t, ws


def quant_per_tensor(X_bits: np.ndarray):
    """Per-tensor quantisation of any bf16 tensor -> (codes, scalar scale)."""
    X = np.ascontiguousarray(X_bits, dtype=np.uint16)
    q = np.empty(X.shape, dtype=np.uint8)
    s = np.empty((1,), dtype=np.float32)
    _load().oracle_quant_per_tensor(_ptr(X), X.size, _ptr(q), _ptr(s))
    return q, float(s[0])


def quant_weight_per_tensor(W_bits: np.ndarray):
    """Per-tensor quantisation of W (Ci x Co) with the codes transposed (Co x Ci)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    Ci, Co = W.shape
    Wq_t = np.empty((Co, Ci), dtype=np.uint8)
    s = np.empty((1,), dtype=np.float32)
    _load().oracle_quant_weight_per_tensor(_ptr(W), Ci, Co, _ptr(Wq_t), _ptr(s))
    return Wq_t, float(s[0])


# --------------------------------------------------------------------------
# GEMM and epilogues
# --------------------------------------------------------------------------

def gemm_acc64(Xq: np.ndarray, Wq_t: np.ndarray, rows=None, col_chunk: int = 4096) -> np.ndarray:
    """acc[t, o] = sum_k dec(Xq[t, k]) * dec(Wq_t[o, k]) in fp64.

    Exact (see MAX_EXACT_K): the library matrix product may sum in any order.
    ``rows`` selects a subset of tokens; ``col_chunk`` only bounds the memory
    of the decoded weight block and does not change any value.
    """
    Ci = Xq.shape[1]
    assert Wq_t.shape[1] == Ci and Ci <= MAX_EXACT_K
    dec = e4m3_decode_table()
    A = dec[Xq if rows is None else Xq[np.asarray(rows)]]
    Co = Wq_t.shape[0]
    acc = np.empty((A.shape[0], Co), dtype=np.float64)
    for o0 in range(0, Co, col_chunk):
        B = dec[Wq_t[o0:o0 + col_chunk]]
        acc[:, o0:o0 + col_chunk] = A @ B.T
    return acc


def scaled_mm_reference(Xq, x_scale, Wq_t, w_scale, rows=None) -> np.ndarray:
    """Tolerance reference of the fused scaled GEMM:
    out[t, o] = bf16_RNE(x_scale[t] * w_scale[o] * acc[t, o]) in fp64.
    Returns bf16 bit patterns [len(rows) or T, Co]."""
    acc = gemm_acc64(Xq, Wq_t, rows)
    xs = np.ascontiguousarray(np.asarray(x_scale, dtype=np.float32)[
        slice(None) if rows is None else np.asarray(rows)])
    ws = np.ascontiguousarray(w_scale, dtype=np.float32)
    out = np.empty(acc.shape, dtype=np.uint16)
    _load().oracle_reference_epilogue_f64(_ptr(acc), acc.shape[0], acc.shape[1],
                                          _ptr(xs), _ptr(ws), _ptr(out))
    return out


def linear_reference(X_bits, Wq_t, w_scale, rows=None):
    """The fused entry: per-token quantisation of X followed by the scaled GEMM.
    Returns (out bf16 bits, Xq, x_scale)."""
    Xq, xs = quant_act(X_bits)
    return scaled_mm_reference(Xq, xs, Wq_t, w_scale, rows), Xq, xs


def naive_step1_f32(Xq, Wq_t, rows=None) -> np.ndarray:
    """Naive step 1: the unscaled FP8 GEMM written out as an fp32 array."""
    return gemm_acc64(Xq, Wq_t, rows).astype(np.float32)


def naive_step2_apply_scales(y32, x_scale, w_scale) -> np.ndarray:
    """Naive step 2: bf16((y * token_scale) * channel_scale), fp32 products."""
    y = np.ascontiguousarray(y32, dtype=np.float32)
    xs = np.ascontiguousarray(x_scale, dtype=np.float32)
    ws = np.ascontiguousarray(w_scale, dtype=np.float32)
    out = np.empty(y.shape, dtype=np.uint16)
    _load().oracle_apply_scales_f32(_ptr(y), y.shape[0], y.shape[1], _ptr(xs), _ptr(ws), _ptr(out))
    return out


def fused_f32(Xq, x_scale, Wq_t, w_scale, rows=None) -> np.ndarray:
    """Fused path with fp32 epilogue arithmetic (no intermediate array)."""
    acc = gemm_acc64(Xq, Wq_t, rows)
    xs = np.ascontiguousarray(np.asarray(x_scale, dtype=np.float32)[
        slice(None) if rows is None else np.asarray(rows)])
    ws = np.ascontiguousarray(w_scale, dtype=np.float32)
    out = np.empty(acc.shape, dtype=np.uint16)
    _load().oracle_fused_epilogue_f32(_ptr(acc), acc.shape[0], acc.shape[1],
                                      _ptr(xs), _ptr(ws), _ptr(out))
    return out


# --------------------------------------------------------------------------
# Sub-byte weight formats (FP6 E3M2 / E2M3, FP4 E2M1)
# --------------------------------------------------------------------------
# Source: the llminfo.tech summary of "Running LLMs at custom floating-points
# (near-lossless FP6)" (FP4-FP7 weights with per-channel quantisation, the
# MX formats named as the likely standard) with the PTPC page's per-output-
# channel weight scale.  The readings are listed in ptpc_oracle.c.

FORMATS = {"e4m3": 0, "e2m1": 1, "e2m3": 2, "e3m2": 3}
FORMAT_BITS = {"e4m3": 8, "e2m1": 4, "e2m3": 6, "e3m2": 6}


def fmt_max(fmt: str) -> float:
    """Largest finite magnitude of a format."""
    return float(_load().oracle_fmt_max(FORMATS[fmt]))


def fmt_decode_table(fmt: str) -> np.ndarray:
    """fp64 value of every code of a format (2^bits entries, sign in the top bit)."""
    lib = _load()
    f = FORMATS[fmt]
    return np.array([lib.oracle_fmt_decode(c, f) for c in range(1 << FORMAT_BITS[fmt])], dtype=np.float64)


def fmt_encode(v, fmt: str) -> np.ndarray:
    """Saturating round-half-to-even codes of fp32 values in a format."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.empty(a.shape, dtype=np.uint8)
    _load().oracle_fmt_encode_array(_ptr(a), a.size, FORMATS[fmt], _ptr(out))
    return out


def quant_weight_fmt(W_bits: np.ndarray, fmt: str):
    """Per-output-channel quantisation of W (Ci x Co bf16 bits) to a format:
    (codes_t [Co, Ci] u8, one code per byte; w_scale [Co] f32 = amax / max)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    Ci, Co = W.shape
    codes = np.empty((Co, Ci), dtype=np.uint8)
    ws = np.empty((Co,), dtype=np.float32)
    _load().oracle_quant_weight_fmt(_ptr(W), Ci, Co, FORMATS[fmt], _ptr(codes), _ptr(ws))
    return codes, ws


def pack_fmt(codes: np.ndarray, fmt: str) -> np.ndarray:
    """Packs [rows, K] codes (one per byte) into the bytes the weight occupies
    in memory: [rows, K * bits / 8]."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, K = c.shape
    assert K % 16 == 0
    lib = _load()
    out = np.empty((rows, int(lib.oracle_packed_row_bytes(K, FORMATS[fmt]))), dtype=np.uint8)
    lib.oracle_pack_fmt(_ptr(c), rows, K, FORMATS[fmt], _ptr(out))
    return out


def gemm_acc64_fmt(Xq: np.ndarray, codes_t: np.ndarray, fmt: str, rows=None, col_chunk: int = 4096) -> np.ndarray:
    """acc[t, o] = sum_k dec_e4m3(Xq[t, k]) * dec_fmt(codes_t[o, k]) in fp64.

    Exact: E4M3 values are integer multiples of 2^-9 and the sub-byte formats'
    of 2^-4 or coarser, every product an integer multiple of 2^-13 below 2^14,
    so sums of up to 2^17 products stay below 2^44 units."""
    Ci = Xq.shape[1]
    assert codes_t.shape[1] == Ci and Ci <= MAX_EXACT_K
    A = e4m3_decode_table()[Xq if rows is None else Xq[np.asarray(rows)]]
    dec = fmt_decode_table(fmt)
    Co = codes_t.shape[0]
    acc = np.empty((A.shape[0], Co), dtype=np.float64)
    for o0 in range(0, Co, col_chunk):
        acc[:, o0:o0 + col_chunk] = A @ dec[codes_t[o0:o0 + col_chunk]].T
    return acc


def scaled_mm_reference_fmt(Xq, x_scale, codes_t, w_scale, fmt: str, rows=None) -> np.ndarray:
    """Tolerance reference of the scaled GEMM with format-f weights:
    bf16_RNE(x_scale[t] * w_scale[o] * acc[t, o]) in fp64 (bf16 bits)."""
    acc = gemm_acc64_fmt(Xq, codes_t, fmt, rows)
    xs = np.ascontiguousarray(np.asarray(x_scale, dtype=np.float32)[
        slice(None) if rows is None else np.asarray(rows)])
    ws = np.ascontiguousarray(w_scale, dtype=np.float32)
    out = np.empty(acc.shape, dtype=np.uint16)
    _load().oracle_reference_epilogue_f64(_ptr(acc), acc.shape[0], acc.shape[1], _ptr(xs), _ptr(ws), _ptr(out))
    return out


def linear_reference_fmt(X_bits, codes_t, w_scale, fmt: str, rows=None):
    """Per-token FP8 quantisation of X, then the scaled GEMM against format-f
    weights.  Returns (out bf16 bits, Xq, x_scale)."""
    Xq, xs = quant_act(X_bits)
    return scaled_mm_reference_fmt(Xq, xs, codes_t, w_scale, fmt, rows), Xq, xs


# --------------------------------------------------------------------------
# Row-split (tensor-parallel) activation quantisation
# --------------------------------------------------------------------------

def row_amax(X_bits: np.ndarray) -> np.ndarray:
    """max |x| of every row of a bf16 [T, Ci] slice (fp32, exact)."""
    X = np.ascontiguousarray(X_bits, dtype=np.uint16)
    out = np.empty((X.shape[0],), dtype=np.float32)
    _load().oracle_row_amax(_ptr(X), X.shape[0], X.shape[1], _ptr(out))
    return out


def quant_act_amax(X_bits: np.ndarray, amax: np.ndarray):
    """Per-token quantisation of a slice with given row maxima (the maxima of
    the whole rows, combined over the slices): (Xq [T, Ci], x_scale [T])."""
    X = np.ascontiguousarray(X_bits, dtype=np.uint16)
    a = np.ascontiguousarray(amax, dtype=np.float32)
    T, Ci = X.shape
    Xq = np.empty((T, Ci), dtype=np.uint8)
    xs = np.empty((T,), dtype=np.float32)
    _load().oracle_quant_act_amax(_ptr(X), T, Ci, _ptr(a), _ptr(Xq), _ptr(xs))
    return Xq, xs


def reference_epilogue(acc64: np.ndarray, x_scale, w_scale) -> np.ndarray:
    """bf16_RNE(x_scale[t] * w_scale[o] * acc[t, o]) in fp64 of a given fp64
    accumulator (the epilogue of scaled_mm_reference)."""
    acc = np.ascontiguousarray(acc64, dtype=np.float64)
    xs = np.ascontiguousarray(x_scale, dtype=np.float32)
    ws = np.ascontiguousarray(w_scale, dtype=np.float32)
    out = np.empty(acc.shape, dtype=np.uint16)
    _load().oracle_reference_epilogue_f64(_ptr(acc), acc.shape[0], acc.shape[1], _ptr(xs), _ptr(ws), _ptr(out))
    return out


# --------------------------------------------------------------------------
# FP8 (E4M3) KV cache and decode attention
# --------------------------------------------------------------------------
# Source: the PTPC page's evaluation commands, which run PTPC-FP8 with
# kv_cache_dtype=fp8_e4m3 (the KV cache stored in E4M3).  The page gives no
# scale rule; the reading here is the PTPC per-token rule applied to every
# (token, KV head) vector of D values: s = amax / 448, codes E4M3_satRNE(x/s)
# (quant_act on the rows of a [T * H, D] view).  The cache is paged: slot
# = block * block_size + offset, codes [num_blocks, block_size, H, D] u8,
# scales [num_blocks, block_size, H] f32.  Decode attention over it is the
# plain definition, in fp64: for query head h (KV head g = h // (Hq / Hkv)),
#   s_l = softmax_scale * sum_d q[h, d] * dec(K[l, g, d]) * k_scale[l, g],
#   p = softmax(s),  out[h, d] = sum_l p_l * dec(V[l, g, d]) * v_scale[l, g],
# rounded to bf16, over the positions l < context_len whose block-table entry
# exists (the table is wide enough), is not negative and lies inside the
# cache; the others are left out, and a sequence left with no position gets
# 0 (the softmax of an empty set is undefined: the library's reading, which
# its header states).

def kv_quantize(KV_bits: np.ndarray):
    """Per-(token, head) E4M3 quantisation of K or V, bf16 [T, H, D]:
    (codes [T, H, D] u8, scales [T, H] f32)."""
    T, H, D = KV_bits.shape
    q, s = quant_act(np.ascontiguousarray(KV_bits).reshape(T * H, D))
    return q.reshape(T, H, D), s.reshape(T, H)


def kv_cache_write(cache_codes, cache_scales, codes, scales, slots, block_size: int):
    """Scatter token rows into the paged cache (in place): token t goes to
    block slots[t] // block_size, offset slots[t] % block_size."""
    for t, slot in enumerate(np.asarray(slots)):
        b, o = divmod(int(slot), block_size)
        cache_codes[b, o] = codes[t]
        cache_scales[b, o] = scales[t]


def decode_attention_reference(q_bits, k_codes, k_scales, v_codes, v_scales, block_tables, context_lens,
                               block_size: int, softmax_scale: float) -> np.ndarray:
    """Decode attention over an E4M3 paged cache, fp64, rounded to bf16.
    q_bits bf16 [B, Hq, D]; returns bf16 bits [B, Hq, D].  Positions without
    a valid block are left out; no position left: the output is 0."""
    B, Hq, D = q_bits.shape
    num_blocks, Hkv = k_codes.shape[0], k_codes.shape[2]
    group = Hq // Hkv
    dec = e4m3_decode_table()
    q = bf16_to_float(q_bits).astype(np.float64)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        L = int(context_lens[b])
        table = np.asarray(block_tables[b])
        pos = np.arange(L)
        bi = pos // block_size
        blocks = np.where(bi < len(table), table[np.minimum(bi, len(table) - 1)], -1) if len(table) else -np.ones(L, int)
        keep = (blocks >= 0) & (blocks < num_blocks)
        if not keep.any():
            continue
        pos, blocks = pos[keep], blocks[keep]
        offs = pos % block_size
        K = dec[k_codes[blocks, offs]] * k_scales[blocks, offs][:, :, None].astype(np.float64)   # [L, Hkv, D]
        V = dec[v_codes[blocks, offs]] * v_scales[blocks, offs][:, :, None].astype(np.float64)
        for h in range(Hq):
            g = h // group
            s = softmax_scale * (K[:, g, :] @ q[b, h])
            p = np.exp(s - s.max())
            p /= p.sum()
            out[b, h] = p @ V[:, g, :]
    return bf16_from_double(out)
