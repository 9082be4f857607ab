"""PTPC-FP8 (per-token activation, per-channel weight FP8) for NVIDIA B200.

Thin Python binding of the C ABI declared in ``include/ptpc.h``; it only
marshals torch tensors (device memory and the current stream) into the
library calls.  Every step of the computation runs in the library's sm_100a
kernels; there is no CPU or PyTorch fallback, and importing this package
fails if ``_lib/libptpc.so`` has not been built
(``python fp8_quantized_gemm_ptpc_b200/build.py``).

Method: "PTPC-FP8: boosting vLLM performance on AMD ROCm" (vLLM blog),
sections "Per-Token Activation + Per-Channel Weight Quantization" and "The
challenge: two-step vs fused".
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libptpc.so")

# ptpc_status
OK = 0
ERR_INVALID_ARG = 1
ERR_MISALIGNED = 2
ERR_UNSUPPORTED_SHAPE = 3
ERR_WORKSPACE_TOO_SMALL = 4
ERR_UNSUPPORTED_DEVICE = 5
ERR_CUDA = 6
ERR_DEVICE_TIMEOUT = 7
ERR_NOT_IMPLEMENTED = 8

# ptpc_weight_format
WEIGHT_FORMATS = {"e4m3": 0, "e2m1": 1, "e2m3": 2, "e3m2": 3}
WEIGHT_BITS = {"e4m3": 8, "e2m1": 4, "e2m3": 6, "e3m2": 6}

# ptpc_op
OP_QUANTIZE_WEIGHTS = 1
OP_SCALED_MM = 2
OP_LINEAR = 3
OP_BENCH_PER_TENSOR = 4
OP_BENCH_UNSCALED_MM = 5

# Every symbol include/ptpc.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
SIGNATURES = {
    "ptpc_quantize_activations": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "ptpc_quantize_weights": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "ptpc_scaled_mm": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "ptpc_linear": (ctypes.c_int, [_P, _I64, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "ptpc_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _I64, _I64, _I64]),
    "ptpc_get_device_status": (ctypes.c_int, [_P, _P]),
    "ptpc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ptpc_gemm_ksplit": (ctypes.c_int, [_I64, _I64, _I64]),
    "ptpc_gemm_tail_split": (ctypes.c_int, [_I64, _I64, _I64, _SZ]),
    "ptpc_gemm_swap_tokens": (ctypes.c_int, [_I64, _I64, _I64, _SZ]),
    "ptpc_selftest_wait_timeout": (ctypes.c_int, [_P, _P]),
    "ptpc_scaled_mm_static_scratch": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "ptpc_static_scratch_status": (ctypes.c_int, [_P]),
    "ptpc_weight_bytes": (ctypes.c_size_t, [ctypes.c_int, _I64, _I64]),
    "ptpc_kv_cache_append": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "ptpc_decode_attention_workspace_size": (ctypes.c_size_t, [_I64, _I64, _I64, _I64]),
    "ptpc_decode_attention_kernel": (ctypes.c_int, [_I64, _I64, _I64, _I64]),
    "ptpc_decode_attention": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I64,
                                             _I64, _I64, ctypes.c_float, _P, _P, _SZ, _P]),
    "ptpc_act_row_amax": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P]),
    "ptpc_quantize_activations_amax": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P]),
    "ptpc_quantize_weights_fmt": (ctypes.c_int, [_P, _I64, _I64, ctypes.c_int, _P, _P, _P, _SZ, _P]),
    "ptpc_scaled_mm_fmt": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "ptpc_linear_fmt": (ctypes.c_int, [_P, _I64, _P, _P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "ptpc_reload_tuning_overrides": (ctypes.c_int, []),
    "ptpc_bench_map_cache_stats": (ctypes.c_int, [_P, _P]),
    "ptpc_bench_map_cache_selftest": (ctypes.c_int, []),
    "ptpc_bench_unscaled_mm_f32": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "ptpc_bench_apply_scales": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _P, _P]),
    "ptpc_bench_clock_probe": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64, _P, _P]),
    "ptpc_bench_quantize_activations_per_tensor": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "ptpc_bench_quantize_weights_per_tensor": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _SZ, _P]),
}


class PtpcError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python fp8_quantized_gemm_ptpc_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        try:
            fn = getattr(lib, name)
        except AttributeError as e:
            raise ImportError(f"{LIB_PATH} does not export {name}: it is older than the sources; rebuild it with "
                              "`python fp8_quantized_gemm_ptpc_b200/build.py`") from e
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.ptpc_status_string(int(status)).decode()


_size_cache: dict = {}


def _ws_need(op: int, T: int, Ci: int, Co: int, device: torch.device) -> int:
    """workspace_size for a call on `device`, remembered per shape (the size
    depends on the shape, the device and the tuning overrides only)."""
    key = (op, T, Ci, Co, device.index)
    n = _size_cache.get(key)
    if n is None:
        n = _size_cache[key] = workspace_size(op, T, Ci, Co)
    return n


def workspace_size(op: int, T: int, Ci: int, Co: int) -> int:
    return int(lib.ptpc_workspace_size(op, T, Ci, Co))


def gemm_ksplit(T: int, Ci: int, Co: int) -> int:
    """CTAs sharing each output tile for this shape on the current device
    (1: whole tiles; 2/4/8: K split over a cluster; 0: invalid)."""
    return int(lib.ptpc_gemm_ksplit(T, Ci, Co))


def gemm_tail_split(T: int, Ci: int, Co: int, ws_bytes: int | None = None) -> int:
    """CTA pairs sharing each tile of the prefill GEMM's split last wave for
    this shape (0: every tile whole), with ws_bytes of GEMM workspace
    (default: what ptpc_workspace_size asks for)."""
    if ws_bytes is None:
        ws_bytes = workspace_size(OP_SCALED_MM, T, Ci, Co)
    return int(lib.ptpc_gemm_tail_split(T, Ci, Co, ws_bytes))


def gemm_swap_tokens(T: int, Ci: int, Co: int, ws_bytes: int | None = None) -> int:
    """Tokens a tile holds when the prefill GEMM's plan for this shape swaps
    its operands (weights as the 256-row operand), 0 otherwise; ws_bytes of
    GEMM workspace (default: what ptpc_workspace_size asks for)."""
    if ws_bytes is None:
        ws_bytes = workspace_size(OP_SCALED_MM, T, Ci, Co)
    return int(lib.ptpc_gemm_swap_tokens(T, Ci, Co, ws_bytes))


def _check(fn: str, status: int):
    if status != OK:
        raise PtpcError(fn, status)


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device):
    """The device's current stream as an address (the argtypes take ints)."""
    if _raw_stream is not None:
        return _raw_stream(device.index if device.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: torch.Tensor):
    return t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def _need_rows(t: torch.Tensor, name: str) -> int:
    """A bf16 [rows, cols] tensor whose rows are contiguous (a dense tensor or
    a column slice of one); returns the row pitch in elements."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be torch.bfloat16, got {t.dtype}")
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be a 2-d tensor with contiguous rows")
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


class Workspace:
    """A zero-filled device buffer for the entry points that take (ws, ws_bytes).

    The library leaves its control words zero after every successful call, so
    one buffer serves any number of calls that do not overlap on the GPU.  A
    workspace belongs to one stream: the buffer is allocated (and zeroed) on
    the stream that is current when it is created or grown, and the caller
    must not use it on two streams at once."""

    def __init__(self, nbytes: int, device):
        self.device = torch.device(device)
        self.buf = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)

    @property
    def nbytes(self) -> int:
        return self.buf.numel()

    def ensure(self, nbytes: int) -> "Workspace":
        """Grow to at least nbytes.  The old buffer goes back to PyTorch's
        caching allocator, which hands it out again only to work ordered after
        what is already queued on the stream it was allocated on, so a kernel
        of that stream that still reads it is not overtaken."""
        if nbytes > self.nbytes:
            self.buf = torch.zeros(int(nbytes), dtype=torch.uint8, device=self.device)
        return self

    def ptr(self):
        return _ptr(self.buf)


_ws_lock = threading.Lock()
_ws_cache: dict = {}


def default_workspace(nbytes: int, device) -> Workspace:
    """The cached workspace of (device, current stream), grown on demand.

    Keyed by stream, not by host thread: calls on two streams get two
    workspaces and never share the quantised activations or the status word
    a ``linear`` call keeps there, while calls on one stream are ordered by
    that stream, which is what makes sharing one buffer between them safe."""
    dev = device if isinstance(device, torch.device) else torch.device(device)
    key = (dev, _stream(dev))
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None:
            with torch.cuda.stream(torch.cuda.current_stream(dev)):
                ws = _ws_cache[key] = Workspace(nbytes, dev)
        return ws.ensure(nbytes)


def release_default_workspaces(device=None) -> int:
    """Drop the cached default workspaces of one device (all devices when
    None) and return how many were dropped; the next call on a stream
    allocates a fresh one.  A prefill-sized ``linear`` keeps its quantised
    activations there (hundreds of MB at T = 8192), so a caller that is done
    with a stream, or with large shapes, can give that memory back.  Safe
    while work is still queued: each buffer returns to PyTorch's caching
    allocator, which reuses it only for later work of the stream it was
    allocated on."""
    if device is not None:
        device = torch.device(device)
        if device.type == "cuda" and device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
    with _ws_lock:
        keys = [k for k in _ws_cache if device is None or k[0] == device]
        for k in keys:
            del _ws_cache[k]
    return len(keys)


# ----------------------------------------------------------------- entry points

def quantize_activations(X: torch.Tensor, Xq: torch.Tensor | None = None, x_scale: torch.Tensor | None = None):
    """Per-token quantisation: X bf16 [T, Ci] (rows contiguous; a column slice
    is fine) -> (Xq uint8 [T, Ci], x_scale fp32 [T])."""
    ldx = _need_rows(X, "X")
    T, Ci = X.shape
    Xq = torch.empty((T, Ci), dtype=torch.uint8, device=X.device) if Xq is None else Xq
    x_scale = torch.empty((T,), dtype=torch.float32, device=X.device) if x_scale is None else x_scale
    _check("ptpc_quantize_activations",
           lib.ptpc_quantize_activations(_ptr(X), T, Ci, ldx, _ptr(Xq), _ptr(x_scale), _stream(X.device)))
    return Xq, x_scale


def row_amax(X: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 [T]: max |x| of every row of X bf16 [T, Ci] (rows contiguous)."""
    ldx = _need_rows(X, "X")
    T, Ci = X.shape
    out = torch.empty((T,), dtype=torch.float32, device=X.device) if out is None else out
    _check("ptpc_act_row_amax", lib.ptpc_act_row_amax(_ptr(X), T, Ci, ldx, _ptr(out), _stream(X.device)))
    return out


def quantize_activations_amax(X: torch.Tensor, amax: torch.Tensor, Xq: torch.Tensor | None = None,
                              x_scale: torch.Tensor | None = None):
    """Per-token quantisation of a row slice X [T, Ci] with the given row
    maxima (combined over the slices) -> (Xq uint8 [T, Ci], x_scale fp32 [T])."""
    ldx = _need_rows(X, "X")
    _need(amax, "amax", torch.float32, 1)
    T, Ci = X.shape
    Xq = torch.empty((T, Ci), dtype=torch.uint8, device=X.device) if Xq is None else Xq
    x_scale = torch.empty((T,), dtype=torch.float32, device=X.device) if x_scale is None else x_scale
    _check("ptpc_quantize_activations_amax",
           lib.ptpc_quantize_activations_amax(_ptr(X), T, Ci, ldx, _ptr(amax), _ptr(Xq), _ptr(x_scale),
                                              _stream(X.device)))
    return Xq, x_scale


def quantize_weights(W: torch.Tensor, ws: Workspace | None = None):
    """Per-output-channel quantisation: W bf16 [Ci, Co] -> (Wq_t uint8 [Co, Ci], w_scale fp32 [Co])."""
    _need(W, "W", torch.bfloat16, 2)
    Ci, Co = W.shape
    Wq_t = torch.empty((Co, Ci), dtype=torch.uint8, device=W.device)
    w_scale = torch.empty((Co,), dtype=torch.float32, device=W.device)
    need = workspace_size(OP_QUANTIZE_WEIGHTS, 0, Ci, Co)
    ws = default_workspace(need, W.device) if ws is None else ws.ensure(need)
    _check("ptpc_quantize_weights",
           lib.ptpc_quantize_weights(_ptr(W), Ci, Co, _ptr(Wq_t), _ptr(w_scale), ws.ptr(), ws.nbytes,
                                     _stream(W.device)))
    return Wq_t, w_scale


def _fmt(fmt: str) -> int:
    if fmt not in WEIGHT_FORMATS:
        raise ValueError(f"weight format must be one of {sorted(WEIGHT_FORMATS)}, got {fmt!r}")
    return WEIGHT_FORMATS[fmt]


def quantize_weights_fmt(W: torch.Tensor, fmt: str, ws: Workspace | None = None):
    """Per-output-channel quantisation of W bf16 [Ci, Co] to a weight format
    ('e4m3', 'e2m1', 'e2m3', 'e3m2') -> (Wq uint8 [Co, Ci * bits / 8] packed
    along Ci, w_scale fp32 [Co])."""
    _need(W, "W", torch.bfloat16, 2)
    Ci, Co = W.shape
    f = _fmt(fmt)
    nbytes = int(lib.ptpc_weight_bytes(f, Ci, Co))
    if nbytes == 0:
        raise ValueError(f"unsupported shape {Ci}x{Co} for weight format {fmt}")
    # 32-byte aligned rows: the caching allocator returns 512-byte aligned blocks
    Wq = torch.empty((Co, nbytes // Co), dtype=torch.uint8, device=W.device)
    w_scale = torch.empty((Co,), dtype=torch.float32, device=W.device)
    need = workspace_size(OP_QUANTIZE_WEIGHTS, 0, Ci, Co)
    ws = default_workspace(need, W.device) if ws is None else ws.ensure(need)
    _check("ptpc_quantize_weights_fmt",
           lib.ptpc_quantize_weights_fmt(_ptr(W), Ci, Co, f, _ptr(Wq), _ptr(w_scale), ws.ptr(), ws.nbytes,
                                         _stream(W.device)))
    return Wq, w_scale


def _packed_ci(Wq: torch.Tensor, fmt: str) -> int:
    return Wq.shape[1] * 8 // WEIGHT_BITS[fmt]


def scaled_mm_fmt(Xq, x_scale, Wq, w_scale, fmt: str, out: torch.Tensor | None = None, ws: Workspace | None = None):
    """Scaled GEMM against weights of a format (from quantize_weights_fmt)."""
    _need(Xq, "Xq", torch.uint8, 2)
    _need(Wq, "Wq", torch.uint8, 2)
    _need(x_scale, "x_scale", torch.float32, 1)
    _need(w_scale, "w_scale", torch.float32, 1)
    T, Ci = Xq.shape
    Co = Wq.shape[0]
    if _packed_ci(Wq, fmt) != Ci or x_scale.shape[0] != T or w_scale.shape[0] != Co:
        raise ValueError("shape mismatch")
    out = torch.empty((T, Co), dtype=torch.bfloat16, device=Xq.device) if out is None else out
    need = _ws_need(OP_SCALED_MM, T, Ci, Co, Xq.device)
    ws = default_workspace(need, Xq.device) if ws is None else ws.ensure(need)
    _check("ptpc_scaled_mm_fmt",
           lib.ptpc_scaled_mm_fmt(_ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), _fmt(fmt), T, Ci, Co,
                                  _ptr(out), ws.ptr(), ws.nbytes, _stream(Xq.device)))
    return out


def linear_fmt(X, Wq, w_scale, fmt: str, out: torch.Tensor | None = None, ws: Workspace | None = None):
    """Fused per-token FP8 quantisation + GEMM against weights of a format."""
    ldx = _need_rows(X, "X")
    _need(Wq, "Wq", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.float32, 1)
    T, Ci = X.shape
    Co = Wq.shape[0]
    if _packed_ci(Wq, fmt) != Ci or w_scale.shape[0] != Co:
        raise ValueError("shape mismatch")
    out = torch.empty((T, Co), dtype=torch.bfloat16, device=X.device) if out is None else out
    need = _ws_need(OP_LINEAR, T, Ci, Co, X.device)
    ws = default_workspace(need, X.device) if ws is None else ws.ensure(need)
    _check("ptpc_linear_fmt",
           lib.ptpc_linear_fmt(_ptr(X), ldx, _ptr(Wq), _ptr(w_scale), _fmt(fmt), T, Ci, Co, _ptr(out), ws.ptr(),
                               ws.nbytes, _stream(X.device)))
    return out


def scaled_mm(Xq, x_scale, Wq_t, w_scale, out: torch.Tensor | None = None, ws: Workspace | None = None):
    """Fused scaled GEMM: out bf16 [T, Co] = bf16((Xq . Wq_t^T) * x_scale[t] * w_scale[o])."""
    _need(Xq, "Xq", torch.uint8, 2)
    _need(Wq_t, "Wq_t", torch.uint8, 2)
    _need(x_scale, "x_scale", torch.float32, 1)
    _need(w_scale, "w_scale", torch.float32, 1)
    T, Ci = Xq.shape
    Co = Wq_t.shape[0]
    if Wq_t.shape[1] != Ci or x_scale.shape[0] != T or w_scale.shape[0] != Co:
        raise ValueError("shape mismatch")
    out = torch.empty((T, Co), dtype=torch.bfloat16, device=Xq.device) if out is None else out
    need = _ws_need(OP_SCALED_MM, T, Ci, Co, Xq.device)
    ws = default_workspace(need, Xq.device) if ws is None else ws.ensure(need)
    _check("ptpc_scaled_mm",
           lib.ptpc_scaled_mm(_ptr(Xq), _ptr(x_scale), _ptr(Wq_t), _ptr(w_scale), T, Ci, Co, _ptr(out),
                              ws.ptr(), ws.nbytes, _stream(Xq.device)))
    return out


def linear(X, Wq_t, w_scale, out: torch.Tensor | None = None, ws: Workspace | None = None):
    """Fused quantise + GEMM: X bf16 [T, Ci] (rows contiguous; a column slice
    is fine) -> out bf16 [T, Co]."""
    ldx = _need_rows(X, "X")
    _need(Wq_t, "Wq_t", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.float32, 1)
    T, Ci = X.shape
    Co = Wq_t.shape[0]
    if Wq_t.shape[1] != Ci or w_scale.shape[0] != Co:
        raise ValueError("shape mismatch")
    out = torch.empty((T, Co), dtype=torch.bfloat16, device=X.device) if out is None else out
    need = _ws_need(OP_LINEAR, T, Ci, Co, X.device)
    ws = default_workspace(need, X.device) if ws is None else ws.ensure(need)
    _check("ptpc_linear",
           lib.ptpc_linear(_ptr(X), ldx, _ptr(Wq_t), _ptr(w_scale), T, Ci, Co, _ptr(out), ws.ptr(), ws.nbytes,
                           _stream(X.device)))
    return out


def scaled_mm_static_scratch(Xq, x_scale, Wq_t, w_scale, out: torch.Tensor | None = None):
    """scaled_mm whose scratch is the library's own static device array (no
    workspace argument, nothing allocated by the library; ``out`` may be
    passed to avoid the output allocation here).  The array is 4 KiB per
    device, of which the GEMM uses its 256-byte status word; calls must not
    overlap on the GPU.  Timeouts are read with static_scratch_status()."""
    _need(Xq, "Xq", torch.uint8, 2)
    _need(Wq_t, "Wq_t", torch.uint8, 2)
    _need(x_scale, "x_scale", torch.float32, 1)
    _need(w_scale, "w_scale", torch.float32, 1)
    T, Ci = Xq.shape
    Co = Wq_t.shape[0]
    if Wq_t.shape[1] != Ci or x_scale.shape[0] != T or w_scale.shape[0] != Co:
        raise ValueError("shape mismatch")
    out = torch.empty((T, Co), dtype=torch.bfloat16, device=Xq.device) if out is None else out
    _check("ptpc_scaled_mm_static_scratch",
           lib.ptpc_scaled_mm_static_scratch(_ptr(Xq), _ptr(x_scale), _ptr(Wq_t), _ptr(w_scale), T, Ci, Co,
                                             _ptr(out), _stream(Xq.device)))
    return out


def static_scratch_status() -> int:
    """Synchronise the current stream and read/clear the status word of the
    static scratch array (timeouts of scaled_mm_static_scratch since the last
    read): OK or ERR_DEVICE_TIMEOUT."""
    return int(lib.ptpc_static_scratch_status(_stream(torch.device("cuda", torch.cuda.current_device()))))


def reload_tuning_overrides():
    """Re-read the PTPC_FORCE_* overrides from the environment (the library
    reads them once otherwise; tuning only).  Workspace sizes remembered by
    the binding are forgotten (a forced plan may need another size)."""
    _check("ptpc_reload_tuning_overrides", lib.ptpc_reload_tuning_overrides())
    _size_cache.clear()


def map_cache_stats():
    """(hits, misses) of the library's host-side tensor-map cache."""
    h, m = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check("ptpc_bench_map_cache_stats", lib.ptpc_bench_map_cache_stats(ctypes.byref(h), ctypes.byref(m)))
    return int(h.value), int(m.value)


def selftest_wait_timeout(ws: Workspace):
    """Launch the failure-path self-test on the current stream: a bounded
    wait that must run out (about 2 s) and set the workspace's status word."""
    _check("ptpc_selftest_wait_timeout", lib.ptpc_selftest_wait_timeout(ws.ptr(), _stream(ws.device)))


def device_status(ws: Workspace) -> int:
    """Synchronise the current stream and read/clear the workspace's device status word."""
    return int(lib.ptpc_get_device_status(ws.ptr(), _stream(ws.device)))


# ------------------------------------------------ measurement-only entry points

def unscaled_mm_f32(Xq, Wq_t, out: torch.Tensor | None = None, ws: Workspace | None = None):
    """Naive step 1: fp32 [T, Co] = Xq . Wq_t^T (no scales)."""
    _need(Xq, "Xq", torch.uint8, 2)
    _need(Wq_t, "Wq_t", torch.uint8, 2)
    T, Ci = Xq.shape
    Co = Wq_t.shape[0]
    out = torch.empty((T, Co), dtype=torch.float32, device=Xq.device) if out is None else out
    need = workspace_size(OP_BENCH_UNSCALED_MM, T, Ci, Co)
    ws = default_workspace(need, Xq.device) if ws is None else ws.ensure(need)
    _check("ptpc_bench_unscaled_mm_f32",
           lib.ptpc_bench_unscaled_mm_f32(_ptr(Xq), _ptr(Wq_t), T, Ci, Co, _ptr(out), ws.ptr(), ws.nbytes,
                                          _stream(Xq.device)))
    return out


def apply_scales(y, x_scale, w_scale, out: torch.Tensor | None = None):
    """Naive step 2: bf16((y * x_scale[t]) * w_scale[o])."""
    _need(y, "y", torch.float32, 2)
    T, Co = y.shape
    out = torch.empty((T, Co), dtype=torch.bfloat16, device=y.device) if out is None else out
    _check("ptpc_bench_apply_scales",
           lib.ptpc_bench_apply_scales(_ptr(y), _ptr(x_scale), _ptr(w_scale), T, Co, _ptr(out),
                                       _stream(y.device)))
    return out


class ClockProbe:
    """Effective SM clock over a measured region (measurement only).

    start(seconds) launches the library's clock probe on a side stream of the
    current device (one sleeping thread, no shared memory); after the region,
    mhz() synchronises the device and returns the median SM clock (MHz) over
    the probe's 1 ms intervals, or None if it recorded fewer than two."""

    def __init__(self, device, max_records: int = 16384):
        self.device = torch.device(device)
        self.records = torch.zeros((max_records, 2), dtype=torch.int64, device=self.device)
        self.count = torch.zeros((1,), dtype=torch.int32, device=self.device)
        self.stream = torch.cuda.Stream(self.device)

    def start(self, seconds: float, period_ns: int = 1_000_000):
        duration = int(max(0.0, min(seconds, 120.0)) * 1e9)
        n = int(min(self.records.shape[0], duration // period_ns + 2))
        _check("ptpc_bench_clock_probe",
               lib.ptpc_bench_clock_probe(_ptr(self.records), max(2, n), period_ns, duration, _ptr(self.count),
                                          ctypes.c_void_p(self.stream.cuda_stream)))

    def mhz(self):
        torch.cuda.synchronize(self.device)
        n = int(self.count.item())
        if n < 2:
            return None
        r = self.records[:n].cpu().numpy().astype("float64")
        dt = r[1:, 0] - r[:-1, 0]
        dc = r[1:, 1] - r[:-1, 1]
        ok = dt > 0
        if not ok.any():
            return None
        import numpy as np
        return float(np.median(dc[ok] / dt[ok] * 1e3))


def quantize_activations_per_tensor(X, Xq=None, x_scale=None, ws: Workspace | None = None):
    """Per-tensor quantisation of X; x_scale [T] holds the one tensor scale T times."""
    ldx = _need_rows(X, "X")
    T, Ci = X.shape
    Xq = torch.empty((T, Ci), dtype=torch.uint8, device=X.device) if Xq is None else Xq
    x_scale = torch.empty((T,), dtype=torch.float32, device=X.device) if x_scale is None else x_scale
    need = workspace_size(OP_BENCH_PER_TENSOR, T, Ci, 0)
    ws = default_workspace(need, X.device) if ws is None else ws.ensure(need)
    _check("ptpc_bench_quantize_activations_per_tensor",
           lib.ptpc_bench_quantize_activations_per_tensor(_ptr(X), T, Ci, ldx, _ptr(Xq), _ptr(x_scale), ws.ptr(),
                                                          ws.nbytes, _stream(X.device)))
    return Xq, x_scale


def quantize_weights_per_tensor(W, ws: Workspace | None = None):
    """Per-tensor quantisation of W; w_scale [Co] holds the one tensor scale Co times."""
    _need(W, "W", torch.bfloat16, 2)
    Ci, Co = W.shape
    Wq_t = torch.empty((Co, Ci), dtype=torch.uint8, device=W.device)
    w_scale = torch.empty((Co,), dtype=torch.float32, device=W.device)
    need = workspace_size(OP_QUANTIZE_WEIGHTS, 0, Ci, Co)
    ws = default_workspace(need, W.device) if ws is None else ws.ensure(need)
    _check("ptpc_bench_quantize_weights_per_tensor",
           lib.ptpc_bench_quantize_weights_per_tensor(_ptr(W), Ci, Co, _ptr(Wq_t), _ptr(w_scale), ws.ptr(),
                                                      ws.nbytes, _stream(W.device)))
    return Wq_t, w_scale


# ------------------------------------------------------------ FP8 KV cache

def kv_cache_append(K, V, slots, k_cache, v_cache, k_scale, v_scale):
    """Quantise K, V bf16 [T, H, D] per (token, head) to E4M3 and write them
    to their slots of the paged caches: k_cache / v_cache uint8
    [num_blocks, block_size, H, D], k_scale / v_scale fp32 [num_blocks,
    block_size, H]; slots int64 [T] (block * block_size + offset, -1 skips)."""
    _need(K, "K", torch.bfloat16, 3)
    _need(V, "V", torch.bfloat16, 3)
    _need(slots, "slots", torch.int64, 1)
    _need(k_cache, "k_cache", torch.uint8, 4)
    _need(v_cache, "v_cache", torch.uint8, 4)
    _need(k_scale, "k_scale", torch.float32, 3)
    _need(v_scale, "v_scale", torch.float32, 3)
    T, H, D = K.shape
    nb, bs = k_cache.shape[:2]
    if V.shape != K.shape or k_cache.shape != (nb, bs, H, D) or v_cache.shape != k_cache.shape or \
            k_scale.shape != (nb, bs, H) or v_scale.shape != k_scale.shape or slots.shape[0] != T:
        raise ValueError("shape mismatch")
    _check("ptpc_kv_cache_append",
           lib.ptpc_kv_cache_append(_ptr(K), _ptr(V), _ptr(slots), T, H, D, bs, nb, _ptr(k_cache), _ptr(v_cache),
                                    _ptr(k_scale), _ptr(v_scale), _stream(K.device)))


def decode_attention_kernel(Hq: int, Hkv: int, D: int, block_size: int) -> str:
    """The decode-attention kernel the library runs for this shape: "mma"
    (warp-level tensor-core tiles) or "tc" (tensor-memory MMAs)."""
    k = int(lib.ptpc_decode_attention_kernel(Hq, Hkv, D, block_size))
    if k == 0:
        raise ValueError("unsupported attention shape")
    return "tc" if k == 2 else "mma"


def decode_attention(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, max_context: int,
                     softmax_scale: float, out: torch.Tensor | None = None, ws: Workspace | None = None):
    """Decode attention over the FP8 paged cache: q bf16 [B, Hq, D],
    block_tables int32 [B, max_blocks], context_lens int32 [B] (each at most
    max_context) -> out bf16 [B, Hq, D]."""
    _need(q, "q", torch.bfloat16, 3)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    B, Hq, D = q.shape
    nb, bs, Hkv, _ = k_cache.shape
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device) if out is None else out
    need = int(lib.ptpc_decode_attention_workspace_size(B, Hq, D, max_context))
    ws = default_workspace(need, q.device) if ws is None else ws.ensure(need)
    _check("ptpc_decode_attention",
           lib.ptpc_decode_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                     _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv, D, bs, nb,
                                     block_tables.shape[1], max_context, float(softmax_scale), _ptr(out), ws.ptr(),
                                     ws.nbytes, _stream(q.device)))
    return out
