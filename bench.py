"""PTPC-FP8 benchmark: fused quantise + scaled-GEMM linear layers on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = the PTPC-FP8 forward of every linear layer of the workload on one
batch of synthetic activations already resident in HBM: per layer, the
per-token activation quantiser and the fused row-wise-scaled FP8 GEMM,
through the library's fused entry point ``ptpc_linear`` (weights are
quantised per output channel once, before timing, as at model load).  The
default workload is the largest single-GPU configuration, Llama-3.1-70B
prefill at T = 8192 (fused gate+up 8192->57344, down 28672->8192).

Prints one JSON line (rank 0).  ``value`` is whole-job TFLOP/s
(2 * T * Ci * Co summed over layers and ranks / the slowest rank's device
time).  The same line carries the GEMM's roofline record, the activation
quantiser inside the step and alone, the weight quantiser, the page's
comparison paths, the end-to-end figure through pinned host memory, the
decode regime (70B up/down at T = 1, 8, 32, 128), a short ragged-T chain
summary and the CPU oracle's throughput on a row sample.  With N > 1 every
rank runs an independent replica of the workload (weak scaling, no data-path
collective).  ``--impl reference`` times the CPU oracle on a bounded row
sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

WORKLOADS = {
    "llama8b_prefill": synthetic.LLAMA8B_PREFILL,
    "decode70b": synthetic.DECODE_70B,
    "llama70b_prefill": synthetic.LLAMA70B_PREFILL,
    "chain70b": synthetic.CHAIN_70B,
    "tiny": synthetic.TINY,
}
METRIC = "fused PTPC-FP8 GEMM TFLOP/s (% FP8 peak); quant GB/s (% HBM) on 1 B200"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama70b_prefill", choices=sorted(WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None, help="override T (default: the workload's first)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip comparison paths, e2e and CPU baseline")
    ap.add_argument("--cpu-rows", type=int, default=512,
                    help="token rows per layer in the CPU-oracle sample (0: all T rows)")
    ap.add_argument("--cpu-steps", type=int, default=2, help="steps in the CPU-oracle sample")
    ap.add_argument("--quant-only", action="store_true",
                    help="time only the per-token activation quantiser on the workload's inputs")
    ap.add_argument("--sweep", action="store_true",
                    help="70B 4-linear chain: fused vs naive two-step vs per-tensor, one JSON line per T")
    ap.add_argument("--sweep-tokens", default=None, help="comma-separated T values for --sweep")
    ap.add_argument("--chain-tokens", default="1,256,300,512,1000,3001",
                    help="T values of the chain summary inside the default line ('' to skip)")
    ap.add_argument("--tp", action="store_true",
                    help="tensor-parallel 70B MLP pair (column- then row-parallel) over the torchrun ranks")
    ap.add_argument("--no-kv", action="store_true", help="skip the FP8 KV-cache decode-attention record")
    ap.add_argument("--decode-tokens", default="1,8,32,128",
                    help="T values of the decode record inside the default line ('' to skip)")
    ap.add_argument("--weight-formats", default="e3m2,e2m1",
                    help="sub-byte weight formats of the decode_subbyte record")
    ap.add_argument("--record", default=None, choices=["decode", "decode_subbyte", "kv_decode", "kv_decode_405b", "kv_decode_long", "prefill_subbyte"],
                    help="print only this sub-record of the default line (a short run for profiling)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def dist_max(value: float, device=None) -> float:
    """Maximum of a per-rank value over all ranks of the default process group
    (the slowest rank's time decides a multi-GPU step)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of the same work
    (weak scaling); the job takes as long as its slowest rank."""
    return flops_per_rank_step * world * steps / (max_ms / 1e3) / 1e12


def workload_layers(wl, T):
    return [(i, L.name, T, L.Ci, L.Co) for i, L in enumerate(wl.layers)]


def layer_flops(layers):
    return sum(2.0 * T * Ci * Co for _, _, T, Ci, Co in layers)


def gemm_bytes(T, Ci, Co):
    """Algorithmic bytes of one fused GEMM launch: Xq, Wq_t, out, both scale vectors."""
    return T * Ci + Ci * Co + 2 * T * Co + 4 * (T + Co)


def quant_bytes(T, Ci):
    """Algorithmic bytes of one activation-quantiser launch: bf16 in, codes + scales out."""
    return 3 * T * Ci + 4 * T


def config_of(wl, layers, l2_note):
    return {
        "workload": wl.name + ": " + ", ".join(f"{n} {Ci}->{Co}" for _, n, _, Ci, Co in layers),
        "tokens": layers[0][2],
        "layers": [{"name": n, "T": T, "Ci": Ci, "Co": Co} for _, n, T, Ci, Co in layers],
        "weights": "bf16 N(0, sigma) quantised per output channel once, before timing",
        "l2": l2_note,
    }


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.power = [], set(), []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report clocks as unavailable
            self.nv = None

    _NAMES = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.power.append(nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self._NAMES.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_min_mhz": min(self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples),
                "power_w_median": statistics.median(self.power) if self.power else None,
                "power_w_max": max(self.power) if self.power else None}


# ----------------------------------------------------------------- reference (CPU oracle) arm

def sample_rows(T, n, seed=0):
    """Token rows of the CPU-oracle sample: all T rows if n >= T; otherwise
    the first and last row, both rows at every 128-row tile boundary, and a
    seeded uniform draw up to n rows in all, sorted."""
    if n <= 0 or n >= T:
        return np.arange(T)
    fixed = {0, T - 1}
    for b in range(128, T, 128):
        fixed.update((b - 1, b))
    fixed = sorted(fixed)
    if len(fixed) >= n:
        pick = np.linspace(0, len(fixed) - 1, n).round().astype(int)
        return np.unique(np.asarray(fixed)[pick])
    rng = np.random.Generator(np.random.PCG64(seed))
    rest = np.setdiff1d(np.arange(T), fixed)
    extra = rng.choice(rest, size=n - len(fixed), replace=False)
    return np.sort(np.concatenate([fixed, extra]))


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] + [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


def cpu_oracle_sample(wl, layers, rows_per_layer, steps, W_bits=None):
    """Times the oracle (as it stands) on a sample of token rows of every
    layer (sample_rows: first/last, every 128-row tile boundary, seeded
    draw): per-token quantisation of those rows and the fp64 scaled GEMM
    against the full weight, which the oracle quantises beforehand (not
    timed).  W_bits optionally passes the layers' bf16 weights already drawn.
    Returns (TFLOP/s, seconds, threads, note)."""
    import oracle
    prep = []
    for j, (i, name, T, Ci, Co) in enumerate(layers):
        rows = sample_rows(T, rows_per_layer, seed=10 + i)
        X = synthetic.make_x(wl, i, T, Ci)[rows]
        W = W_bits[j] if W_bits is not None else synthetic.make_w(wl, i, Ci, Co)
        Wq_t, ws = oracle.quant_weight(W)
        prep.append((np.ascontiguousarray(X), Wq_t, ws, len(rows), T, Ci, Co))
    flops = sum(2.0 * r * Ci * Co for _, _, _, r, _, Ci, Co in prep)
    t0 = time.perf_counter()
    for _ in range(steps):
        for X, Wq_t, ws, r, T, Ci, Co in prep:
            oracle.linear_reference(X, Wq_t, ws)
    dt = time.perf_counter() - t0
    sampled = all(r < T for _, _, _, r, T, _, _ in prep)
    note = (f"{prep[0][3]} of {prep[0][4]} token rows per layer (first/last, every 128-row tile boundary, seeded "
            f"draw) x {len(prep)} layers x {steps} steps: oracle per-token quantisation + fp64 GEMM against the "
            f"full weight; TFLOP/s of the sample"
            + ("; the oracle's time for a whole step is extrapolated from it (per row x T)" if sampled else ""))
    return flops * steps / dt / 1e12, dt, cpu_threads(), note


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    T = args.tokens or wl.tokens[0]
    layers = workload_layers(wl, T)
    rows = T if args.cpu_rows <= 0 else max(1, min(args.cpu_rows, T))
    W_bits = [synthetic.make_w(wl, i, Ci, Co) for i, _, _, Ci, Co in layers]
    if args.warmup > 0:
        cpu_oracle_sample(wl, layers, min(rows, 16), 1, W_bits)
    steps = max(1, min(args.steps, 3))
    tflops, dt, threads, note = cpu_oracle_sample(wl, layers, rows, steps, W_bits)
    flops = layer_flops(layers)
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
        "ms_per_step": flops / (tflops * 1e12) * 1e3,
        "ms_per_step_note": "whole step of the workload at the sample's rate (extrapolated per row x T)"
                            if rows < T else "measured",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, layers, "CPU run"),
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": note},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm

def traffic_record(kernel_src_hash, key):
    """DRAM bytes (read + write) of one step's GEMM launches for workload
    `key`, from the committed ncu summary, if that was taken on the current
    kernel source; None otherwise."""
    path = os.path.join(ROOT, "profiles", "gemm_dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_src_sha256") != kernel_src_hash:
        return None
    e = d.get("entries", {}).get(key)
    return None if e is None else e.get("dram_bytes_per_step")


def kernel_src_hash():
    h = hashlib.sha256()
    for f in ("gemm.cu", "sm100.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "fp8_quantized_gemm_ptpc_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def decode_record(ptpc, dev, peaks, tokens, steps):
    """The decode regime on its own: the 70B up (8192 -> 28672) and down
    (28672 -> 8192) layers through ptpc_linear at small T, weights quantised
    once.  Each layer's weight (235 MB of codes) is larger than L2, and the two
    alternate, so every weight byte comes from HBM on every call.  Reports
    the step time, the GEMM launches against the HBM roofline (algorithmic
    bytes: weight codes, activation codes, output, scales), the K split each
    layer runs with, and the host time per call (library and binding)."""
    import ctypes

    import torch
    wl = synthetic.DECODE_70B
    stream = torch.cuda.current_stream(dev)
    Ls = []
    for i, L in enumerate(wl.layers):
        Wb = torch.from_numpy(synthetic.make_w(wl, i, L.Ci, L.Co).view(np.int16)).to(dev).view(torch.bfloat16)
        Wq, ws = ptpc.quantize_weights(Wb)
        del Wb
        Ls.append((L, Wq, ws))
    out = {}
    for T in tokens:
        Xs = [torch.from_numpy(synthetic.make_x(wl, i, T, L.Ci).view(np.int16)).to(dev).view(torch.bfloat16)
              for i, (L, _, _) in enumerate(Ls)]
        outs = [torch.empty((T, L.Co), dtype=torch.bfloat16, device=dev) for L, _, _ in Ls]
        wsps = [ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, L.Ci, L.Co), dev) for L, _, _ in Ls]
        q = [(torch.empty((T, L.Ci), dtype=torch.uint8, device=dev), torch.empty((T,), dtype=torch.float32, device=dev))
             for L, _, _ in Ls]

        def step():
            for j, (L, Wq, ws) in enumerate(Ls):
                ptpc.linear(Xs[j], Wq, ws, out=outs[j], ws=wsps[j])

        for _ in range(3):
            step()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_step = e0.elapsed_time(e1) / steps
        # per launch: events around the quantiser and the GEMM of every layer
        ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in Ls] for _ in range(steps)]
        for it in range(steps):
            for j, (L, Wq, ws) in enumerate(Ls):
                ev[it][j][0].record(stream)
                ptpc.quantize_activations(Xs[j], *q[j])
                ev[it][j][1].record(stream)
                ptpc.scaled_mm(q[j][0], q[j][1], Wq, ws, out=outs[j], ws=wsps[j])
                ev[it][j][2].record(stream)
        torch.cuda.synchronize(dev)
        g_ms = [sum(ev[it][j][1].elapsed_time(ev[it][j][2]) for it in range(steps)) / steps for j in range(len(Ls))]
        q_ms = [sum(ev[it][j][0].elapsed_time(ev[it][j][1]) for it in range(steps)) / steps for j in range(len(Ls))]
        g_bytes = [gemm_bytes(T, L.Ci, L.Co) for L, _, _ in Ls]
        g_gbs = sum(g_bytes) / (sum(g_ms) / 1e3) / 1e9
        step_bytes = sum(g_bytes) + sum(quant_bytes(T, L.Ci) for L, _, _ in Ls)
        # host time per call: the C ABI through ctypes with arguments marshalled
        # once, and the Python binding (argument checks, stream lookup); the
        # GPU stays busy, so these are enqueue costs
        L0, Wq0, ws0 = Ls[0]
        P = ctypes.c_void_p
        args = (P(Xs[0].data_ptr()), L0.Ci, P(Wq0.data_ptr()), P(ws0.data_ptr()), T, L0.Ci, L0.Co,
                P(outs[0].data_ptr()), wsps[0].ptr(), wsps[0].nbytes, P(stream.cuda_stream))
        n_calls = 100
        h0, m0 = ptpc.map_cache_stats()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(n_calls):
            ptpc.lib.ptpc_linear(*args)
        t1 = time.perf_counter()
        torch.cuda.synchronize(dev)
        t2 = time.perf_counter()
        for _ in range(n_calls):
            ptpc.linear(Xs[0], Wq0, ws0, out=outs[0], ws=wsps[0])
        t3 = time.perf_counter()
        torch.cuda.synchronize(dev)
        h1, m1 = ptpc.map_cache_stats()
        out[str(T)] = {
            "ms_per_step": ms_step, "layers": [f"{L.name} {L.Ci}->{L.Co}" for L, _, _ in Ls],
            "gemm_ms": {L.name: g for (L, _, _), g in zip(Ls, g_ms)},
            "quant_ms": {L.name: x for (L, _, _), x in zip(Ls, q_ms)},
            "ksplit": {L.name: ptpc.gemm_ksplit(T, L.Ci, L.Co) for L, _, _ in Ls},
            "roofline": {"bound": "hbm", "achieved": g_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": g_gbs / peaks["hbm_gbs"], "algorithmic_bytes": sum(g_bytes),
                         "peak_src": f"{peaks['src']} HBM copy"},
            "step_gbs": step_bytes / (ms_step / 1e3) / 1e9,
            "step_frac_of_hbm": step_bytes / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"],
            "host_us_per_call_abi": (t1 - t0) / n_calls * 1e6,
            "host_us_per_call_binding": (t3 - t2) / n_calls * 1e6,
            "tensor_map_cache": {"hits": h1 - h0, "misses": m1 - m0},
        }
        del Xs, outs, wsps, q, ev
    del Ls
    torch.cuda.empty_cache()
    return {"workload": wl.name, "steps": steps,
            "l2": "each layer's weight (235 MB of codes) exceeds the 126 MB L2 and the layers alternate: "
                  "weights stream from HBM on every call",
            "per_T": out}


def decode_subbyte_record(ptpc, dev, peaks, tokens, steps, fmts=("e3m2", "e2m1")):
    """The 70B decode layers with FP6 (E3M2) and FP4 (E2M1) per-channel
    weights: the same step as the decode record (per-token FP8 activations
    quantised per call), the weights streaming 3/4 or 1/2 of the FP8 bytes.
    Reports per T the step time, the weight bytes a step streams and the
    GEMM launches against the HBM roofline on their algorithmic bytes."""
    import torch
    wl = synthetic.DECODE_70B
    stream = torch.cuda.current_stream(dev)
    res = {}
    for fmt in fmts:
        bits = ptpc.WEIGHT_BITS[fmt]
        Ls = []
        for i, L in enumerate(wl.layers):
            Wb = torch.from_numpy(synthetic.make_w(wl, i, L.Ci, L.Co).view(np.int16)).to(dev).view(torch.bfloat16)
            Wq, ws = ptpc.quantize_weights_fmt(Wb, fmt)
            del Wb
            Ls.append((L, Wq, ws))
        per_T = {}
        for T in tokens:
            Xs = [torch.from_numpy(synthetic.make_x(wl, i, T, L.Ci).view(np.int16)).to(dev).view(torch.bfloat16)
                  for i, (L, _, _) in enumerate(Ls)]
            outs = [torch.empty((T, L.Co), dtype=torch.bfloat16, device=dev) for L, _, _ in Ls]
            wsps = [ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, L.Ci, L.Co), dev) for L, _, _ in Ls]
            q = [(torch.empty((T, L.Ci), dtype=torch.uint8, device=dev),
                  torch.empty((T,), dtype=torch.float32, device=dev)) for L, _, _ in Ls]

            def step():
                for j, (L, Wq, ws) in enumerate(Ls):
                    ptpc.linear_fmt(Xs[j], Wq, ws, fmt, out=outs[j], ws=wsps[j])

            for _ in range(3):
                step()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record(stream)
            for _ in range(steps):
                step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms_step = e0.elapsed_time(e1) / steps
            ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in Ls] for _ in range(steps)]
            for j, (L, Wq, ws) in enumerate(Ls):
                ptpc.quantize_activations(Xs[j], *q[j])
            for it in range(steps):
                for j, (L, Wq, ws) in enumerate(Ls):
                    ev[it][j][0].record(stream)
                    ptpc.scaled_mm_fmt(q[j][0], q[j][1], Wq, ws, fmt, out=outs[j], ws=wsps[j])
                    ev[it][j][1].record(stream)
            torch.cuda.synchronize(dev)
            g_ms = [sum(ev[it][j][0].elapsed_time(ev[it][j][1]) for it in range(steps)) / steps
                    for j in range(len(Ls))]
            w_bytes = sum(L.Ci * L.Co * bits // 8 for L, _, _ in Ls)
            g_bytes = sum(L.Ci * L.Co * bits // 8 + T * L.Ci + 2 * T * L.Co + 4 * (T + L.Co) for L, _, _ in Ls)
            g_gbs = g_bytes / (sum(g_ms) / 1e3) / 1e9
            per_T[str(T)] = {
                "ms_per_step": ms_step, "weight_bytes_per_step": w_bytes,
                "weight_bytes_vs_fp8": w_bytes / sum(L.Ci * L.Co for L, _, _ in Ls),
                "gemm_ms": {L.name: g for (L, _, _), g in zip(Ls, g_ms)},
                "roofline": {"bound": "hbm", "achieved": g_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": g_gbs / peaks["hbm_gbs"], "algorithmic_bytes": g_bytes},
            }
            del Xs, outs, wsps, q, ev
        res[fmt] = per_T
        del Ls
        torch.cuda.empty_cache()
    return {"workload": wl.name + ", sub-byte per-channel weights, FP8 per-token activations", "steps": steps,
            "per_format": res}


def prefill_subbyte_record(ptpc, dev, peaks, steps, fmts=("e3m2", "e2m1"), T=8192):
    """The 70B prefill layers (gate+up 8192 -> 57344, down 28672 -> 8192) at
    T = 8192 with FP6 (E3M2) and FP4 (E2M1) per-channel weights: the same
    step as the default line (per-token FP8 activations quantised per call)
    through ptpc_linear_fmt.  The mixed-format MMA runs at the FP8 rate, so
    the roofline is the same burst FP8 figure."""
    import torch
    wl = synthetic.LLAMA70B_PREFILL
    stream = torch.cuda.current_stream(dev)
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    flops = sum(2.0 * T * L.Ci * L.Co for L in wl.layers)
    Xs = [torch.from_numpy(synthetic.make_x(wl, i, T, L.Ci).view(np.int16)).to(dev).view(torch.bfloat16)
          for i, L in enumerate(wl.layers)]
    outs = [torch.empty((T, L.Co), dtype=torch.bfloat16, device=dev) for L in wl.layers]
    wsps = [ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, L.Ci, L.Co), dev) for L in wl.layers]
    res = {}
    for fmt in fmts:
        Ws = []
        for i, L in enumerate(wl.layers):
            Wb = torch.from_numpy(synthetic.make_w(wl, i, L.Ci, L.Co).view(np.int16)).to(dev).view(torch.bfloat16)
            Ws.append(ptpc.quantize_weights_fmt(Wb, fmt))
            del Wb

        def step():
            for j, (Wq, ws) in enumerate(Ws):
                ptpc.linear_fmt(Xs[j], Wq, ws, fmt, out=outs[j], ws=wsps[j])

        for _ in range(3):
            step()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / steps
        tf = flops / (ms / 1e3) / 1e12
        res[fmt] = {"ms_per_step": ms, "tflops": tf, "frac_of_fp8_peak": tf / fp8_peak,
                    "weight_bytes_vs_fp8": ptpc.WEIGHT_BITS[fmt] / 8}
        del Ws
        torch.cuda.empty_cache()
    del Xs, outs, wsps
    torch.cuda.empty_cache()
    return {"workload": f"Llama-3.1-70B prefill T={T} (gate+up, down), sub-byte per-channel weights", "steps": steps,
            "peak": fp8_peak, "unit": "TFLOP/s", "note": "step TFLOP/s (quantiser + GEMM launches)",
            "per_format": res}


def kv_decode_record(ptpc, dev, peaks, B=32, ctx=4096, Hq=64, Hkv=8, D=128, bs=16, steps=50, model="Llama-3.1-70B"):
    """Decode attention of a Llama-3.1-70B-shaped layer (64 query heads on 8
    KV heads, D = 128; Llama-3.1-405B: 128 query heads) over the FP8 paged cache: B sequences of ctx cached
    positions, blocks of bs positions in a shuffled order.  Algorithmic bytes
    per step: the codes of K and V, their scales, q and the output.  Also
    times appending one new token per sequence (the decode step's write): on
    the device (a CUDA graph of the calls replayed) and called from Python."""
    import math

    import torch
    rng = np.random.Generator(np.random.PCG64(1234))
    nblk = B * ctx // bs
    tables = rng.permutation(nblk).astype(np.int32).reshape(B, ctx // bs)
    kc = torch.empty((nblk, bs, Hkv, D), dtype=torch.uint8, device=dev)
    vc = torch.empty_like(kc)
    ksc = torch.empty((nblk, bs, Hkv), dtype=torch.float32, device=dev)
    vsc = torch.empty_like(ksc)
    # fill the cache through the append kernel, one chunk of tokens at a time
    slots_all = (tables[:, :, None] * bs + np.arange(bs)[None, None, :]).reshape(-1)
    g = torch.Generator(device=dev)
    g.manual_seed(99)
    for c0 in range(0, slots_all.size, 65536):
        sl = torch.from_numpy(slots_all[c0:c0 + 65536].astype(np.int64)).to(dev)
        K = torch.randn((sl.numel(), Hkv, D), device=dev, generator=g).to(torch.bfloat16)
        V = torch.randn((sl.numel(), Hkv, D), device=dev, generator=g).to(torch.bfloat16)
        ptpc.kv_cache_append(K, V, sl, kc, vc, ksc, vsc)
        del K, V
    q = torch.randn((B, Hq, D), device=dev, generator=g).to(torch.bfloat16)
    bt = torch.from_numpy(tables).to(dev)
    lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
    ws = ptpc.Workspace(int(ptpc.lib.ptpc_decode_attention_workspace_size(B, Hq, D, ctx)), dev)
    stream = torch.cuda.current_stream(dev)
    fn = lambda: ptpc.decode_attention(q, kc, vc, ksc, vsc, bt, lens, ctx, 1 / math.sqrt(D), out=out, ws=ws)
    for _ in range(3):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    nbytes = B * ctx * Hkv * (2 * D + 8) + 2 * (2 * B * Hq * D)
    # one new token per sequence: the decode step's cache write.  Called from
    # Python back to back the loop is bound by the binding's host time; the
    # device time comes from a CUDA graph of the same calls replayed.
    Kn = torch.randn((B, Hkv, D), device=dev, generator=g).to(torch.bfloat16)
    sl = torch.from_numpy(slots_all[:B].astype(np.int64)).to(dev)
    for _ in range(3):
        ptpc.kv_cache_append(Kn, Kn, sl, kc, vc, ksc, vsc)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        ptpc.kv_cache_append(Kn, Kn, sl, kc, vc, ksc, vsc)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_app_host = e0.elapsed_time(e1) / steps
    n_graph = 20
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(n_graph):
            ptpc.kv_cache_append(Kn, Kn, sl, kc, vc, ksc, vsc)
    graph.replay()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(5):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_app = e0.elapsed_time(e1) / (5 * n_graph)
    del graph
    gbs = nbytes / (ms / 1e3) / 1e9
    rec = {
        "workload": f"{model} decode attention: {B} sequences x {ctx} cached positions, {Hq} query / "
                    f"{Hkv} KV heads, D = {D}, {bs}-position blocks (shuffled), E4M3 codes + per-(token, head) scales",
        "kernel": ptpc.decode_attention_kernel(Hq, Hkv, D, bs),
        "ms_per_step": ms, "algorithmic_bytes": nbytes,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "peak_src": f"{peaks['src']} HBM copy"},
        "bf16_cache_bytes_would_be": B * ctx * Hkv * 2 * D * 2,
        "append_one_token_per_sequence_us": ms_app * 1e3,
        "append_one_token_per_sequence_us_called_from_python": ms_app_host * 1e3,
    }
    del kc, vc, ksc, vsc, q, out, ws
    torch.cuda.empty_cache()
    return rec


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import fp8_quantized_gemm_ptpc_b200 as ptpc

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    wl = WORKLOADS[args.workload]
    T = args.tokens or wl.tokens[0]
    layers = workload_layers(wl, T)
    peaks = load_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops"]                 # nominal fp8:bf16 ratio 2
    fp8_peak_sus = 2.0 * peaks["bf16_tflops_sustained"]
    cpu_baseline_here = rank == 0 and world == 1 and not args.no_extras

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    # inputs, resident in HBM; weights quantised once (model load)
    L = []
    W_bits = []
    for i, name, T_, Ci, Co in layers:
        X = to_dev(synthetic.make_x(wl, i, T_, Ci))
        wb = synthetic.make_w(wl, i, Ci, Co)
        if cpu_baseline_here:
            W_bits.append(wb)
        Wb = to_dev(wb)
        del wb
        Wq_t, w_scale = ptpc.quantize_weights(Wb)
        Wq_pt, ws_pt = ptpc.quantize_weights_per_tensor(Wb)
        out = torch.empty((T_, Co), dtype=torch.bfloat16, device=dev)
        wsp = ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T_, Ci, Co), dev)
        L.append(dict(name=name, T=T_, Ci=Ci, Co=Co, X=X, W=Wb, Wq_t=Wq_t, ws=w_scale, Wq_pt=Wq_pt, ws_pt=ws_pt,
                      out=out, wsp=wsp))
    torch.cuda.synchronize(dev)
    working_set = sum(d["X"].numel() * 2 + d["Wq_t"].numel() + d["out"].numel() * 2 for d in L)
    l2_note = (f"inputs larger than L2: {working_set / 1e6:.0f} MB touched per step > 126 MB L2, no flush"
               if working_set > L2_BYTES else
               f"working set {working_set / 1e6:.1f} MB fits in L2 (no flush)")

    def step():
        for d in L:
            ptpc.linear(d["X"], d["Wq_t"], d["ws"], out=d["out"], ws=d["wsp"])

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    def max_over_ranks(v):
        return dist_max(v, dev)

    def timed(fn, steps, before=None):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier()
        if before is not None:
            before()
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        barrier()
        return e0.elapsed_time(e1)

    K, W = args.steps, max(3, args.warmup)
    # ---- the activation quantiser alone on the step's inputs, measured
    # before any GEMM has run (a kernel timed alone: burst conditions; every
    # input is larger than L2, so each pass reads X from HBM)
    bufs = [(torch.empty((d["T"], d["Ci"]), dtype=torch.uint8, device=dev),
             torch.empty((d["T"],), dtype=torch.float32, device=dev)) for d in L]
    q_bytes = sum(quant_bytes(d["T"], d["Ci"]) for d in L)
    Kq = max(10, min(4 * K, 200))
    qfn = lambda: [ptpc.quantize_activations(d["X"], *bufs[j]) for j, d in enumerate(L)]
    for _ in range(3):
        qfn()
    ms_q = max_over_ranks(timed(qfn, Kq)) / Kq
    qprobe = ptpc.ClockProbe(dev)
    timed(qfn, Kq, before=lambda: qprobe.start(ms_q * Kq * 1.05 / 1e3))
    q_alone = q_bytes / (ms_q / 1e3) / 1e9
    quant_isolated = {
        "value": q_alone, "unit": "GB/s", "achieved": q_alone, "peak": peaks["hbm_gbs"],
        "frac": q_alone / peaks["hbm_gbs"], "bytes_per_pass": q_bytes, "ms_per_pass": ms_q, "passes": Kq,
        "inputs": [[d["T"], d["Ci"]] for d in L], "sm_mhz_device": qprobe.mhz(),
        "peak_src": f"{peaks['src']} HBM copy",
        "note": "ptpc_quantize_activations alone, every layer input of the step in turn, back to back, "
                "before the GEMM loops; algorithmic bytes 3 per element + 4 per row",
    }

    for _ in range(W):
        step()
    with ClockSampler(local) as clk:
        ms = timed(step, K)
    # ---- per-kernel device times, right after the timed loop: the same
    # launches as ptpc_linear (quantiser, then GEMM) through the two separate
    # entry points, with events on the launch stream around each launch and no
    # host synchronisation inside the loop
    Kk = max(10, min(K, 200))
    for _ in range(3):
        for j, d in enumerate(L):
            ptpc.quantize_activations(d["X"], *bufs[j])
            ptpc.scaled_mm(bufs[j][0], bufs[j][1], d["Wq_t"], d["ws"], out=d["out"], ws=d["wsp"])
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in L] for _ in range(Kk)]
    barrier()
    for it in range(Kk):
        for j, d in enumerate(L):
            e = evs[it][j]
            e[0].record(stream)
            ptpc.quantize_activations(d["X"], *bufs[j])
            e[1].record(stream)
            ptpc.scaled_mm(bufs[j][0], bufs[j][1], d["Wq_t"], d["ws"], out=d["out"], ws=d["wsp"])
            e[2].record(stream)
    barrier()
    q_ms = [sum(evs[it][j][0].elapsed_time(evs[it][j][1]) for it in range(Kk)) / Kk for j in range(len(L))]
    g_ms = [sum(evs[it][j][1].elapsed_time(evs[it][j][2]) for it in range(Kk)) / Kk for j in range(len(L))]
    # The SM clock seen by the device over the same loop, repeated: the clock
    # probe runs beside it on a side stream (kept out of the timed region
    # above, which it could perturb).
    probe = ptpc.ClockProbe(dev)
    ms_probe = timed(step, K, before=lambda: probe.start(ms * 1.05 / 1e3))
    probe_mhz = probe.mhz()
    ms = max_over_ranks(ms)
    flops = layer_flops(layers)
    value = whole_job_tflops(flops, world, K, ms)
    launches = K * 2 * len(L)

    # The GEMM's time inside the timed steps: the step's device time less its
    # quantiser launches (launch gaps stay charged to the GEMM, so this is an
    # upper bound on its launch durations and `achieved` a lower bound).
    gemm_step_ms = ms / K - sum(q_ms)
    gemm_tflops = flops / (gemm_step_ms / 1e3) / 1e12
    g_bytes = sum(gemm_bytes(d["T"], d["Ci"], d["Co"]) for d in L)
    gemm_gbs = g_bytes / (gemm_step_ms / 1e3) / 1e9
    loop_tflops = flops / (sum(g_ms) / 1e3) / 1e12
    ridge = fp8_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)      # FLOP per byte
    hbm_bound = flops / g_bytes < ridge
    q_gbs = q_bytes / (sum(q_ms) / 1e3) / 1e9
    dram = traffic_record(kernel_src_hash(), f"{args.workload}:T={T}")

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e4m3 -> f32 accumulate, bf16 out", "data": "synthetic",
        "config": dict(config_of(wl, layers, l2_note), parallelism=f"replicas x{world}" if world > 1 else "1 GPU"),
        "frac_of_fp8_peak": value / world / fp8_peak,
        "clocks": clk.summary() | {"sm_mhz_device": probe_mhz,
                                   "sm_mhz_device_src": "median over 1 ms intervals of clock64 / globaltimer on "
                                                        "one SM, during a repeat of the timed loop",
                                   "repeat_ms_per_step": ms_probe / K},
        "gpu_launches": launches,
        "roofline": ({
            "bound": "hbm", "achieved": gemm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gemm_gbs / peaks["hbm_gbs"], "traffic": dram,
            "peak_src": f"{peaks['src']} HBM copy",
        } if hbm_bound else {
            # the timed loop lasts milliseconds, not seconds: the burst FP8
            # figure is the denominator; the sustained one is reported beside it
            "bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
            "frac": gemm_tflops / fp8_peak, "traffic": dram,
            "peak_src": f"{peaks['src']} bf16 burst x 2 (fp8:bf16 nominal ratio 4.5 : 2.25 PFLOP/s)",
            "sustained_peak": fp8_peak_sus, "frac_of_sustained": gemm_tflops / fp8_peak_sus,
        }) | {
            "kernel": "ptpc scaled GEMM (fused epilogue), all layers of one step",
            "traffic_unit": "bytes per step (dram__bytes_read.sum + dram__bytes_write.sum over the step's GEMM launches)",
            "algorithmic_flops_per_step": flops, "algorithmic_bytes_per_step": g_bytes,
            "gemm_tflops": gemm_tflops, "gemm_gbs": gemm_gbs, "gemm_ms_per_step": gemm_step_ms,
            "achieved_src": "algorithmic FLOPs / (timed step device time - its quantiser launches, "
                            "the latter timed by events in a loop of the same launches right after)",
            "per_launch_loop": {
                "tflops": loop_tflops, "ms_per_step": sum(g_ms),
                "per_layer_ms": {d["name"]: g for d, g in zip(L, g_ms)},
                "note": "events around each GEMM launch in that loop; it runs later than the timed "
                        "steps, so at the lower clock that the power cap has reached by then"},
            "sm_mhz_device": probe_mhz,
        },
        "quant_isolated": quant_isolated,
        "quant": {
            "value": q_gbs, "unit": "GB/s", "peak": peaks["hbm_gbs"], "frac": q_gbs / peaks["hbm_gbs"],
            "bytes_per_step": q_bytes, "per_layer_ms": {d["name"]: q for d, q in zip(L, q_ms)},
            "peak_src": f"{peaks['src']} HBM copy",
            "note": "inside the step: each launch timed by events between the GEMMs (launch gap included), "
                    "at the clock the GEMMs' power draw leaves",
        },
    }

    # ---- per-output-channel weight quantiser (run once per weight at load time)
    wq_ms = []
    for d in L:
        Wb = d.pop("W")
        wsq = ptpc.Workspace(ptpc.workspace_size(ptpc.OP_QUANTIZE_WEIGHTS, 0, d["Ci"], d["Co"]), dev)
        for _ in range(2):
            ptpc.quantize_weights(Wb, ws=wsq)
        n_it = 5
        wq_ms.append(max_over_ranks(timed(lambda: ptpc.quantize_weights(Wb, ws=wsq), n_it)) / n_it)
        del Wb
    wq_elems = sum(d["Ci"] * d["Co"] for d in L)
    wq_bytes = sum(3 * d["Ci"] * d["Co"] + 4 * d["Co"] for d in L)
    line["quant_weights"] = {
        "value": wq_bytes / (sum(wq_ms) / 1e3) / 1e9, "unit": "GB/s", "peak": peaks["hbm_gbs"],
        "frac": wq_bytes / (sum(wq_ms) / 1e3) / 1e9 / peaks["hbm_gbs"],
        "algorithmic_bytes": wq_bytes, "kernel_bytes": 5 * wq_elems + 8 * sum(d["Co"] for d in L),
        "per_layer_ms": {d["name"]: t for d, t in zip(L, wq_ms)},
        "note": "one-time, at weight load; the kernel reads W twice (column maxima, then codes)",
    }

    if not args.no_extras:
        # ---- comparison paths of the page: naive two-step and per-tensor scaling
        ys = [torch.empty((d["T"], d["Co"]), dtype=torch.float32, device=dev) for d in L]
        pt_ws = [ptpc.Workspace(ptpc.workspace_size(ptpc.OP_BENCH_PER_TENSOR, d["T"], d["Ci"], 0), dev) for d in L]

        def naive():
            for j, d in enumerate(L):
                ptpc.quantize_activations(d["X"], *bufs[j])
                ptpc.unscaled_mm_f32(bufs[j][0], d["Wq_t"], out=ys[j], ws=d["wsp"])
                ptpc.apply_scales(ys[j], bufs[j][1], d["ws"], out=d["out"])

        def per_tensor():
            for j, d in enumerate(L):
                ptpc.quantize_activations_per_tensor(d["X"], *bufs[j], ws=pt_ws[j])
                ptpc.scaled_mm(bufs[j][0], bufs[j][1], d["Wq_pt"], d["ws_pt"], out=d["out"], ws=d["wsp"])

        Kc = max(5, min(K, 100))
        for fn in (naive, per_tensor):
            for _ in range(3):
                fn()
        ms_naive = max_over_ranks(timed(naive, Kc)) / Kc
        ms_pt = max_over_ranks(timed(per_tensor, Kc)) / Kc
        ms_sep = sum(q_ms) + sum(g_ms)
        line["paths"] = {
            "fused_ptpc_linear_ms": ms / K,
            "quantize_then_scaled_mm_ms": ms_sep,
            "naive_two_step_ms": ms_naive,
            "per_tensor_ms": ms_pt,
            "fused_speedup_over_naive": ms_naive / (ms / K),
            "ptpc_over_per_tensor_throughput": ms_pt / (ms / K),
        }
        del ys
        for d in L:
            d.pop("Wq_pt")
            d.pop("ws_pt")
        torch.cuda.empty_cache()

        # ---- end to end through the public API: pinned host in, pinned host out.
        # Every step copies each layer's input host -> device, runs ptpc.linear
        # and copies the output device -> host.  The copies run on their own
        # streams (one per direction: the two copy engines and the SMs work at
        # the same time), ordered against the compute by events; device
        # buffers alternate between two sets so that a step's copies overlap
        # the previous step's compute.
        hx = [d["X"].cpu().pin_memory() for d in L]
        ho = [torch.empty((d["T"], d["Co"]), dtype=torch.bfloat16).pin_memory() for d in L]
        nb = 2
        dx = [[torch.empty_like(d["X"]) for d in L] for _ in range(nb)]
        dout = [[torch.empty_like(d["out"]) for d in L] for _ in range(nb)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [[torch.cuda.Event() for _ in L] for _ in range(nb)]    # input copied
        ev_done = [[torch.cuda.Event() for _ in L] for _ in range(nb)]  # linear finished
        ev_out = [[torch.cuda.Event() for _ in L] for _ in range(nb)]   # output copied
        used = [[False] * len(L) for _ in range(nb)]
        it = [0]

        def e2e_step():
            b = it[0] % nb
            it[0] += 1
            for j, d in enumerate(L):
                if used[b][j]:
                    s_in.wait_event(ev_done[b][j])      # dx[b][j] no longer read
                with torch.cuda.stream(s_in):
                    dx[b][j].copy_(hx[j], non_blocking=True)
                ev_in[b][j].record(s_in)
                stream.wait_event(ev_in[b][j])
                if used[b][j]:
                    stream.wait_event(ev_out[b][j])     # dout[b][j] already copied out
                ptpc.linear(dx[b][j], d["Wq_t"], d["ws"], out=dout[b][j], ws=d["wsp"])
                ev_done[b][j].record(stream)
                s_out.wait_event(ev_done[b][j])
                with torch.cuda.stream(s_out):
                    ho[j].copy_(dout[b][j], non_blocking=True)
                ev_out[b][j].record(s_out)
                used[b][j] = True

        def e2e_timed(steps):
            torch.cuda.synchronize(dev)
            barrier()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            s_in.wait_event(e0)
            for _ in range(steps):
                e2e_step()
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            return e0.elapsed_time(e1)

        Ke = max(5, min(K, 30))
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks(e2e_timed(Ke)) / Ke
        # the pipelined path computes what the device-resident fused step computes
        for j, d in enumerate(L):
            ref = ptpc.linear(d["X"], d["Wq_t"], d["ws"], ws=d["wsp"])
            if not torch.equal(ho[j].view(torch.int16), ref.cpu().view(torch.int16)):
                raise RuntimeError(f"end-to-end output of layer {d['name']} differs from the device path")
            del ref
        line["e2e"] = {
            "value": flops * world / (ms_e2e / 1e3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(sum(h.numel() * 2 for h in hx)),
            "d2h_bytes_per_step": int(sum(h.numel() * 2 for h in ho)),
            "ms_per_step": ms_e2e,
            "pipelining": "per-direction copy streams, two device buffer sets",
        }
        del hx, ho, dx, dout

    # the step's own buffers are no longer needed
    del L, bufs, evs
    torch.cuda.empty_cache()

    if not args.no_extras:
        # ---- the decode regime and a short ragged-T chain summary
        dec_tokens = [int(t) for t in args.decode_tokens.split(",") if t.strip()]
        if dec_tokens:
            line["decode"] = decode_record(ptpc, dev, peaks, dec_tokens, steps=max(20, min(K * 2, 100)))
            line["decode_subbyte"] = decode_subbyte_record(ptpc, dev, peaks, [t for t in dec_tokens if t in (1, 128)]
                                                           or dec_tokens[:1], steps=max(20, min(K * 2, 100)))
        if not args.no_kv:
            line["kv_decode"] = kv_decode_record(ptpc, dev, peaks)
            line["kv_decode_long"] = kv_decode_record(ptpc, dev, peaks, ctx=32768, steps=10)
        line["prefill_subbyte"] = prefill_subbyte_record(ptpc, dev, peaks, steps=max(5, min(K, 20)))
        chain_tokens = [int(t) for t in args.chain_tokens.split(",") if t.strip()]
        if chain_tokens:
            Ws = chain_weights(ptpc, dev)
            line["chain"] = {
                "workload": synthetic.CHAIN_70B.name + ": qkv 8192->10240, o 8192->8192, gate_up 8192->57344, "
                                                       "down 28672->8192, dynamic re-quantisation between layers",
                "per_T": [chain_measure(ptpc, dev, Ws, t, peaks, graph=False) for t in chain_tokens],
                "roofline_note": "roofline_ms = max(algorithmic FLOPs / burst FP8 peak, algorithmic bytes of "
                                 "quantisers and GEMMs / HBM copy bandwidth)",
            }
            del Ws
            torch.cuda.empty_cache()

        if cpu_baseline_here:
            rows = T if args.cpu_rows <= 0 else max(1, min(args.cpu_rows, T))
            tf, dt, threads, note = cpu_oracle_sample(wl, layers, rows, max(1, args.cpu_steps), W_bits)
            line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": note, "seconds": dt}
    del W_bits

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def run_quant_only(args):
    """Times ptpc_quantize_activations alone on every layer input of the
    workload (no weights are generated)."""
    import torch

    import fp8_quantized_gemm_ptpc_b200 as ptpc

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    wl = WORKLOADS[args.workload]
    T = args.tokens or wl.tokens[0]
    layers = workload_layers(wl, T)
    peaks = load_peaks()
    bufs = []
    for i, name, T_, Ci, Co in layers:
        X = torch.from_numpy(synthetic.make_x(wl, i, T_, Ci).view(np.int16)).to(dev).view(torch.bfloat16)
        bufs.append((name, X, torch.empty((T_, Ci), dtype=torch.uint8, device=dev),
                     torch.empty((T_,), dtype=torch.float32, device=dev)))
    K, W = args.steps, max(3, args.warmup)
    for _ in range(W):
        for _, X, Xq, xs in bufs:
            ptpc.quantize_activations(X, Xq, xs)
    per = {}
    with ClockSampler(dev.index or 0) as clk:
        for name, X, Xq, xs in bufs:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record(stream)
            for _ in range(K):
                ptpc.quantize_activations(X, Xq, xs)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            per[name] = e0.elapsed_time(e1) / K
    total_bytes = sum(quant_bytes(X.shape[0], X.shape[1]) for _, X, _, _ in bufs)
    gbs = total_bytes / (sum(per.values()) / 1e3) / 1e9
    print(json.dumps({
        "metric": "per-token activation quantiser GB/s (algorithmic 3 B/element + 4 B/row)", "value": gbs,
        "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": W, "higher_is_better": True,
        "frac_of_hbm": gbs / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"], "data": "synthetic",
        "config": {"workload": wl.name, "tokens": T, "inputs": [[X.shape[0], X.shape[1]] for _, X, _, _ in bufs]},
        "per_input_ms": per, "clocks": clk.summary(),
    }), flush=True)
    return 0


def chain_weights(ptpc, dev):
    """The 70B chain's four weights, quantised per output channel and per
    tensor: [(Layer, (Wq_t, w_scale), (Wq_t_pt, w_scale_pt))]."""
    import torch
    wl = synthetic.CHAIN_70B
    Ws = []
    for i, L in enumerate(wl.layers):
        Wb = torch.from_numpy(synthetic.make_w(wl, i, L.Ci, L.Co).view(np.int16)).to(dev).view(torch.bfloat16)
        Ws.append((L, ptpc.quantize_weights(Wb), ptpc.quantize_weights_per_tensor(Wb)))
        del Wb
    return Ws


def chain_roofline_ms(T, layers, peaks):
    """Roofline time of one chain pass: the slower of its algorithmic FP8
    FLOPs at the burst FP8 peak and its algorithmic bytes (quantiser + GEMM of
    every layer) at the HBM copy bandwidth."""
    flops = sum(2.0 * T * L.Ci * L.Co for L in layers)
    nbytes = sum(quant_bytes(T, L.Ci) + gemm_bytes(T, L.Ci, L.Co) for L in layers)
    return max(flops / (2.0 * peaks["bf16_tflops"] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e3


def chain_measure(ptpc, dev, Ws, T, peaks, graph=True, K=None):
    """One T of the chain QKV -> O -> gate+up -> down with dynamic per-token
    re-quantisation between layers: O reads QKV output columns [0, 8192) and
    down reads gate+up output columns [0, 28672) (column slices, no copies).
    The fused PTPC entry point, the page's naive two-step path (unscaled fp32
    GEMM, then a scaling kernel) and per-tensor scaling are timed side by side
    (CUDA events on the launch stream, after 3 warm-up passes)."""
    import torch
    wl = synthetic.CHAIN_70B
    stream = torch.cuda.current_stream(dev)
    flops_tok = sum(2.0 * L.Ci * L.Co for L, _, _ in Ws)
    X0 = torch.from_numpy(synthetic.make_x(wl, 0, T, wl.layers[0].Ci).view(np.int16)).to(dev).view(torch.bfloat16)
    outs = [torch.empty((T, L.Co), dtype=torch.bfloat16, device=dev) for L, _, _ in Ws]
    wsps = [ptpc.Workspace(ptpc.workspace_size(ptpc.OP_LINEAR, T, L.Ci, L.Co), dev) for L, _, _ in Ws]
    ys = [torch.empty((T, L.Co), dtype=torch.float32, device=dev) for L, _, _ in Ws]
    qs = [(torch.empty((T, L.Ci), dtype=torch.uint8, device=dev), torch.empty((T,), dtype=torch.float32, device=dev))
          for L, _, _ in Ws]
    pts = [ptpc.Workspace(ptpc.workspace_size(ptpc.OP_BENCH_PER_TENSOR, T, L.Ci, 0), dev) for L, _, _ in Ws]

    def layer_input(i):
        return X0 if i == 0 else outs[i - 1][:, :Ws[i][0].Ci]

    def fused():
        for i, (L, (Wq, ws), _) in enumerate(Ws):
            ptpc.linear(layer_input(i), Wq, ws, out=outs[i], ws=wsps[i])

    def naive():
        for i, (L, (Wq, ws), _) in enumerate(Ws):
            Xq, xs = ptpc.quantize_activations(layer_input(i), *qs[i])
            ptpc.unscaled_mm_f32(Xq, Wq, out=ys[i], ws=wsps[i])
            ptpc.apply_scales(ys[i], xs, ws, out=outs[i])

    def per_tensor():
        for i, (L, _, (Wq, ws)) in enumerate(Ws):
            Xq, xs = ptpc.quantize_activations_per_tensor(layer_input(i), *qs[i], ws=pts[i])
            ptpc.scaled_mm(Xq, xs, Wq, ws, out=outs[i], ws=wsps[i])

    paths = [("fused", fused), ("naive", naive), ("per_tensor", per_tensor)]
    g = None
    if graph:
        # the fused chain captured once into a CUDA graph and replayed (the
        # library only enqueues work on the current stream)
        for _ in range(2):
            fused()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        capture_stream = torch.cuda.Stream(dev)
        with torch.cuda.stream(capture_stream):
            with torch.cuda.graph(g, stream=capture_stream):
                fused()
        torch.cuda.synchronize(dev)
        paths.insert(1, ("fused_graph", g.replay))

    K = K or max(3, min(200, int(4e13 / (flops_tok * T))))
    res = {}
    for name, fn in paths:
        for _ in range(3):
            fn()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = e0.elapsed_time(e1) / K
    roof = chain_roofline_ms(T, [L for L, _, _ in Ws], peaks)
    rec = {
        "T": T, "steps": K, "fused_ms": res["fused"], "naive_ms": res["naive"], "per_tensor_ms": res["per_tensor"],
        "fused_tflops": flops_tok * T / (res["fused"] / 1e3) / 1e12,
        "roofline_ms": roof, "fused_frac_of_roofline": roof / res["fused"],
        "fused_speedup_over_naive": res["naive"] / res["fused"],
        "ptpc_over_per_tensor_throughput": res["per_tensor"] / res["fused"],
    }
    if graph:
        rec["fused_graph_ms"] = res["fused_graph"]
    del g, X0, outs, wsps, ys, qs, pts
    torch.cuda.empty_cache()
    return rec


def run_sweep(args):
    """Every T of the 70B chain (or --sweep-tokens), one JSON line each."""
    import torch

    import fp8_quantized_gemm_ptpc_b200 as ptpc

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    wl = synthetic.CHAIN_70B
    tokens = ([int(t) for t in args.sweep_tokens.split(",")] if args.sweep_tokens else list(wl.tokens))
    peaks = load_peaks()
    Ws = chain_weights(ptpc, dev)
    for T in tokens:
        rec = chain_measure(ptpc, dev, Ws, T, peaks)
        print(json.dumps({"kind": "chain_sweep", "workload": wl.name} | rec), flush=True)
    return 0


def run_tp(args):
    """Tensor-parallel 70B MLP pair on N ranks (one GPU each, NCCL between
    them): gate+up 8192 -> 57344 column-parallel (no collective), then down
    28672 -> 8192 row-parallel on each rank's slice of the gate+up output
    (the first 28672 / N of its columns, standing in for the SwiGLU between
    the layers): a MAX all-reduce of T row maxima and a SUM all-reduce of the
    T x 8192 fp32 accumulators.  Prints one JSON line (rank 0) with the step
    time as the maximum over ranks and whole-job TFLOP/s."""
    import torch
    import torch.distributed as dist

    from fp8_quantized_gemm_ptpc_b200.tp import ColumnParallelLinear, RowParallelLinear

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wl = synthetic.LLAMA70B_PREFILL
    T = args.tokens or wl.tokens[0]
    to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
    X = to_dev(synthetic.make_x(wl, 0, T, 8192))
    gate_up = ColumnParallelLinear(to_dev(synthetic.make_w(wl, 0, 8192, 57344)), rank, world)
    down = RowParallelLinear(to_dev(synthetic.make_w(wl, 1, 28672, 8192)), rank, world)
    width = down.k1 - down.k0

    def step():
        h = gate_up.forward(X)
        return down.forward(h[:, :width])

    stream = torch.cuda.current_stream(dev)
    K, W = args.steps, max(3, args.warmup)
    for _ in range(W):
        step()
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = dist_max(e0.elapsed_time(e1), dev) / K
    flops = 2.0 * T * 8192 * 57344 + 2.0 * T * 28672 * 8192        # the whole layer pair, over all ranks
    if rank == 0:
        print(json.dumps({
            "metric": "tensor-parallel PTPC-FP8 70B MLP pair TFLOP/s", "value": flops / (ms / 1e3) / 1e12,
            "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "data": "synthetic",
            "config": {"workload": f"70B gate_up 8192->57344 column-parallel + down 28672->8192 row-parallel, T={T}",
                       "parallelism": f"tp{world}"},
        }), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def run_record(args):
    """One sub-record of the default line on its own (1 GPU), printed as one
    JSON line: a short command to profile the decode GEMMs or the decode
    attention with."""
    import torch

    import fp8_quantized_gemm_ptpc_b200 as ptpc
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    steps = max(3, args.steps)
    tokens = [int(t) for t in args.decode_tokens.split(",") if t.strip()]
    if args.record == "decode":
        rec = decode_record(ptpc, dev, peaks, tokens, steps=steps)
    elif args.record == "decode_subbyte":
        rec = decode_subbyte_record(ptpc, dev, peaks, tokens, steps=steps,
                                    fmts=tuple(f for f in args.weight_formats.split(",") if f))
    elif args.record == "prefill_subbyte":
        rec = prefill_subbyte_record(ptpc, dev, peaks, steps=steps,
                                     fmts=tuple(f for f in args.weight_formats.split(",") if f))
    elif args.record == "kv_decode_405b":
        rec = kv_decode_record(ptpc, dev, peaks, Hq=128, steps=steps, model="Llama-3.1-405B")
    elif args.record == "kv_decode_long":
        rec = kv_decode_record(ptpc, dev, peaks, ctx=32768, steps=steps)
    else:
        rec = kv_decode_record(ptpc, dev, peaks, steps=steps)
    print(json.dumps({"record": args.record} | rec), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.quant_only:
        return run_quant_only(args)
    if args.sweep:
        return run_sweep(args)
    if args.tp:
        return run_tp(args)
    if args.record:
        return run_record(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
