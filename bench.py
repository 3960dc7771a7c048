"""Benchmark: Qwen2.5-0.5B-shaped M=1 decode step on Q8_0 weights, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-components]

One step = the 121 weight matmuls of one decode token (24 layers x {qkv 896->1152,
wo 896->896, gate 896->4864, up 896->4864, down 4864->896} + lm_head 896->151936)
on Q8_0 blocks with fp32 activations (M=1), stream-ordered and replayed as one CUDA
graph with programmatic dependent launch. Default schedule ("multi", 97 launches):
gate and up of each layer, which read the same activation vector, share one
qmm_q8_gemv_multi launch; every other matmul is one qmm_q8_gemv_ex call.
`--schedule gemv` issues the 121 matmuls as 121 qmm_q8_gemv_ex calls. Weights are seeded
synthetic tensors with the shapes of that model (no trained weights are used);
they total 524,833,792 bytes per step, more than the 126 MB L2, so no flush is
needed between steps. value = decode tokens/s (steps/s) summed over ranks.

Under torchrun (N > 1) every rank decodes its own sequence on its own copy of
the weights (data-parallel replicas, weak scaling); the only collective is the
max-over-ranks reduction of the measured time.

`--impl reference` times the CPU oracle (oracle/) on the host cores on a bounded
sample of the same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

METRIC = "Q8_0/Q4_0 GEMV HBM GB/s (% of B200 peak); decode-step tok/s equiv; prefill TFLOP/s"
UNIT = "tok/s"
WORKLOAD = ("Qwen2.5-0.5B-shaped M=1 decode step: 121 Q8_0 GEMVs (24 x qkv 896->1152, wo 896->896, "
            "gate/up 896->4864, down 4864->896, + lm_head 896->151936)")


def step_bytes():
    """Algorithmic bytes of one decode step: weight blocks + fp32 x read + fp32 y written."""
    w = x = y = 0
    for _, n, k in syn.decode_step_shapes():
        w += n * (k // 32) * 34
        x += k * 4
        y += n * 4
    return w, x, y


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------------- distributed plumbing

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return units_per_rank * world / (max_ms / 1000.0)


# --------------------------------------------------------------------------- clocks

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    def __init__(self, torch_device_index: int, period_s: float = 0.02):
        self.period = period_s
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml as nv
            import torch

            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            self.h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self._reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # noqa: BLE001 - report, do not fail the bench
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM), int(self._reasons(self.h)),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        if self._thread:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "error": getattr(self, "err", "")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        bits = 0
        for _, b, _ in self.samples:
            bits |= b
        reasons = [name for bit, name in REASON_BITS.items() if bits & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "power_w_max": round(max(s[2] for s in self.samples), 1)}


# --------------------------------------------------------------------------- the decode-step workload

class DecodeStep:
    """121 Q8_0 weight matrices resident in HBM, their activations and outputs.

    Default: every matmul reads its own activation vector (N(0,1), one slice of
    one concatenated buffer) -- the decode-step workload as specified. With
    chain=True the matmuls read each other's outputs along the model's data
    flow (synthetic.decode_step_sources: qkv <- previous down, wo <- qkv,
    gate/up <- wo, down <- up, lm_head <- last down) and the Q8_0 scales are
    drawn with synthetic.chain_dscale, so 121 chained products stay O(1); only
    the first input vector comes from the host."""

    def __init__(self, seed: int, device, keep_host: bool, chain: bool = False):
        import torch

        self.shapes = syn.decode_step_shapes()
        self.chain = chain
        self.host_w = [] if keep_host else None
        self.host_x = []
        self.W = []
        xs = []
        for i, (_, n, k) in enumerate(self.shapes):
            g = syn.rng(syn.sub_seed(seed, i))
            if chain:
                wb, _, _ = syn.q8_0_weights(g, n, k, dscale=syn.chain_dscale(k))
            else:
                wb, _, _ = syn.q8_0_weights(g, n, k)
            self.W.append(torch.from_numpy(wb).to(device))
            if keep_host:
                self.host_w.append(wb)
            if not chain or i == 0:
                x = syn.act_f32(g, 1, k)
                self.host_x.append(x)
                xs.append(x.reshape(-1))
        self.x_offsets = np.cumsum([0] + [x.size for x in xs])
        self.y_offsets = np.cumsum([0] + [n for _, n, _ in self.shapes])
        self.host_xcat = torch.from_numpy(np.concatenate(xs)).pin_memory()
        self.X = self.host_xcat.to(device)
        self.Y = torch.zeros(int(self.y_offsets[-1]), dtype=torch.float32, device=device)
        self.host_logits = torch.empty(self.shapes[-1][1], dtype=torch.float32).pin_memory()
        xp, yp = self.X.data_ptr(), self.Y.data_ptr()
        self.y_ptrs = [yp + 4 * int(self.y_offsets[i]) for i in range(len(self.shapes))]
        if chain:
            src = syn.decode_step_sources()
            self.sources = src
            self.x_ptrs = [xp if j < 0 else self.y_ptrs[j] for j in src]
        else:
            self.sources = None
            self.x_ptrs = [xp + 4 * int(self.x_offsets[i]) for i in range(len(self.shapes))]

    def launch(self, qmm, stream_handle: int, flags: int):
        """The 121 matmuls, one qmm_q8_gemv_ex call each."""
        lib = qmm.lib
        for i, (_, n, k) in enumerate(self.shapes):
            st = lib.qmm_q8_gemv_ex(1, n, k, 32, self.W[i].data_ptr(), self.x_ptrs[i], self.y_ptrs[i], flags,
                                    stream_handle)
            if st != 0:
                raise qmm.QmmError(st, "qmm_q8_gemv_ex")

    def launch_multi(self, qmm, stream_handle: int, flags: int):
        """The same matmul set with each layer's gate and up projections as one
        qmm_q8_gemv_multi launch over their shared activation vector (97 launches).
        Without chain=True gate and up have different inputs; the launch then
        reads the gate's for both (same bytes, same kernels)."""
        import ctypes

        lib = qmm.lib
        i = 0
        while i < len(self.shapes):
            name, n, k = self.shapes[i]
            if name.endswith(".gate") and i + 1 < len(self.shapes) and self.shapes[i + 1][0].endswith(".up"):
                n2 = self.shapes[i + 1][1]
                N = (ctypes.c_int64 * 2)(n, n2)
                W = (ctypes.c_void_p * 2)(self.W[i].data_ptr(), self.W[i + 1].data_ptr())
                Y = (ctypes.c_void_p * 2)(self.y_ptrs[i], self.y_ptrs[i + 1])
                st = lib.qmm_q8_gemv_multi(1, k, 32, 2, N, W, self.x_ptrs[i], Y, flags, stream_handle)
                if st != 0:
                    raise qmm.QmmError(st, "qmm_q8_gemv_multi")
                i += 2
                continue
            st = lib.qmm_q8_gemv_ex(1, n, k, 32, self.W[i].data_ptr(), self.x_ptrs[i], self.y_ptrs[i], flags,
                                    stream_handle)
            if st != 0:
                raise qmm.QmmError(st, "qmm_q8_gemv_ex")
            i += 1

    def launch_auto(self, qmm, stream_handle: int, flags: int, qx, dx):
        """The same matmul set through qmm_q8_gemv_auto: short-K GEMVs whose
        slices fit on chip as fused Q8xQ8 (quantised activations), the rest fp32.
        qx / dx: scratch for the codes and scales (largest K)."""
        lib = qmm.lib
        for i, (_, n, k) in enumerate(self.shapes):
            st = lib.qmm_q8_gemv_auto(1, n, k, 32, self.W[i].data_ptr(), self.x_ptrs[i], self.y_ptrs[i],
                                      qx.data_ptr(), dx.data_ptr(), flags, stream_handle)
            if st != 0:
                raise qmm.QmmError(st, "qmm_q8_gemv_auto")

    def schedule(self, name: str):
        """The launch function of a named schedule ("gemv": 121 launches, "multi": 97,
        "auto": 121 qmm_q8_gemv_auto calls sharing the step's code/scale buffers)."""
        if name == "auto":
            if not hasattr(self, "_qx"):
                import torch

                kmax = max(k for _, _, k in self.shapes)
                self._qx = torch.empty(kmax, dtype=torch.int8, device=self.X.device)
                self._dx = torch.empty(kmax // 32, dtype=torch.float32, device=self.X.device)
            return lambda qmm, h, flags: self.launch_auto(qmm, h, flags, self._qx, self._dx)
        return {"gemv": self.launch, "multi": self.launch_multi}[name]

    def launches(self, name: str) -> int:
        return len(self.shapes) - QWEN_LAYERS if name == "multi" else len(self.shapes)

    def x_of(self, i: int, Y_host=None):
        """Host copy of matmul i's input vector (from Y_host, the step's outputs, in chain mode)."""
        k = self.shapes[i][2]
        if self.chain and self.sources[i] >= 0:
            j = self.sources[i]
            return np.asarray(Y_host[int(self.y_offsets[j]):int(self.y_offsets[j]) + k], dtype=np.float32).reshape(1, k)
        return self.host_x[0 if self.chain else i]

    def logits(self):
        return self.Y[int(self.y_offsets[-2]):int(self.y_offsets[-1])]


QWEN_LAYERS = syn.QWEN05B_LAYERS


def step_graph(qmm, step: DecodeStep, stream, schedule: str, flags: int):
    """The benchmark's decode step as a CUDA graph: one eager call of the
    schedule (outside capture), then the same calls captured on `stream`."""
    import torch

    fn = step.schedule(schedule)
    fn(qmm, stream.cuda_stream, flags)
    torch.cuda.synchronize()
    return capture(lambda h: fn(qmm, h, flags), stream)


def capture(fn, stream):
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(torch.cuda.current_stream().cuda_stream)
    return g


def time_graph(graph, stream, reps: int) -> float:
    """Average ms of one replay over `reps` back-to-back replays (CUDA events on `stream`)."""
    import torch

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


# --------------------------------------------------------------------------- components (rank 0, N=1)

def component_single_gemv(qmm, dev_peak_gbs, n=1152, k=896, reps_graph=4):
    """Single GEMV (M=1, K=896, N=1152): back-to-back launches over rotating weight copies
    totalling > 2x L2, so every launch streams its weights from HBM."""
    import torch

    props = torch.cuda.get_device_properties(0)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20)
    wbytes = n * (k // 32) * 34
    copies = max(8, int(2.2 * l2 // wbytes) + 1)
    g = syn.rng(0)
    wb, _, _ = syn.q8_0_weights(g, n, k)
    x = torch.from_numpy(syn.act_f32(g, 1, k)).cuda()
    W0 = torch.from_numpy(wb).cuda()
    Ws = [W0.clone() for _ in range(copies)]
    Y = torch.empty(n, device="cuda")
    s = torch.cuda.Stream()
    out = {}
    for name, flags in (("graph_pdl_early_weights", qmm.QMM_FLAG_EARLY_WEIGHTS), ("graph_pdl", 0)):
        def fn(h, flags=flags):
            for w in Ws:
                st = qmm.lib.qmm_q8_gemv_ex(1, n, k, 32, w.data_ptr(), x.data_ptr(), Y.data_ptr(), flags, h)
                assert st == 0
        fn(s.cuda_stream)
        torch.cuda.synchronize()
        gr = capture(fn, s)
        time_graph(gr, s, 2)
        ms = time_graph(gr, s, reps_graph) / copies
        bytes_ = wbytes + k * 4 + n * 4
        out[name] = {"us_per_gemv": round(ms * 1e3, 3), "GB_s": round(bytes_ / ms / 1e6, 1),
                     "frac_hbm": round(bytes_ / ms / 1e6 / dev_peak_gbs, 4)}
        del gr
    out["bytes_per_gemv"] = wbytes + k * 4 + n * 4
    out["note"] = f"{copies} rotating weight copies (> 2x L2) in one CUDA graph"
    return out


def component_lm_head(qmm, step: DecodeStep, dev_peak_gbs, reps=20):
    """The largest GEMV of the step (lm_head 896->151936, 145 MB of blocks): one
    launch alone per graph replay, and per launch in a chain of dependent
    launches over three weight copies (as in the step: programmatic dependent
    launch, weights streamed ahead of the dependency)."""
    import torch

    n, k = step.shapes[-1][1], step.shapes[-1][2]
    s = torch.cuda.Stream()
    W = step.W[-1]
    xp = step.X.data_ptr() + 4 * int(step.x_offsets[-2])
    yp = step.Y.data_ptr() + 4 * int(step.y_offsets[-2])
    bytes_ = n * (k // 32) * 34 + k * 4 + n * 4

    def fn(h):
        assert qmm.lib.qmm_q8_gemv_ex(1, n, k, 32, W.data_ptr(), xp, yp, 0, h) == 0
    fn(s.cuda_stream)
    gr = capture(fn, s)
    time_graph(gr, s, 3)
    ms = time_graph(gr, s, reps)
    out = {"us": round(ms * 1e3, 2), "GB_s": round(bytes_ / ms / 1e6, 1),
           "frac_hbm": round(bytes_ / ms / 1e6 / dev_peak_gbs, 4), "bytes": bytes_}
    Ws = [W] + [W.clone() for _ in range(2)]

    def chain(h):
        for w in Ws:
            assert qmm.lib.qmm_q8_gemv_ex(1, n, k, 32, w.data_ptr(), xp, yp, qmm.QMM_FLAG_EARLY_WEIGHTS, h) == 0
    chain(s.cuda_stream)
    torch.cuda.synchronize()
    gr2 = capture(chain, s)
    time_graph(gr2, s, 3)
    ms2 = time_graph(gr2, s, reps) / len(Ws)
    out["chain"] = {"us": round(ms2 * 1e3, 2), "GB_s": round(bytes_ / ms2 / 1e6, 1),
                    "frac_hbm": round(bytes_ / ms2 / 1e6 / dev_peak_gbs, 4)}
    del gr2, Ws
    return out


def component_step_schedule(qmm, step: DecodeStep, schedule: str, dev_peak_gbs, reps=200):
    """The decode step's matmul set under another schedule than the headline's
    ("gemv": 121 qmm_q8_gemv_ex launches; "multi": gate and up of each layer in
    one qmm_q8_gemv_multi launch, 97 launches; same bytes)."""
    import torch

    s = torch.cuda.Stream()
    gr = step_graph(qmm, step, s, schedule, qmm.QMM_FLAG_EARLY_WEIGHTS)
    time_graph(gr, s, 20)
    ms = time_graph(gr, s, reps)
    del gr
    bytes_ = sum(n * (k // 32) * 34 + k * 4 + n * 4 for _, n, k in step.shapes)
    return {"ms_per_step": round(ms, 5), "tok_s": round(1e3 / ms, 2), "launches": step.launches(schedule),
            "GB_s": round(bytes_ / ms / 1e6, 1), "frac_hbm": round(bytes_ / ms / 1e6 / dev_peak_gbs, 4)}


def component_step_auto(qmm, step: DecodeStep, dev_peak_gbs, reps=200):
    """The decode step's matmul set through the per-K choice (qmm_q8_gemv_auto):
    short-K GEMVs as fused Q8xQ8 on quantised activations, long-K ones fp32 --
    a different numerical contract from the headline's fp32 activations."""
    out = component_step_schedule(qmm, step, "auto", dev_peak_gbs, reps)
    out["note"] = "qkv, wo, gate, up as fused Q8xQ8 (quantised activations); down and lm_head fp32"
    return out


def component_gateup(qmm, dev_peak_gbs, m=8, n=17408, k=5120, reps=10):
    """Fused Q4_0 gate/up SwiGLU (M=8, K=5120, N=17408) vs the unfused path (two
    projection launches + silu*mul); three rotating weight pairs (> L2)."""
    import torch

    g = syn.rng(3)
    pairs = [(torch.from_numpy(syn.q4_0_weights(g, n, k)[0]).cuda(), torch.from_numpy(syn.q4_0_weights(g, n, k)[0]).cuda())
             for _ in range(3)]
    x = torch.from_numpy(syn.act_f32(g, m, k)).cuda()
    Y = torch.empty(m, n, device="cuda")
    G, U = torch.empty(m, n, device="cuda"), torch.empty(m, n, device="cuda")
    s = torch.cuda.Stream()
    out = {}

    def fused(h):
        for wg, wu in pairs:
            assert qmm.lib.qmm_q4_swiglu_gateup_ex(m, n, k, 32, wg.data_ptr(), wu.data_ptr(), x.data_ptr(),
                                                   Y.data_ptr(), qmm.QMM_FLAG_EARLY_WEIGHTS, h) == 0

    def unfused(h):
        for wg, wu in pairs:
            assert qmm.lib.qmm_q4_gateup_unfused(m, n, k, 32, wg.data_ptr(), wu.data_ptr(), x.data_ptr(),
                                                 G.data_ptr(), U.data_ptr(), Y.data_ptr(), h) == 0

    bytes_ = 2 * n * (k // 32) * 18 + m * k * 4 + m * n * 4
    for name, fn in (("fused", fused), ("unfused", unfused)):
        fn(s.cuda_stream)
        torch.cuda.synchronize()
        gr = capture(fn, s)
        time_graph(gr, s, 3)
        us = time_graph(gr, s, reps) / len(pairs) * 1e3
        out[name] = {"us": round(us, 2), "GB_s": round(bytes_ / us / 1e3, 1),
                     "frac_hbm": round(bytes_ / us / 1e3 / dev_peak_gbs, 4)}
        del gr
    out["bytes"] = bytes_
    out["flops"] = 2 * 2 * m * n * k
    out["fused_vs_unfused_time"] = round(out["fused"]["us"] / out["unfused"]["us"] - 1.0, 4)
    return out


def component_q4_gemv(qmm, dev_peak_gbs, reps=10):
    """Q4_0 GEMV (one projection): M=1 at K=5120, N=17408 and the M=8 down
    projection K=17408, N=5120; three rotating weight copies (> L2) in a chain."""
    import torch

    out = {}
    g = syn.rng(5)
    for name, m, n, k in (("m1_k5120_n17408", 1, 17408, 5120), ("m8_k17408_n5120", 8, 5120, 17408)):
        Ws = [torch.from_numpy(syn.q4_0_weights(g, n, k)[0]).cuda() for _ in range(3)]
        x = torch.from_numpy(syn.act_f32(g, m, k)).cuda()
        Y = torch.empty(m, n, device="cuda")
        s = torch.cuda.Stream()

        def fn(h):
            for w in Ws:
                assert qmm.lib.qmm_q4_gemv(m, n, k, 32, w.data_ptr(), x.data_ptr(), Y.data_ptr(),
                                           qmm.QMM_FLAG_EARLY_WEIGHTS, h) == 0
        fn(s.cuda_stream)
        torch.cuda.synchronize()
        gr = capture(fn, s)
        time_graph(gr, s, 3)
        ms = time_graph(gr, s, reps) / len(Ws)
        bytes_ = n * (k // 32) * 18 + m * k * 4 + m * n * 4
        out[name] = {"us": round(ms * 1e3, 2), "GB_s": round(bytes_ / ms / 1e6, 1),
                     "frac_hbm": round(bytes_ / ms / 1e6 / dev_peak_gbs, 4), "bytes": bytes_}
        del gr, Ws
    return out


def component_q8q8(qmm, dev_peak_gbs, reps_graph=4):
    """Q8xQ8 decode GEMV (M=1) at K=896/N=4864 and K=4864/N=896: the GEMV on
    quantized activations alone, activation quantization + GEMV as two launches
    and as one fused launch, and the fp32
    activation GEMV of the same shape for comparison; rotating weight copies
    (> 2x L2) in one CUDA graph."""
    import torch

    props = torch.cuda.get_device_properties(0)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20)
    out = {}
    for n, k in ((4864, 896), (896, 4864)):
        wbytes = n * (k // 32) * 34
        copies = max(8, int(2.2 * l2 // wbytes) + 1)
        g = syn.rng(2)
        W0 = torch.from_numpy(syn.q8_0_weights(g, n, k)[0]).cuda()
        Ws = [W0.clone() for _ in range(copies)]
        x = torch.from_numpy(syn.act_f32(g, 1, k)).cuda()
        qx = torch.empty(k, dtype=torch.int8, device="cuda")
        dx = torch.empty(k // 32, device="cuda")
        Y = torch.empty(n, device="cuda")
        s = torch.cuda.Stream()
        lib = qmm.lib
        fl = qmm.QMM_FLAG_EARLY_WEIGHTS

        def gemv_q8(h):
            for w in Ws:
                assert lib.qmm_q8q8_gemv_ex(1, n, k, 32, w.data_ptr(), qx.data_ptr(), dx.data_ptr(), Y.data_ptr(), fl, h) == 0

        def quant_gemv(h):
            for w in Ws:
                assert lib.qmm_quantize_act_q8(1, k, 32, x.data_ptr(), qx.data_ptr(), dx.data_ptr(), h) == 0
                assert lib.qmm_q8q8_gemv_ex(1, n, k, 32, w.data_ptr(), qx.data_ptr(), dx.data_ptr(), Y.data_ptr(), fl, h) == 0

        def gemv_f32(h):
            for w in Ws:
                assert lib.qmm_q8_gemv_ex(1, n, k, 32, w.data_ptr(), x.data_ptr(), Y.data_ptr(), fl, h) == 0

        def fused(h):
            for w in Ws:
                assert lib.qmm_q8q8_gemv_fused(1, n, k, 32, w.data_ptr(), x.data_ptr(), qx.data_ptr(), dx.data_ptr(),
                                               Y.data_ptr(), fl, h) == 0

        res = {}
        for name, fn, extra in (("q8q8_gemv", gemv_q8, k + (k // 32) * 4),
                                ("quantize_plus_q8q8_gemv", quant_gemv, k * 4),
                                ("q8q8_gemv_fused", fused, k * 4 + k + (k // 32) * 4),
                                ("f32_gemv_same_shape", gemv_f32, k * 4)):
            fn(s.cuda_stream)
            torch.cuda.synchronize()
            gr = capture(fn, s)
            time_graph(gr, s, 2)
            ms = time_graph(gr, s, reps_graph) / copies
            bytes_ = wbytes + extra + n * 4
            res[name] = {"us": round(ms * 1e3, 3), "GB_s": round(bytes_ / ms / 1e6, 1),
                         "frac_hbm": round(bytes_ / ms / 1e6 / dev_peak_gbs, 4)}
            del gr
        res["note"] = f"{copies} rotating weight copies; per-call times in a chain of stream-ordered launches"
        out[f"k{k}_n{n}"] = res
    return out


def component_prefill(qmm, pk, reps=10):
    """Prefill panels on the tensor cores: TFLOP/s per shape (rotating weight copies
    > L2 where the weights are small; activations bf16 N(0,1)); a chain of calls with
    early weights (weight blocks streamed while the previous call finishes)."""
    import torch

    shapes = [("q8_m32_k896_n4864", syn.Q8_0, 32, 4864, 896), ("q8_m32_k4864_n896", syn.Q8_0, 32, 896, 4864),
              ("q8_m1024_k896_n4864", syn.Q8_0, 1024, 4864, 896), ("q8_m1024_k4864_n896", syn.Q8_0, 1024, 896, 4864),
              ("q4_m1024_k5120_n17408", syn.Q4_0, 1024, 17408, 5120)]
    out = {}
    g = syn.rng(4)
    for name, wt, m, n, k in shapes:
        wbytes = n * (k // 32) * (34 if wt == syn.Q8_0 else 18)
        copies = max(1, int(3 * 126e6 // wbytes) + 1) if wbytes < 200e6 else 1
        copies = min(copies, 64)
        W0 = torch.from_numpy(syn.weights(g, wt, n, k)).cuda()
        Ws = [W0] + [W0.clone() for _ in range(copies - 1)]
        X = torch.from_numpy(syn.act_bf16_bits(g, m, k).view(np.int16)).cuda()
        Y = torch.empty(m, n, device="cuda")
        s = torch.cuda.Stream()

        def fn(h, Ws=Ws, X=X, Y=Y, wt=wt, m=m, n=n, k=k):
            for w in Ws:
                assert qmm.lib.qmm_quant_matmul_prefill_ex(wt, m, n, k, 32, w.data_ptr(), X.data_ptr(), Y.data_ptr(),
                                                           qmm.QMM_FLAG_EARLY_WEIGHTS, h) == 0
        fn(s.cuda_stream)
        torch.cuda.synchronize()
        gr = capture(fn, s)
        time_graph(gr, s, 2)
        us = time_graph(gr, s, reps) / len(Ws) * 1e3
        flops = 2 * m * n * k
        bytes_ = wbytes + m * k * 2 + m * n * 4
        out[name] = {"us": round(us, 2), "TFLOP_s": round(flops / us / 1e6, 1),
                     "frac_tensor_burst": round(flops / us / 1e6 / pk["bf16_tflops"], 4),
                     "GB_s": round(bytes_ / us / 1e3, 1), "frac_hbm": round(bytes_ / us / 1e3 / pk["hbm_gbs"], 4),
                     "weight_copies": len(Ws)}
        del gr, Ws
    return out


# --------------------------------------------------------------------------- CPU oracle baseline

def oracle_step_sample(step_w, step_x, shapes, frac: float, threads: int):
    """Run the oracle on the first ceil(frac * N) rows of every GEMV of a step, with
    `threads` host threads over disjoint row windows. Returns seconds."""
    import oracle

    jobs = []
    for i, (_, n, k) in enumerate(shapes):
        rows = max(1, int(np.ceil(frac * n)))
        per = max(1, (rows + threads - 1) // threads)
        for r0 in range(0, rows, per):
            jobs.append((i, n, r0, min(rows, r0 + per)))
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda j: oracle.gemv(syn.Q8_0, step_w[j[0]], step_x[j[0]], j[1], window=(0, 1, j[2], j[3])),
                    jobs))
    return time.perf_counter() - t0


def cpu_baseline(step_w, step_x, shapes, budget_s: float = 10.0):
    """The oracle timed on the host cores: on all of them (the reported value) and
    on one thread, each on whole decode steps or a row fraction of one when a
    step is slower than the budget, repeated until ~budget_s of work."""
    def timed(threads, budget):
        t_probe = oracle_step_sample(step_w, step_x, shapes, 0.01, threads)
        full_est = t_probe / 0.01
        frac = min(1.0, max(0.001, budget / max(full_est, 1e-9)))
        done = t = 0.0
        steps = 0
        while t < budget and steps < 200:
            t += oracle_step_sample(step_w, step_x, shapes, frac, threads)
            done += frac
            steps += 1
        return done / t, steps, frac, t

    threads = os.cpu_count() or 1
    v_all, steps, frac, t = timed(threads, budget_s)
    v_one, steps1, frac1, t1 = timed(1, budget_s / 2)
    return {"value": round(v_all, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{steps} x first {frac:.1%} of the rows of all 121 GEMVs of a decode step (fp64 C oracle, "
                      f"{threads} threads over row windows), {t:.1f} s; tok/s = steps done / time",
            "single_thread": {"value": round(v_one, 3), "unit": UNIT, "cores": 1,
                              "sample": f"{steps1} x first {frac1:.1%} of the rows of all 121 GEMVs, one thread, "
                                        f"{t1:.1f} s"}}


def run_reference(args):
    """Reference arm: the CPU oracle timed on a bounded sample of the decode step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle

    oracle.build()
    shapes = syn.decode_step_shapes()
    host_w, host_x = [], []
    for i, (_, n, k) in enumerate(shapes):
        g = syn.rng(syn.sub_seed(args.seed, i))
        host_w.append(syn.q8_0_weights(g, n, k)[0])
        host_x.append(syn.act_f32(g, 1, k))
    threads = os.cpu_count() or 1
    t_probe = oracle_step_sample(host_w, host_x, shapes, 0.01, threads)
    full_est = t_probe / 0.01
    total_budget = 150.0
    per_step = total_budget / (args.steps + args.warmup)
    frac = min(1.0, max(1e-4, per_step / max(full_est, 1e-9)))
    for _ in range(args.warmup):
        oracle_step_sample(host_w, host_x, shapes, frac, threads)
    t = 0.0
    for _ in range(args.steps):
        t += oracle_step_sample(host_w, host_x, shapes, frac, threads)
    value = args.steps * frac / t
    sample = (f"each step: first {frac:.3%} of the rows of all 121 GEMVs (fp64 C oracle, {threads} threads over "
              f"row windows); tok/s = steps * fraction / time")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * t / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- traffic from the committed ncu summary

def committed_traffic(kernel_src: str, summary: str):
    """DRAM bytes of one decode step recorded in a profiles/ summary, if the kernel
    source is unchanged since (the summary records the source's sha1)."""
    try:
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        src = open(os.path.join(ROOT, "decode_gemv_qmm_b200", "csrc", kernel_src), "rb").read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_step:\s*([0-9]+)", text)
    h = re.search(r"kernel_source_sha1:\s*([0-9a-f]{40})", text)
    if not m or not h or h.group(1) != hashlib.sha1(src).hexdigest():
        return None
    return int(m.group(1))


# --------------------------------------------------------------------------- single-kernel cases (profiling)

def run_case(spec: str, reps: int, seed: int):
    """Launch one named kernel `reps` times back to back (eager, stream-ordered)
    and print the average time of the last reps-1. For profiler captures; the
    numbers it prints are not benchmark values.

    gemv:N:K            qmm_q8_gemv, M=1
    multi:N1,N2,..:K    qmm_q8_gemv_multi, M=1 (projections of one activation vector)
    q8q8:N:K            qmm_quantize_act_q8 + qmm_q8q8_gemv, M=1
    q8q8f:N:K           qmm_q8q8_gemv_fused, M=1
    q4gemv:M:N:K        qmm_q4_gemv
    gateup:M:N:K        qmm_q4_swiglu_gateup
    prefill:q8|q4:M:N:K qmm_quant_matmul_prefill
    decode_step         the 121 GEMVs of one decode step
    """
    import torch

    import decode_gemv_qmm_b200 as qmm

    torch.cuda.set_device(0)
    parts = spec.split(":")
    g = syn.rng(seed)
    launches = []
    if parts[0] == "gemv":
        n, k = int(parts[1]), int(parts[2])
        W = torch.from_numpy(syn.q8_0_weights(g, n, k)[0]).cuda()
        x = torch.from_numpy(syn.act_f32(g, 1, k)).cuda()
        y = torch.empty(1, n, device="cuda")
        launches.append(lambda: qmm.qmm_q8_gemv(W, x, n, y))
    elif parts[0] == "multi":
        ns, k = [int(v) for v in parts[1].split(",")], int(parts[2])
        Ws = [torch.from_numpy(syn.q8_0_weights(g, n, k)[0]).cuda() for n in ns]
        x = torch.from_numpy(syn.act_f32(g, 1, k)).cuda()
        ys = [torch.empty(1, n, device="cuda") for n in ns]
        launches.append(lambda: qmm.qmm_q8_gemv_multi(Ws, x, ns, ys))
    elif parts[0] == "q8q8":
        n, k = int(parts[1]), int(parts[2])
        W = torch.from_numpy(syn.q8_0_weights(g, n, k)[0]).cuda()
        x = torch.from_numpy(syn.act_f32(g, 1, k)).cuda()
        qx = torch.empty(1, k, dtype=torch.int8, device="cuda")
        dx = torch.empty(1, k // 32, device="cuda")
        y = torch.empty(1, n, device="cuda")
        launches.append(lambda: (qmm.qmm_quantize_act_q8(x, qx, dx), qmm.qmm_q8q8_gemv(W, qx, dx, n, y)))
    elif parts[0] == "q8q8f":
        n, k = int(parts[1]), int(parts[2])
        W = torch.from_numpy(syn.q8_0_weights(g, n, k)[0]).cuda()
        x = torch.from_numpy(syn.act_f32(g, 1, k)).cuda()
        qx = torch.empty(1, k, dtype=torch.int8, device="cuda")
        dx = torch.empty(1, k // 32, device="cuda")
        y = torch.empty(1, n, device="cuda")
        launches.append(lambda: qmm.qmm_q8q8_gemv_fused(W, x, n, y, qx, dx))
    elif parts[0] == "q4gemv":
        m, n, k = int(parts[1]), int(parts[2]), int(parts[3])
        W = torch.from_numpy(syn.q4_0_weights(g, n, k)[0]).cuda()
        x = torch.from_numpy(syn.act_f32(g, m, k)).cuda()
        y = torch.empty(m, n, device="cuda")
        launches.append(lambda: qmm.qmm_q4_gemv(W, x, n, y))
    elif parts[0] == "gateup":
        m, n, k = int(parts[1]), int(parts[2]), int(parts[3])
        Wg = torch.from_numpy(syn.q4_0_weights(g, n, k)[0]).cuda()
        Wu = torch.from_numpy(syn.q4_0_weights(g, n, k)[0]).cuda()
        x = torch.from_numpy(syn.act_f32(g, m, k)).cuda()
        y = torch.empty(m, n, device="cuda")
        launches.append(lambda: qmm.qmm_q4_swiglu_gateup(Wg, Wu, x, n, y))
    elif parts[0] == "prefill":
        wt = syn.Q8_0 if parts[1] == "q8" else syn.Q4_0
        m, n, k = int(parts[2]), int(parts[3]), int(parts[4])
        W = torch.from_numpy(syn.weights(g, wt, n, k)).cuda()
        X = torch.from_numpy(syn.act_bf16_bits(g, m, k).view(np.int16)).cuda()
        Y = torch.empty(m, n, device="cuda")
        launches.append(lambda: qmm.qmm_quant_matmul_prefill(wt, W, X, n, Y))
    elif parts[0] == "decode_step":
        step = DecodeStep(seed, torch.device("cuda", 0), keep_host=False)
        launches.append(lambda: step.launch(qmm, torch.cuda.current_stream().cuda_stream, qmm.QMM_FLAG_EARLY_WEIGHTS))
    else:
        raise SystemExit(f"unknown case {spec!r}")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for r in range(reps):
        if r == 1:
            e0.record()
        for f in launches:
            f()
    e1.record()
    torch.cuda.synchronize()
    if reps > 1:
        print(json.dumps({"case": spec, "reps": reps, "us_per_rep": round(e0.elapsed_time(e1) * 1e3 / (reps - 1), 2),
                          "note": "eager launches for profiling; not a benchmark value"}))
    return 0


# --------------------------------------------------------------------------- tensor parallel (column shards)

def run_tensor_parallel(args):
    """The decode step with every weight matrix's rows split over the ranks
    (decode_gemv_qmm_b200.shard: rank r owns rows [r N / G, (r + 1) N / G) of
    each matrix, computes its slice with qmm_q8_gemv and the slices are
    all-gathered after each matmul). Strong scaling: all ranks work on the same
    token, value = steps/s of the whole job. Launches are eager (the NCCL
    all-gathers are not captured in a CUDA graph)."""
    import datetime

    import torch
    import torch.distributed as dist

    import decode_gemv_qmm_b200 as qmm
    from decode_gemv_qmm_b200 import shard

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    shapes = syn.decode_step_shapes()
    Wl, Xs, Yl = [], [], []
    for i, (_, n, k) in enumerate(shapes):
        g = syn.rng(syn.sub_seed(args.seed, i))
        wb, _, _ = syn.q8_0_weights(g, n, k)
        x = syn.act_f32(g, 1, k)
        r0, r1 = shard.row_range(n, rank, world)
        Wl.append(torch.from_numpy(np.ascontiguousarray(shard.weight_shard(wb, n, k, rank, world))).to(dev))
        Xs.append(torch.from_numpy(x).to(dev))
        Yl.append(torch.empty((1, r1 - r0), dtype=torch.float32, device=dev))

    def step():
        outs = []
        for i, (_, n, k) in enumerate(shapes):
            qmm.qmm_q8_gemv(Wl[i], Xs[i], Yl[i].shape[1], Yl[i], flags=qmm.QMM_FLAG_EARLY_WEIGHTS)
            outs.append(shard.gather_rows(Yl[i], n, rank, world))
        return outs

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if rank == 0:
        wb, xb, yb = step_bytes()
        line = {"metric": METRIC, "value": round(args.steps / (ms / 1000.0), 2), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic",
                "config": {"workload": WORKLOAD, "M": 1, "weight_format": "Q8_0", "bytes_per_step": wb + xb + yb,
                           "parallelism": f"tp{world} (column shards, all-gather after each matmul; eager)"},
                "gpu_launches": len(shapes) * args.steps}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# --------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="qmm", choices=["qmm", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None, help="launch one named kernel (see run_case) instead of the benchmark")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--schedule", default="multi", choices=["gemv", "multi"],
                    help="decode-step schedule: 121 qmm_q8_gemv_ex launches, or gate+up of each layer in one "
                         "qmm_q8_gemv_multi launch (97)")
    ap.add_argument("--parallel", default="dp", choices=["dp", "tp"],
                    help="N > 1: data-parallel replicas (default) or column-sharded weights (tp)")
    args = ap.parse_args(argv)
    if args.case:
        return run_case(args.case, args.reps, args.seed)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.parallel == "tp":
        return run_tensor_parallel(args)

    import torch

    rank, world, local_rank = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    import decode_gemv_qmm_b200 as qmm

    pk = peaks()
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    step = DecodeStep(args.seed, device, keep_host=want_cpu)
    stream = torch.cuda.Stream()
    flags = qmm.QMM_FLAG_EARLY_WEIGHTS
    graph = step_graph(qmm, step, stream, args.schedule, flags)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()

    # timed region: K steps, barrier + synchronize on both sides
    sampler = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with sampler:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms_total, world, device)
    ms_step = ms_max / args.steps
    value = aggregate(args.steps, world, ms_max)

    # e2e: host activations -> device, the step, logits -> host (pinned), every step
    h2d = step.host_xcat.numel() * 4
    d2h = step.host_logits.numel() * 4
    logits = step.logits()
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(10, min(args.steps, 2000))
    with torch.cuda.stream(stream):
        f0.record(stream)
        for _ in range(e2e_steps):
            step.X.copy_(step.host_xcat, non_blocking=True)
            graph.replay()
            step.host_logits.copy_(logits, non_blocking=True)
        f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, device)
    e2e_value = aggregate(e2e_steps, world, e2e_ms)

    wb, xb, yb = step_bytes()
    bytes_step = wb + xb + yb
    launches = step.launches(args.schedule)
    achieved_gbs = bytes_step / (ms_step * 1e6)
    traffic = committed_traffic("q8_gemv.cu", "q8_gemv_decode_step.md")
    roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved_gbs / pk["hbm_gbs"], 4),
                "traffic": (round(traffic / launches) if traffic else None),
                "kernel": f"q8_gemv ({launches} launches per step: fp32 register-resident, tensor-core resident "
                          "and streaming variants)",
                "per_launch": {"algorithmic_bytes": round(bytes_step / launches),
                               "avg_duration_us": round(ms_step * 1e3 / launches, 3)},
                "peak_source": pk["source"], "vs_8TBs_spec": round(achieved_gbs / 8000.0, 4)}
    clocks = sampler.summary()

    components = None
    if rank == 0 and world == 1 and not args.no_components:
        components = {"lm_head_896x151936": component_lm_head(qmm, step, pk["hbm_gbs"]),
                      ("decode_step_121_gemv" if args.schedule == "multi" else "decode_step_gate_up_multi"):
                          component_step_schedule(qmm, step, "gemv" if args.schedule == "multi" else "multi",
                                                  pk["hbm_gbs"]),
                      "decode_step_per_k_q8q8": component_step_auto(qmm, step, pk["hbm_gbs"]),
                      "single_gemv_896x1152": component_single_gemv(qmm, pk["hbm_gbs"]),
                      "q4_gateup_m8_k5120_n17408": component_gateup(qmm, pk["hbm_gbs"]),
                      "q8q8_gemv": component_q8q8(qmm, pk["hbm_gbs"]),
                      "q4_gemv": component_q4_gemv(qmm, pk["hbm_gbs"]),
                      "prefill": component_prefill(qmm, pk)}

    cpu = None
    if want_cpu:
        cpu = cpu_baseline(step.host_w, step.host_x, step.shapes)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOAD, "M": 1, "weight_format": "Q8_0", "bytes_per_step": bytes_step,
                           "l2": "inputs larger than L2 (524,833,792 weight bytes per step; no flush)",
                           "launch": (("CUDA graph of 121 qmm_q8_gemv_ex calls" if args.schedule == "gemv" else
                                       "CUDA graph of 97 calls: qkv, wo, down, lm_head by qmm_q8_gemv_ex, gate + up "
                                       "of each layer by one qmm_q8_gemv_multi")
                                      + ", programmatic dependent launch, QMM_FLAG_EARLY_WEIGHTS"),
                           "parallelism": f"dp{world} (independent decode per rank)"},
                "GB_s": round(achieved_gbs, 1), "roofline": roofline, "clocks": clocks,
                "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h,
                        "how": "pinned host activations copied in, graph replay, logits copied out, every step"},
                "gpu_launches": launches * args.steps, "cpu_baseline": cpu, "components": components}
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
