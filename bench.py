"""Benchmark of the W4A4 + low-rank linear layer on B200.

One step = one pass of the whole hot path (kernel 1: smoothing + NVFP4 activation quantization +
low-rank down-projection; kernel 2: block-scaled FP4 GEMM + up-projection + epilogue) over every
linear of the workload, on seeded synthetic inputs already resident in HBM. L2 is flushed (a 256 MB
write) between timed steps, outside the timed events. Timing: CUDA events on the launching stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl svdq|reference]
                  [--dynamic-scale] [--lora R] [--no-fp8r] [--no-cpu-baseline] [--l2-clean]

On one GPU the line also carries the row-wise FP8 variant of the same workload, measured in a
child process under the same protocol (``fp8r_variant``), and for the MLP workloads the chain with
the down layer's kernel 1 fused into the gate/up GEMM's epilogue (``mlp_fused``).

N > 1 runs under torchrun as independent replicas (the layer has no exchange step), weak scaling.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_diffusion_transformer_svdquant_b200 import synth  # noqa: E402

METRIC = "W4A4+low-rank linear TFLOPS, % of B200 dense FP4 peak; tokens/s per layer"
DEFAULT_WORKLOAD = "qkv_2048"
FP4_PER_BF16 = 4.0   # nominal dense FP4 / dense bf16 tensor throughput on B200 (9 / 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0   # nominal dense FP8 / dense bf16 (4.5 / 2.25 PFLOP/s)
FLUSH_BYTES = 256 << 20
# DRAM bytes (read + write) per launch of the GEMM, from the ncu capture summarised in
# profiles/pair_gemm_kernel_qkv2048.md, keyed by a hash of the code of the kernel sources it was
# taken on (comments excluded); any change to that code makes the figure stale and it is reported
# as null.
PROFILED_GEMM_TRAFFIC = {("qkv_2048", "a23f28693bc5"): 50.25e6 + 259.95e6}
# The same for kernel 1 (profiles/quant_act_kernel_qkv2048.md), keyed by a hash of its source.
PROFILED_K1_TRAFFIC = {("qkv_2048", "20785f4e459c"): 104.06e6 + 6.59e6}


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs (read-only)."""

    def __init__(self, index: int, period_s: float = 0.001):
        self.index, self.period, self.samples, self.reasons = index, period_s, [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: clocks are reported as unavailable
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {"hw_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
                 "hw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
                 "sw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
                 "sw_power_cap": getattr(nv, "nvmlClocksThrottleReasonSwPowerCap", 0x4)}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for k, bit in names.items():
                    if mask & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def code_hash(files) -> str:
    """Hash of the code of kernel sources: every line with its // comment and surrounding blanks
    removed, blank lines dropped, so that a change to comments alone keeps a profiled figure valid."""
    import hashlib
    import re
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "bit_diffusion_transformer_svdquant_b200", "csrc", f)) as fh:
            for line in fh:
                code = re.sub(r"//.*", "", line).strip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:12]


def gemm_source_hash() -> str:
    return code_hash(("svdq_gemm.cuh", "svdq_ptx.cuh"))


def k1_source_hash() -> str:
    return code_hash(("svdq_quant.cuh", "svdq_ptx.cuh"))


def max_over_ranks(value: float, device) -> float:
    """Largest value over all ranks (the slowest replica sets the time)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def layer_flops(spec):
    """(2MNK, 2Mr(K+N)): the FP4 contraction and the whole low-rank branch (down- and up-projection)."""
    return 2.0 * spec.M * spec.N * spec.K, 2.0 * spec.M * spec.r * (spec.K + spec.N)


def gemm_kernel_flops(spec):
    """Method FLOPs inside the GEMM kernel: the FP4 contraction 2MNK plus the branch's up-projection
    2MrN (the down-projection 2MKr runs in kernel 1)."""
    return 2.0 * spec.M * spec.N * spec.K + 2.0 * spec.M * spec.r * spec.N


def kernel1_bytes(spec):
    """Algorithmic HBM bytes of kernel 1: read X (bf16), write codes + scales + U (bf16 hi and lo)."""
    return spec.M * spec.K * 2 + spec.M * spec.K // 2 + spec.M * spec.K // 16 + spec.M * spec.r * 4


# ---------------------------------------------------------------------------------------------- GPU arm
def build_layers(wl, dev, lora=0):
    import bit_diffusion_transformer_svdquant_b200 as svdq
    from bit_diffusion_transformer_svdquant_b200.prepare import concat_lora, prepare_layer

    layers = []
    prev_out = None
    for li, spec in enumerate(wl.layers):
        d = synth.make_linear_inputs(spec)
        chained = wl.name.startswith("mlp") and prev_out is not None
        X = prev_out if chained else d["X"].to(dev)
        p = prepare_layer(X, d["W"].to(dev), spec.r, dev)
        if lora:
            # a synthetic LoRA adapter on the branch: A ~ N(0, 1/K), B ~ N(0, 0.05^2), seeded
            g = torch.Generator().manual_seed(1000 + li)
            A = torch.randn(spec.K, lora, generator=g, dtype=torch.float64) / spec.K ** 0.5
            B = torch.randn(lora, spec.N, generator=g, dtype=torch.float64) * 0.05
            p = concat_lora(p, A, B)
            spec = dataclasses.replace(spec, r=spec.r + lora)
        w = svdq.PackedWeight(p["R"], p["L1s"], p["L2"], p["inv_lambda"], swiglu=spec.swiglu)
        del p
        g_x = svdq.calibrate_act(X, w)
        act = svdq.QuantizedAct(spec.M, spec.K, spec.r, dev)
        bias = d["bias"].to(dev) if spec.bias else None
        n_out = spec.N // 2 if spec.swiglu else spec.N
        Y = torch.empty(spec.M, n_out, dtype=torch.bfloat16, device=dev)
        # the layer's dense bf16 weight [N, K] for the cuBLAS baseline
        layers.append({"spec": spec, "X": X, "w": w, "g_x": g_x, "act": act, "bias": bias, "Y": Y,
                       "W_dense": d["W"].to(dev)})
        if wl.name.startswith("mlp"):
            svdq.quantize_act(X, w, g_x, act)
            svdq.gemm(act, w, bias, out=Y)
            prev_out = Y
    torch.cuda.synchronize(dev)
    return layers


def run_step(layers, dynamic=False):
    import bit_diffusion_transformer_svdquant_b200 as svdq
    for L in layers:
        if dynamic:
            svdq.calibrate_act(L["X"], L["w"], out=L["g_x"])
        svdq.quantize_act(L["X"], L["w"], L["g_x"], L["act"])
        svdq.gemm(L["act"], L["w"], L["bias"], out=L["Y"])


def baseline_step(layers):
    """The same layer(s) in plain bf16 through cuBLAS: y = X W^T + bias (SiLU(gate) * up for SwiGLU)."""
    for L in layers:
        y = torch.nn.functional.linear(L["X"], L["W_dense"], L["bias"])
        if L["spec"].swiglu:
            h = y.shape[1] // 2
            y = torch.nn.functional.silu(y[:, :h]) * y[:, h:]


def flush_l2(flush, clean=None):
    """The L2 flush between timed steps (outside the events): write `flush`, 256 MB > L2. With
    `clean` (a second 256 MB buffer) also read that afterwards, so that the step starts with clean
    L2 lines rather than up to ~126 MB of dirty flush lines that its first kernel writes back."""
    flush.zero_()
    if clean is not None:
        torch.sum(clean, dtype=torch.int64)


def time_per_step(fn, steps, flush, stream, clean=None):
    """Mean CUDA-event time of fn() over `steps` runs, with the L2 flushed (outside the events)
    before each."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush_l2(flush, clean)
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)


def two_pass(run, n_marks, K, flush, stream, dev, clean=None, wall=None):
    """Times K steps of run(mark) twice under the L2-flush protocol (flush outside the events).

    Pass 1 records events only at the step boundaries, with mark a no-op: the step time. An event
    between two kernels on the stream costs a few microseconds of drain before the next launch and
    keeps the next kernel from starting while the previous one finishes, so none is recorded there.
    Pass 2 records an event at every mark(j), j = 0 .. n_marks - 1, which run calls after each of
    its kernels: their durations. Returns (mean step ms of pass 1, [mean ms from the step start to
    mark 0, from mark 0 to mark 1, ...] of pass 2, clock record of pass 1). With `wall` (a list),
    the host wall time of pass 1 is appended to it."""
    se = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t0 = time.perf_counter()
        for e0, e1 in se:
            flush_l2(flush, clean)
            e0.record(stream)
            run(lambda j: None)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        if wall is not None:
            wall.append(time.perf_counter() - t0)
    step_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in se)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks + 1)] for _ in range(K)]
    for row in ev:
        flush_l2(flush, clean)
        row[0].record(stream)
        run(lambda j, row=row: row[j + 1].record(stream))
    torch.cuda.synchronize(dev)
    parts = [statistics.mean(row[j].elapsed_time(row[j + 1]) for row in ev) for j in range(n_marks)]
    return step_ms, parts, clk.summary()


def gpu_arm(args, rank, world, dev):
    import bit_diffusion_transformer_svdquant_b200 as svdq

    wl = synth.WORKLOADS[args.workload]
    layers = build_layers(wl, dev, lora=args.lora)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev) if args.l2_clean else None
    stream = torch.cuda.current_stream(dev)

    dyn = args.dynamic_scale
    for _ in range(args.warmup):
        run_step(layers, dynamic=dyn)
    torch.cuda.synchronize(dev)
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out during warm-up")

    K = args.steps
    n_l = len(layers)
    per = 3 if dyn else 2   # marks per layer: [after the amax pass,] after kernel 1, after the GEMM

    def run(mark):
        for i, L in enumerate(layers):
            if dyn:
                svdq.calibrate_act(L["X"], L["w"], out=L["g_x"])
                mark(per * i)
            svdq.quantize_act(L["X"], L["w"], L["g_x"], L["act"])
            mark(per * i + per - 2)
            svdq.gemm(L["act"], L["w"], L["bias"], out=L["Y"])
            mark(per * i + per - 1)

    if world > 1:
        torch.distributed.barrier()
    wall = []
    step_ms, parts, clocks = two_pass(run, per * n_l, K, flush, stream, dev, clean, wall)
    if world > 1:
        torch.distributed.barrier()
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out during the timed region")
    t_wall = wall[0]
    total_ms = step_ms * K
    kc_ms = [parts[per * i] if dyn else 0.0 for i in range(n_l)]
    k1_ms = [parts[per * i + per - 2] for i in range(n_l)]
    k2_ms = [parts[per * i + per - 1] for i in range(n_l)]
    split_ms = sum(parts)
    total_ms = max_over_ranks(total_ms, dev)

    flops_main = sum(layer_flops(L["spec"])[0] for L in layers)
    flops_lr = sum(layer_flops(L["spec"])[1] for L in layers)
    tokens = layers[0]["spec"].M
    ms_per_step = total_ms / K
    value = world * flops_main / (ms_per_step * 1e-3) / 1e12

    # dominant kernel: the GEMM of the largest layer
    big = max(range(n_l), key=lambda i: layer_flops(layers[i]["spec"])[0])
    spec_b = layers[big]["spec"]
    k2_avg = k2_ms[big]
    peaks = read_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    gemm_flops = gemm_kernel_flops(spec_b)
    achieved = gemm_flops / (k2_avg * 1e-3) / 1e12
    k1_avg = k1_ms
    k1_gbs = [kernel1_bytes(layers[i]["spec"]) / (k1_avg[i] * 1e-3) / 1e9 for i in range(n_l)]
    big1 = max(range(n_l), key=lambda i: kernel1_bytes(layers[i]["spec"]))

    e2e = e2e_arm(args, layers, dev, world)

    # The same steps after a flush that leaves clean lines (the 256 MB write followed by a 256 MB
    # read): kernel 1, the first kernel of a step, then does not also write back the write-flush's
    # dirty lines. Reported beside the headline, which keeps the plain write-flush.
    clean_side = None
    if clean is None:
        clean_buf = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        c_ms, c_parts, _ = two_pass(run, per * n_l, min(K, 50), flush, stream, dev, clean_buf)
        del clean_buf
        c_k1 = [c_parts[per * i + per - 2] for i in range(n_l)]
        c_k2 = [c_parts[per * i + per - 1] for i in range(n_l)]
        c_ms = max_over_ranks(c_ms, dev)
        clean_side = {
            "ms_per_step": round(c_ms, 5),
            "frac_fp4_peak_e2e": round(flops_main / (c_ms * 1e-3) / 1e12 / fp4_peak, 4),
            "quantize_act_us": [round(x * 1e3, 2) for x in c_k1],
            "quantize_act_frac_hbm": [round(kernel1_bytes(layers[i]["spec"]) / (c_k1[i] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
                                      for i in range(n_l)],
            "gemm_us": [round(x * 1e3, 2) for x in c_k2],
            "what": "the same steps with a 256 MB read after each 256 MB write-flush (outside the events), so "
                    "that each step starts on clean L2 lines"}
        if svdq.device_status() != 0:
            raise RuntimeError("device wait ran out in the clean-flush pass")

    # The same step replayed from a CUDA graph (both kernels of every layer captured once), and the
    # bf16 cuBLAS baseline on the same shapes; same timing protocol, fewer steps.
    side_steps = max(3, min(K, 50))
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        run_step(layers, dynamic=dyn)
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_step(layers, dynamic=dyn)
    graph.replay()
    graph_ms = time_per_step(graph.replay, side_steps, flush, stream, clean)
    del graph
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out in the graph replays")
    for _ in range(3):
        baseline_step(layers)
    base_ms = time_per_step(lambda: baseline_step(layers), side_steps, flush, stream, clean)
    graph_ms = max_over_ranks(graph_ms, dev)
    base_ms = max_over_ranks(base_ms, dev)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3/16) + bf16 low-rank, fp32 acc",
        "data": "synthetic (seeded; FLUX-class token counts)",
        "config": {"workload": wl.name, "description": wl.description,
                   "layers": [f"{L['spec'].M}x{L['spec'].K}x{L['spec'].N} r={L['spec'].r}"
                              + (" swiglu" if L["spec"].swiglu else "") + (" bias" if L["spec"].bias else "")
                              for L in layers],
                   "l2": "flushed between timed steps (256 MB write" + (", then a 256 MB read" if args.l2_clean else "")
                         + ", outside the events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "lora_rank": args.lora,
                   "activation_scale": "dynamic (amax pass every step)" if dyn else "static (calibrated once)"},
        "tokens_per_s": round(world * tokens / (ms_per_step * 1e-3), 1),
        "tflops_incl_lowrank": round(world * (flops_main + flops_lr) / (ms_per_step * 1e-3) / 1e12, 2),
        "frac_fp4_peak_e2e": round(value / world / fp4_peak, 4),
        "kernels": {
            "quantize_act_us": [round(x * 1e3, 2) for x in k1_avg],
            "quantize_act_gbs": [round(x, 1) for x in k1_gbs],
            "quantize_act_frac_hbm": [round(x / peaks["hbm_gbs"], 4) for x in k1_gbs],
            "gemm_us": [round(k2_ms[i] * 1e3, 2) for i in range(n_l)],
            "step_us_with_an_event_after_each_kernel": round(split_ms * 1e3, 2),
            **({"dynamic_scale_us": [round(kc_ms[i] * 1e3, 2) for i in range(n_l)]} if dyn else {}),
        },
        "roofline": {"bound": "tensor", "kernel": "pair_gemm_kernel<Nvfp4Gemm>", "achieved": round(achieved, 1),
                     "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / fp4_peak, 4),
                     "traffic": PROFILED_GEMM_TRAFFIC.get((wl.name, gemm_source_hash())),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                     "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {FP4_PER_BF16}"
                                    " (nominal dense FP4/bf16 ratio)",
                     "algorithmic": f"{gemm_flops / 1e9:.1f} GFLOP per launch (2MNK + 2MrN)"},
        "roofline_kernel1": {"bound": "hbm", "kernel": "quant_act_kernel", "achieved": round(k1_gbs[big1], 1),
                             "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
                             "frac": round(k1_gbs[big1] / peaks["hbm_gbs"], 4),
                             "traffic": PROFILED_K1_TRAFFIC.get((wl.name, k1_source_hash())),
                             "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                             "peak_source": f"{peaks['source']} HBM copy bandwidth",
                             "algorithmic": f"{kernel1_bytes(layers[big1]['spec']) / 1e6:.1f} MB per launch "
                                            "(2MK + MK/2 + MK/16 + 4Mr: X read; codes, scales, U hi/lo written)"},
        "e2e": e2e,
        "cuda_graph": {"value": round(world * flops_main / (graph_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                       "ms_per_step": round(graph_ms, 5), "steps": side_steps,
                       "what": "the timed step (kernel 1 + GEMM of every layer) captured once and replayed"},
        "bf16_cublas_baseline": {"value": round(world * flops_main / (base_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                                 "ms_per_step": round(base_ms, 5), "steps": side_steps,
                                 "what": "torch.nn.functional.linear in bf16 (cuBLAS) + bias, SiLU(gate)*up for "
                                         "SwiGLU, same shapes",
                                 "speedup_of_this_path": round(base_ms / ms_per_step, 3)},
        "gpu_launches": (4 if dyn else 2) * n_l * K,
        "clocks": clocks,
        "wall_s_timed_region": round(t_wall, 3),
        **({"l2_clean_variant": clean_side} if clean_side is not None else {}),
    }
    return out


E2E_CHUNKS = 8


def e2e_arm(args, layers, dev, world):
    """The same metric through the public API with host buffers: every step copies the first
    layer's X from pinned host memory, runs the layer(s) and copies the last layer's output back to
    pinned host memory. The layer is row-independent and its activation scale static, so the step
    runs as E2E_CHUNKS row chunks (each a normal library call on its rows) in a three-stream
    pipeline: the host-to-device copy of chunk i+1 and the device-to-host copy of chunk i-1 overlap
    the kernels of chunk i (PCIe is full duplex). Timed with CUDA events on the default stream,
    which waits for the last copy of every step."""
    import bit_diffusion_transformer_svdquant_b200 as svdq
    stream = torch.cuda.current_stream(dev)
    M = layers[0]["spec"].M
    X_dev = layers[0]["X"]
    X_host = X_dev.cpu().pin_memory()
    Y_last = layers[-1]["Y"]
    Y_host = torch.empty(Y_last.shape, dtype=Y_last.dtype).pin_memory()
    # row chunks on 128-row boundaries
    step_rows = -(-M // (E2E_CHUNKS * 128)) * 128
    bounds = [(r0, min(M, r0 + step_rows)) for r0 in range(0, M, step_rows)]
    acts = [[svdq.QuantizedAct(r1 - r0, L["spec"].K, L["spec"].r, dev) for L in layers] for r0, r1 in bounds]
    s_h2d, s_cmp, s_d2h = (torch.cuda.Stream(dev) for _ in range(3))
    n = len(bounds)
    ev_h = [torch.cuda.Event() for _ in range(n)]
    ev_c = [torch.cuda.Event() for _ in range(n)]
    ev_d = [torch.cuda.Event() for _ in range(n)]
    first = [True]

    def step():
        for s_ in (s_h2d, s_cmp, s_d2h):
            s_.wait_stream(stream)
        for i, (r0, r1) in enumerate(bounds):
            with torch.cuda.stream(s_h2d):
                if not first[0]:
                    s_h2d.wait_event(ev_c[i])       # the previous step's kernels have read X rows i
                X_dev[r0:r1].copy_(X_host[r0:r1], non_blocking=True)
                ev_h[i].record(s_h2d)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_h[i])
                if not first[0]:
                    s_cmp.wait_event(ev_d[i])       # the previous step's copy has read Y rows i
                x = X_dev[r0:r1]
                for L, a in zip(layers, acts[i]):
                    svdq.quantize_act(x, L["w"], L["g_x"], a)
                    x = svdq.gemm(a, L["w"], L["bias"], out=L["Y"][r0:r1])
                ev_c[i].record(s_cmp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_c[i])
                Y_host[r0:r1].copy_(Y_last[r0:r1], non_blocking=True)
                ev_d[i].record(s_d2h)
        first[0] = False
        for s_ in (s_h2d, s_cmp, s_d2h):
            stream.wait_stream(s_)

    if args.dynamic_scale:
        raise ValueError("the pipelined end-to-end leg needs a static activation scale")
    steps = max(3, min(args.steps, 20))
    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out in the end-to-end loop")
    # the pipelined result against the resident whole-M call (chunks may split kernel 1's K range
    # differently, which changes U's fp32 summation order, so this is a difference, not equality)
    for L in layers:
        svdq.quantize_act(L["X"], L["w"], L["g_x"], L["act"])
        svdq.gemm(L["act"], L["w"], L["bias"], out=L["Y"])
    torch.cuda.synchronize(dev)
    ref = Y_last.float().cpu()
    rel = float((Y_host.float() - ref).abs().max() / ref.abs().max())
    flops = sum(layer_flops(L["spec"])[0] for L in layers)
    return {"value": round(world * flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": X_host.numel() * X_host.element_size(),
            "d2h_bytes_per_step": Y_host.numel() * Y_host.element_size(), "chunks": n,
            "max_rel_diff_vs_resident": rel,
            "what": f"pinned host X -> device -> layer(s) -> pinned host Y, {n} row chunks pipelined over "
                    "three streams (copy in, kernels, copy out)"}


# ---------------------------------------------------------------------------------- row-wise FP8 variant
def fp8r_arm(args, dev):
    """The row-wise FP8 (W8A8) variant of the same workload under the same timing protocol: per layer
    the row-scale and quantizing passes (one call) and the FP8 GEMM. Also a sanity figure: the
    relative error of each layer's bf16 output on its first 256 rows against the unquantized
    product computed by torch in fp32."""
    import bit_diffusion_transformer_svdquant_b200 as svdq
    from bit_diffusion_transformer_svdquant_b200.prepare import prepare_layer

    wl = synth.WORKLOADS[args.workload]
    layers = []
    prev_out = None
    for spec in wl.layers:
        d = synth.make_linear_inputs(spec)
        chained = wl.name.startswith("mlp") and prev_out is not None
        X = prev_out if chained else d["X"].to(dev)
        W_dense = d["W"].to(dev)
        p = prepare_layer(X, W_dense, spec.r, dev)
        w = svdq.Fp8rWeight(p["R"], p["L1s"], p["L2"], p["inv_lambda"], swiglu=spec.swiglu)
        del p
        act = svdq.Fp8rAct(spec.M, spec.K, spec.r, dev)
        bias = d["bias"].to(dev) if spec.bias else None
        n_out = spec.N // 2 if spec.swiglu else spec.N
        Y = torch.empty(spec.M, n_out, dtype=torch.bfloat16, device=dev)
        layers.append({"spec": spec, "X": X, "w": w, "act": act, "bias": bias, "Y": Y, "W_dense": W_dense})
        if wl.name.startswith("mlp"):
            svdq.linear_fp8r(X, w, bias, act=act, out=Y)
            prev_out = Y
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev) if args.l2_clean else None

    def step(mark=lambda j: None):
        for i, L in enumerate(layers):
            svdq.quantize_act_fp8r(L["X"], L["w"], L["act"])
            mark(2 * i)
            svdq.gemm_fp8r(L["act"], L["w"], L["bias"], out=L["Y"])
            mark(2 * i + 1)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out during the FP8 warm-up")
    K, n_l = args.steps, len(layers)
    ms, parts, clocks = two_pass(step, 2 * n_l, K, flush, stream, dev, clean)
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out in the FP8 timed region")
    k1 = [parts[2 * i] for i in range(n_l)]
    k2 = [parts[2 * i + 1] for i in range(n_l)]
    flops_main = sum(layer_flops(L["spec"])[0] for L in layers)
    big = max(range(n_l), key=lambda i: layer_flops(layers[i]["spec"])[0])
    peaks = read_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    achieved = gemm_kernel_flops(layers[big]["spec"]) / (k2[big] * 1e-3) / 1e12
    rel = []
    for L in layers:
        rows = min(256, L["spec"].M)
        ref = L["X"][:rows].float() @ L["W_dense"].float().T
        if L["bias"] is not None:
            ref = ref + L["bias"].float()
        if L["spec"].swiglu:
            h = ref.shape[1] // 2
            ref = torch.nn.functional.silu(ref[:, :h]) * ref[:, h:]
        rel.append(round(float((L["Y"][:rows].float() - ref).norm() / ref.norm()), 5))
    return {"value": round(flops_main / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
            "steps": K, "warmup": args.warmup, "dtype": "fp8 e4m3 row-wise + bf16 low-rank, fp32 acc",
            "kernels": {"quantize_act_us": [round(x * 1e3, 2) for x in k1],
                        "gemm_us": [round(x * 1e3, 2) for x in k2]},
            "roofline": {"bound": "tensor", "kernel": "pair_gemm_kernel<Fp8Gemm>", "achieved": round(achieved, 1),
                         "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4),
                         "traffic": None,
                         "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s x "
                                        f"{FP8_PER_BF16} (nominal dense FP8/bf16 ratio)",
                         "algorithmic": f"{gemm_kernel_flops(layers[big]['spec']) / 1e9:.1f} GFLOP per launch "
                                        "(2MNK + 2MrN)"},
            "rel_err_vs_unquantized_first_rows": rel,
            "gpu_launches": 3 * n_l * K, "clocks": clocks,
            "what": "the same workload through the row-wise FP8 kernels (row-scale pass, quantizing pass, "
                    "kind::f8f6f4 GEMM), run in a separate process"}


def fp8r_side(args):
    """fp8r_arm in a child process (see child_side)."""
    return child_side(args, "--fp8r-only")


# ------------------------------------------------------------------ MLP chain with kernel 1 fused
def mlp_fused_arm(args, dev):
    """The MLP workload with the down layer's kernel 1 fused into the gate/up GEMM's SwiGLU epilogue:
    per step kernel 1 of the gate/up layer, the fused GEMM (+ its small finalize pass) and the down
    GEMM; h does not cross HBM. Same timing protocol. Also the relative difference of the down
    layer's output from the unfused chain's, on the same inputs and scales."""
    import bit_diffusion_transformer_svdquant_b200 as svdq

    wl = synth.WORKLOADS[args.workload]
    up, dn = build_layers(wl, dev)                # the unfused chain: h -> Y of the first layer
    scratch = torch.empty(svdq._lib.lib().svdq_mlp_scratch_bytes(up["spec"].M, dn["spec"].r), dtype=torch.uint8,
                          device=dev)
    act_dn = svdq.QuantizedAct(dn["spec"].M, dn["spec"].K, dn["spec"].r, dev)
    Y = torch.empty_like(dn["Y"])
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev) if args.l2_clean else None

    def step(mark=lambda j: None):
        svdq.quantize_act(up["X"], up["w"], up["g_x"], up["act"])
        mark(0)
        svdq.gemm_swiglu_quant(up["act"], up["w"], up["bias"], dn["w"], dn["g_x"], act_dn, scratch)
        mark(1)
        svdq.gemm(act_dn, dn["w"], dn["bias"], out=Y)
        mark(2)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out during the fused warm-up")
    # the unfused chain on the same inputs and scales, for the difference figure
    run_step([up, dn])
    torch.cuda.synchronize(dev)
    ref = dn["Y"].float()
    diff = float((Y.float() - ref).norm() / ref.norm())
    K = args.steps
    ms, part, clocks = two_pass(step, 3, K, flush, stream, dev, clean)
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out in the fused timed region")
    # the unfused chain (kernel 1 + GEMM per layer, h through HBM) under the same protocol
    unf = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for s in range(K):
        flush_l2(flush, clean)
        unf[s][0].record(stream)
        run_step([up, dn])
        unf[s][1].record(stream)
    torch.cuda.synchronize(dev)
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out in the unfused timed region")
    ms_unf = statistics.mean(a.elapsed_time(b) for a, b in unf)
    flops = layer_flops(up["spec"])[0] + layer_flops(dn["spec"])[0]
    return {"value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
            "unfused_ms_per_step": round(ms_unf, 5), "saving_us": round((ms_unf - ms) * 1e3, 2),
            "steps": K, "warmup": args.warmup,
            "kernels_us": {"quantize_act_up": round(part[0] * 1e3, 2), "gemm_swiglu_quant": round(part[1] * 1e3, 2),
                           "gemm_down": round(part[2] * 1e3, 2)},
            "rel_diff_vs_unfused_chain": round(diff, 7), "gpu_launches": 4 * K, "clocks": clocks,
            "what": "gate/up GEMM with the down layer's kernel 1 fused into its SwiGLU epilogue, then the down "
                    "GEMM; run in a separate process"}


def config_row_arm(args, dev):
    """Compact figures of one workload under the main protocol (write-flush between steps, CUDA
    events): the side table of the other workloads in the default line."""
    import bit_diffusion_transformer_svdquant_b200 as svdq
    wl = synth.WORKLOADS[args.workload]
    layers = build_layers(wl, dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        run_step(layers)
    torch.cuda.synchronize(dev)
    K, n_l = args.steps, len(layers)

    def run(mark):
        for i, L in enumerate(layers):
            svdq.quantize_act(L["X"], L["w"], L["g_x"], L["act"])
            mark(2 * i)
            svdq.gemm(L["act"], L["w"], L["bias"], out=L["Y"])
            mark(2 * i + 1)

    ms, parts, _ = two_pass(run, 2 * n_l, K, flush, stream, dev)
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out")
    # the same step captured once in a CUDA graph and replayed, under the same protocol: where the
    # layer is small, the launches are a visible part of the step
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        run_step(layers)
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_step(layers)
    graph.replay()
    graph_ms = time_per_step(graph.replay, K, flush, stream)
    del graph
    if svdq.device_status() != 0:
        raise RuntimeError("device wait ran out in the graph replays")
    k1 = [parts[2 * i] for i in range(n_l)]
    k2 = [parts[2 * i + 1] for i in range(n_l)]
    peaks = read_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    flops = sum(layer_flops(L["spec"])[0] for L in layers)
    value = flops / (ms * 1e-3) / 1e12
    return {"value": round(value, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
            "frac_fp4_peak_e2e": round(value / fp4_peak, 4),
            "tokens_per_s": round(layers[0]["spec"].M / (ms * 1e-3), 1),
            "quantize_act_us": [round(x * 1e3, 2) for x in k1],
            "quantize_act_frac_hbm": [round(kernel1_bytes(L["spec"]) / (x * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
                                      for L, x in zip(layers, k1)],
            "gemm_us": [round(x * 1e3, 2) for x in k2],
            "gemm_frac_fp4_peak": [round(gemm_kernel_flops(L["spec"]) / (x * 1e-3) / 1e12 / fp4_peak, 4)
                                   for L, x in zip(layers, k2)],
            "cuda_graph_ms_per_step": round(graph_ms, 5),
            "steps": K}


SIDE_WORKLOADS = ("tiny", "qkv_1024", "mlp_1024", "edit_2048")


def configs_side(args):
    """config_row_arm for every other workload, each in a child process."""
    out = {}
    for name in SIDE_WORKLOADS:
        if name != args.workload:
            out[name] = child_side(args, "--config-row-only", workload=name)
    return out


def child_side(args, flag, workload=None):
    """An arm of this script in a child process (its own CUDA context and a time limit), so that
    nothing in it can affect the main measurement; any failure comes back as {"error": ...}."""
    cmd = [sys.executable, os.path.abspath(__file__), flag, "--workload", workload or args.workload,
           "--steps", str(max(3, min(args.steps, 50))), "--warmup", "3"] + (["--l2-clean"] if getattr(args, "l2_clean", False) else [])
    try:
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
        lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
        if r.returncode != 0 or not lines:
            return {"error": f"exit {r.returncode}: {(r.stderr or r.stdout)[-600:]}"}
        return json.loads(lines[-1])
    except Exception as e:  # a time-out or an unparsable line: reported, never raised
        return {"error": repr(e)[:600]}


# ---------------------------------------------------------------------------------------------- CPU oracle
def oracle_setup(wl, rows_hint=64):
    """The oracle's offline preparation for every layer of the workload (not timed)."""
    from oracle import svdquant
    prepared = []
    for spec in wl.layers:
        d = synth.make_linear_inputs(spec)
        X, W = synth.bf16_values(d["X"]), synth.bf16_values(d["W"])
        p = svdquant.prepare_layer(X, W, spec.r)
        g_x = svdquant.calibrate_activation_scale(X, p["inv_lambda"])
        wq = svdquant.quantize_weight(p["R"])
        b = synth.bf16_values(d["bias"]) if spec.bias else None
        prepared.append({"spec": spec, "X": X, "p": p, "g_x": g_x, "wq": wq, "b": b})
    return prepared


def oracle_step(prepared, rows):
    from oracle import svdquant
    for P in prepared:
        svdquant.layer_forward(P["X"][:rows], P["p"], P["g_x"], P["wq"], P["b"], P["spec"].swiglu)


def choose_rows(prepared, target_s):
    """Rows of the workload whose oracle forward takes about target_s on this host (the per-call
    weight decode is a fixed cost, so the time is fitted as a + b * rows from two trials)."""
    M = prepared[0]["spec"].M
    oracle_step(prepared, 32)  # warm caches and BLAS threads
    ts = []
    for rows in (64, 256):
        t0 = time.perf_counter()
        oracle_step(prepared, rows)
        ts.append(time.perf_counter() - t0)
    b = max((ts[1] - ts[0]) / 192.0, 1e-6)
    a = max(ts[0] - 64 * b, 0.0)
    return int(max(16, min(M, (target_s - a) / b)))


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"), default=0)
        if n:
            return n
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline(wl, target_s=15.0):
    prepared = oracle_setup(wl)
    rows = choose_rows(prepared, target_s)
    from oracle import svdquant
    t0 = time.perf_counter()
    oracle_step(prepared, rows)
    dt = time.perf_counter() - t0
    # the activation-quantization part of the same forward on its own (numpy, vectorised); the
    # rest is weight decode, the fp64 GEMMs (BLAS) and the epilogue
    t0 = time.perf_counter()
    for P in prepared:
        svdquant.quantize_activations(P["X"][:rows], P["p"]["inv_lambda"], P["g_x"])
    dq = time.perf_counter() - t0
    flops = sum(2.0 * rows * P["spec"].N * P["spec"].K for P in prepared)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{rows} of {prepared[0]['spec'].M} token rows through every layer of {wl.name} "
                      f"(fp64 numpy oracle, weights prepared offline), {dt:.1f} s",
            "split_s": {"quantize_activations": round(dq, 2), "gemm_and_rest": round(max(dt - dq, 0.0), 2)}}


def reference_arm(args):
    wl = synth.WORKLOADS[args.workload]
    prepared = oracle_setup(wl)
    rows = choose_rows(prepared, target_s=min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_step(prepared, rows)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(prepared, rows)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    flops = sum(2.0 * rows * P["spec"].N * P["spec"].K for P in prepared)
    value = flops / (ms * 1e-3) / 1e12
    sample = (f"{rows} of {prepared[0]['spec'].M} token rows per step through every layer of {wl.name} "
              f"(fp64 numpy oracle on host cores)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": wl.name, "description": wl.description},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="svdq", choices=["svdq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dynamic-scale", action="store_true",
                    help="compute the activation scale from each step's X (an extra amax pass)")
    ap.add_argument("--lora", type=int, default=0,
                    help="rank of a synthetic LoRA adapter concatenated onto each layer's branch")
    ap.add_argument("--no-fp8r", action="store_true", help="skip the row-wise FP8 side measurement")
    ap.add_argument("--l2-clean", action="store_true",
                    help="after each 256 MB write-flush also read 256 MB, so steps start with clean L2 lines")
    ap.add_argument("--fp8r-only", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--mlp-fused-only", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--config-row-only", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--no-side-configs", action="store_true",
                    help="skip the side table of the other workloads")
    ap.add_argument("--no-mlp-fused", action="store_true",
                    help="skip the fused-chain side measurement of the MLP workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.fp8r_only:
        print(json.dumps(fp8r_arm(args, dev)), flush=True)
        return
    if args.mlp_fused_only:
        print(json.dumps(mlp_fused_arm(args, dev)), flush=True)
        return
    if args.config_row_only:
        print(json.dumps(config_row_arm(args, dev)), flush=True)
        return
    if world > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    try:
        out = gpu_arm(args, rank, world, dev)
        if rank == 0:
            if world == 1 and not args.no_fp8r:
                out["fp8r_variant"] = fp8r_side(args)
            if world == 1 and not args.no_mlp_fused:
                # the MLP chain with the down layer's kernel 1 fused, on this workload if it is an
                # MLP, else on the 1024^2 MLP
                mlp_wl = args.workload if args.workload.startswith("mlp") else "mlp_1024"
                out["mlp_fused"] = {"workload": mlp_wl, **child_side(args, "--mlp-fused-only", workload=mlp_wl)}
            if world == 1 and not args.no_side_configs:
                out["configs"] = configs_side(args)
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(synth.WORKLOADS[args.workload])
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
