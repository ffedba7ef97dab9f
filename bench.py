"""Benchmark of the MoE expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Default workload: decode, T = 1 token through 40 distinct seeded layers
(H 2048, I 512, 256 experts top-8 + 1 shared, 4-bit group 64), 18.2 GB of
packed weights resident and cycled, so every step streams its weights from
HBM (inputs larger than L2; no flush needed).  One step = the whole hot path
(route, permute, expert FFN, combine) of all 40 layers, replayed as one CUDA
graph.  A second, smaller measurement covers the T = 2048 prefill layer, and
a report-only one the T = 8 (H 512), T = 512 Zipf-skewed and T = 16384
hot-expert layers (``other_configs``, L2 flushed between iterations).

Prints one JSON line on rank 0.  Under torchrun every rank runs its own
replica (weak scaling, no collective on the data path); the time is the max
over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

LAYERS = 40
UNIT = "tokens/s"
METRIC = "MoE expert-layer tokens/s (layer passes per second, T=1 decode over 40 layers)"

# Algorithmic bytes of one decode layer-token (H 2048, I 512, G 64): each of
# the 9 active experts (8 routed + shared) streams its packed gate_up and down
# codes plus (scale, bias) pairs once; activations are 2 KB-scale.
H, I, E, K, G = 2048, 512, 256, 8, 64
EXPERT_BYTES = (2 * I * H + H * I) // 2 + (2 * I * (H // G) + H * (I // G)) * 4
ROUTER_BYTES = E * H * 2
FFN_BYTES_T1 = 9 * EXPERT_BYTES + H * 2 + H * 4      # + x (bf16) + y_acc (fp32)
LAYER_BYTES_T1 = FFN_BYTES_T1 + ROUTER_BYTES


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=mx, reasons=sorted(reasons), samples=0)
        return dict(sm_mhz=float(np.median(sm)), sm_max_mhz=mx, reasons=sorted(reasons), samples=len(sm))


# ------------------------------------------------------------ distributed


# Kernel sources whose ncu summaries under profiles/ carry DRAM traffic per launch.
KERNEL_SOURCES = {
    "ffn_decode": ["bit_dequant_expert_b200/csrc/ffn_decode.cu"],
    "ffn_tc": ["bit_dequant_expert_b200/csrc/ffn_tc.cu"],
}
KERNEL_HEADERS = ["bit_dequant_expert_b200/csrc/common.cuh", "bit_dequant_expert_b200/csrc/ptx.cuh",
                  "bit_dequant_expert_b200/csrc/topk.cuh", "bit_dequant_expert_b200/csrc/kernels.h"]


def kernel_source_hash(name: str) -> str:
    """sha256 over the code of a kernel's source file and the headers it
    includes: `//` comments, trailing blanks and empty lines do not count."""
    import hashlib
    import re
    h = hashlib.sha256()
    root = os.path.dirname(os.path.abspath(__file__))
    for rel in KERNEL_SOURCES[name] + KERNEL_HEADERS:
        with open(os.path.join(root, rel)) as f:
            for line in f:
                code = re.sub(r"(^|\s)//.*$", "", line).rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()


def profiled_traffic(name: str, summary: str):
    """DRAM bytes (read + write) per launch from profiles/<summary>, or None when
    the summary is missing or the kernel's sources changed since it was taken."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", summary)
    try:
        fields = dict(line.split(":", 1) for line in open(path).read().splitlines() if ":" in line)
    except OSError:
        return None
    if fields.get("source_sha256", "").strip() != kernel_source_hash(name):
        return None
    try:
        return int(fields["traffic_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def aggregate(local_ms: float, local_units: float, world: int):
    """(max time over ranks, total units over ranks); collectives only when world > 1."""
    if world <= 1:
        return local_ms, local_units
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    u = torch.tensor([local_units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------- oracle timing


def cpu_model() -> str:
    """The host CPU's model name from /proc/cpuinfo (empty if unreadable)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def omp_threads() -> int:
    try:
        import ctypes
        return int(ctypes.CDLL("libgomp.so.1").omp_get_max_threads())
    except OSError:
        return os.cpu_count() or 1


def time_oracle_decode(layers: list, budget_s: float):
    """Layer-tokens/s of the oracle on the first layers (T = 1 each), within about budget_s."""
    import oracle
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.layer(layers[done % len(layers)])
        done += 1
        if time.perf_counter() - t0 >= budget_s and done >= 1:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def _omp_set_threads(n: int) -> None:
    import ctypes
    ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))


def time_oracle_layer(lay: dict, budget_s: float):
    """Tokens/s of the oracle on a prefix of the layer's tokens (with its
    logit bias): the prefix doubles from 1 token while the next call is
    expected to fit in budget_s; returns (rate, tokens, seconds) of the last
    call."""
    import oracle
    T = lay["x"].shape[0]
    n, spent, last = 1, 0.0, None
    while True:
        tok = np.arange(n, dtype=np.int32)
        t0 = time.perf_counter()
        oracle.layer(lay, tokens=tok)
        dt = time.perf_counter() - t0
        spent += dt
        last = (n / dt, n, dt)
        if n >= T or spent + 2.2 * dt > budget_s:
            return last
        n = min(2 * n, T)


def time_oracle_other_configs(budget_s: float, ids=(0, 2, 4), single_thread=(0, 2)):
    """The oracle's layer tokens/s on each configuration, on all OpenMP
    threads and, for the smaller ones, on one thread."""
    import gen
    out = {}
    full = omp_threads()
    for cid in ids:
        lay = gen.make_layer(gen.config(cid))
        runs = [("all", full)] + ([("1", 1)] if cid in single_thread else [])
        out[str(cid)] = {}
        for label, nt in runs:
            _omp_set_threads(nt)
            try:
                rate, n, dt = time_oracle_layer(lay, budget_s)
            finally:
                _omp_set_threads(full)
            out[str(cid)][label] = {"value": rate, "unit": UNIT, "cores": nt, "cpu": cpu_model(), "kind": "oracle",
                                    "sample": "first %d of %d tokens in one call, %.2f s" % (n, lay["x"].shape[0], dt)}
    return out


# ------------------------------------------------------------- workloads


def build_decode(device):
    """40 seeded layers resident on the device; returns (layers, host copies of the first 3)."""
    import gen
    from bit_dequant_expert_b200.layer import MoELayer, to_device
    spec = gen.config(1)
    layers, host = [], []
    x_all = np.empty((LAYERS, H), dtype=np.uint16)
    for l in range(LAYERS):
        lay = gen.make_layer(spec, l)
        layers.append(MoELayer(lay, max_tokens=1, device=device))
        x_all[l] = lay["x"][0]
        if l < 3:
            host.append(lay)
        del lay
    x_dev = to_device(x_all, device)
    return layers, host, x_dev, x_all


def _timed_replays(replay, n, stream):
    """Device time (ms) of n calls of replay() on stream, CUDA events on that stream."""
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(n):
        replay()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


def _capture(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def _launch_count(layer, T):
    """Kernels one forward() of the layer launches: two for the fused decode
    layer (moe_decode_layer), else the four calls' count."""
    import bit_dequant_expert_b200 as m
    if layer.fused_ok(T):
        return 2
    return m.moe_launch_count(layer.cfg, T, layer.mode, layer.path)


def run_decode(device, steps, warmup, world, peaks):
    import torch
    layers, host, x_dev, x_host = build_decode(device)
    y_dev = torch.empty(LAYERS, H, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.Stream(device=device)

    def step():
        for l in range(LAYERS):
            layers[l].forward(x_dev[l:l + 1], y_out=y_dev[l:l + 1])

    def ffn_only():
        for l in range(LAYERS):
            layers[l].expert_ffn(x_dev[l:l + 1], 1)

    with torch.cuda.stream(stream):
        step()                       # eager pass: sets kernel attributes before capture
        ffn_only()
    torch.cuda.synchronize()
    g_step = _capture(step, stream)
    g_ffn = _capture(ffn_only, stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g_step.replay()
            g_ffn.replay()
    torch.cuda.synchronize()

    # whole-path timing (clock samples cover a pre-roll, the timed region and a post-roll)
    sampler = ClockSampler(device.index or 0)
    sampler.start()
    with torch.cuda.stream(stream):
        roll = max(1, int(0.6 / max(_timed_replays(g_step.replay, 3, stream) / 3e3, 1e-6)))
        _timed_replays(g_step.replay, roll, stream)
        barrier(world)
        torch.cuda.synchronize()
        total_ms = _timed_replays(g_step.replay, steps, stream)
        barrier(world)
        _timed_replays(g_step.replay, roll, stream)
    clocks = sampler.stop()
    ms_step = total_ms / steps

    # the expert FFN kernel on its own (moe_expert_ffn, 40 launches per replay of its
    # own graph): not part of the step, reported beside the step's roofline
    with torch.cuda.stream(stream):
        ffn_ms = _timed_replays(g_ffn.replay, steps, stream) / (steps * LAYERS)
    achieved = FFN_BYTES_T1 / (ffn_ms * 1e-3) / 1e9
    roofline_ffn = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"],
                    "traffic": profiled_traffic("ffn_decode", "ffn_decode_t1_ncu.txt"),
                    "kernel": "k_decode<0> (moe_expert_ffn at T=1: gate/up + SwiGLU, then down + vector reductions into y_acc)",
                    "algorithmic_bytes": FFN_BYTES_T1, "avg_launch_us": ffn_ms * 1e3,
                    "peak_source": peaks["source"] + " hbm_gbs"}

    # end to end through the public API: pinned host x -> device, 40 layers, y -> pinned host
    x_pin = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_pin = torch.empty(LAYERS, H, dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        x_dev.copy_(x_pin, non_blocking=True)
        g_step.replay()
        y_pin.copy_(y_dev, non_blocking=True)
        stream.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            e2e_step()
        e2e_ms = _timed_replays(e2e_step, steps, stream) / steps
    e2e = {"value": LAYERS / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": LAYERS * H * 2,
           "d2h_bytes_per_step": LAYERS * H * 2, "ms_per_step": e2e_ms}

    # the step's dominant work, timed over the timed region above: per layer pass the fused
    # decode kernel (route + permute + expert FFN) and its combine, router + expert bytes
    layer_bytes = LAYER_BYTES_T1
    layer_us = ms_step * 1e3 / LAYERS
    layer_gbs = layer_bytes / (layer_us * 1e-6) / 1e9
    roofline = {"bound": "hbm", "achieved": layer_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": layer_gbs / peaks["hbm_gbs"],
                "traffic": profiled_traffic("ffn_decode", "decode_layer_t1_ncu.txt"),
                "kernel": "moe_decode_layer: k_decode<1> (route + permute + expert FFN) + k_combine_scatter",
                "algorithmic_bytes": layer_bytes, "avg_layer_us": layer_us, "launches_per_layer": 2,
                "traffic_note": "ncu DRAM bytes of the layer kernel's launch",
                "peak_source": peaks["source"] + " hbm_gbs"}
    breakdown = _breakdown(layers, [x_dev[l:l + 1] for l in range(LAYERS)], 1, steps, stream)
    launches = _launch_count(layers[0], 1) * LAYERS
    return {"ms_per_step": ms_step, "units_per_step": LAYERS * 1, "roofline": roofline,
            "roofline_ffn": roofline_ffn, "e2e": e2e,
            "clocks": clocks, "gpu_launches": launches * steps, "breakdown_us_per_layer": breakdown,
            "_host_layers": host}


def _breakdown(layers, xs, T, steps, stream):
    """Device time per layer of each of the four calls, each captured alone (us)."""
    import torch
    parts = {
        "route": lambda: [L.route(x, T) for L, x in zip(layers, xs)],
        "permute": lambda: [L.permute(T) for L in layers],
        "expert_ffn": lambda: [L.expert_ffn(x, T) for L, x in zip(layers, xs)],
        "combine": lambda: [L.combine(T) for L in layers],
    }
    out = {}
    for name, fn in parts.items():
        g = _capture(fn, stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
            out[name] = 1e3 * _timed_replays(g.replay, steps, stream) / (steps * len(layers))
    return out


def run_prefill(device, steps, warmup, world, peaks):
    """T = 2048 prefill layer (uniform router): tokens/s and the expert-FFN tensor roofline."""
    import torch
    import gen
    from bit_dequant_expert_b200 import MOE_MODE_PAIRS
    from bit_dequant_expert_b200.layer import MoELayer, to_device
    spec = gen.config(3)
    lay = gen.make_layer(spec)
    T = spec.T
    # pairs mode: the down GEMM writes bf16 rows, the combine sums them in slot order
    L = MoELayer(lay, max_tokens=T, device=device, mode=MOE_MODE_PAIRS)
    x = to_device(lay["x"], device)
    del lay
    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        L.forward(x)
    torch.cuda.synchronize()
    g = _capture(lambda: L.forward(x), stream)
    gf = _capture(lambda: L.expert_ffn(x, T), stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        ms = _timed_replays(g.replay, steps, stream) / steps
        for _ in range(warmup):
            gf.replay()
        ffn_ms = _timed_replays(gf.replay, steps, stream) / steps
    breakdown = _breakdown([L], [x], T, steps, stream)
    rows = (K + 1) * T
    flops = 2.0 * rows * (2 * I * H + H * I)
    tflops = flops / (ffn_ms * 1e-3) / 1e12
    wbytes = (E + 1) * EXPERT_BYTES
    return {"workload": "prefill: T=2048, uniform router (H 2048, I 512, E 256 top-8 + shared, G 64)",
            "value": T / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "ffn_ms": ffn_ms,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops"],
                         "traffic": profiled_traffic("ffn_tc", "ffn_tc_prefill_t2048_ncu.txt"),
                         "kernel": "moe_expert_ffn (T=2048)", "algorithmic_flops": flops,
                         "peak_source": peaks["source"] + " bf16_tflops (burst)",
                         "hbm_frac_of_weight_bytes": wbytes / (ffn_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "gpu_launches_per_step": _launch_count(L, T),
            "breakdown_us": breakdown,
            "l2": "inputs larger than L2 (455.8 MB of packed weights per layer)"}


def run_expert_parallel(device, steps, warmup, world, rank, peaks):
    """The expert-parallel layer (bit_dequant_expert_b200.ep): T = 2048 tokens
    per rank, 256/N experts per rank, NCCL all-to-alls between ranks.  Timed
    with CUDA events on the current stream around `steps` calls; each call
    synchronises the host twice (the row counts set the exchange splits)."""
    import torch
    import gen
    from bit_dequant_expert_b200 import ep
    spec = gen.config(3)
    T = spec.T
    weights = gen.make_weights(spec, 0)                  # the same layer on every rank
    x_host = gen.make_activations(spec, rank)["x"]       # each rank its own tokens
    ops = ep.CudaEPOps(ep.shard_weights(weights, world, rank), spec.E, world, max_tokens=T, device=device)
    del weights
    L = ep.ExpertParallelLayer(ops, E=spec.E)
    x = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).to(device)
    for _ in range(warmup):
        L.forward(x)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        y = L.forward(x)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    barrier(world)
    # end to end: pinned host x in, y out, every step
    x_pin = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_pin = torch.empty(T, spec.H, dtype=torch.bfloat16).pin_memory()
    s.record()
    for _ in range(steps):
        x.copy_(x_pin, non_blocking=True)
        y = L.forward(x)
        y_pin.copy_(y, non_blocking=True)
    e.record()
    torch.cuda.synchronize()
    e2e_ms = s.elapsed_time(e) / steps
    errs = ops.device_errors()
    return {"ms_per_step": ms, "e2e_ms": e2e_ms, "T": T, "device_errors": errs,
            "recv_rows": L.last["recv"], "send_rows": L.last["send"],
            "bytes_per_step": {"h2d": int(x_pin.numel() * 2), "d2h": int(y_pin.numel() * 2)}}


FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # 148 SMs x 128 fp32 lanes x fma x clocks.max.sm


def run_gdn(device, steps, warmup, peaks):
    """The Gated DeltaNet scan (gdn_scan, one launch per layer): decode
    (8 sequences x 1 token) and verification (1 sequence x 4 tokens) steps
    over 30 layers with a state each, updated in place step after step, and
    a 2048-token prefill of one layer.  CUDA graph of a step, CUDA events on
    its stream."""
    import torch
    import gen
    import bit_dequant_expert_b200 as m

    def dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    out = {}
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    for name, ci in (("decode", 1), ("verify", 2), ("prefill", 3)):
        spec = gen.scan_config(ci)
        B, T, Hk, Hv, dk, dv = spec.B, spec.T, spec.Hk, spec.Hv, spec.dk, spec.dv
        layers = []
        for l in range(spec.layers):
            d = gen.make_scan(spec, l)
            t = {n: dev(d[n]) for n in ("q", "k", "v", "g", "beta", "S0")}
            t["o"] = torch.empty(B, T, Hv, dv, dtype=torch.bfloat16, device=device)
            t["scale"] = d["scale"]
            layers.append(t)
        stream = torch.cuda.Stream(device=device)

        def step():
            for t in layers:
                m.gdn_scan(B, T, Hk, Hv, dk, dv, t["q"], t["k"], t["v"], t["g"], t["beta"], t["scale"], t["S0"],
                           t["S0"], t["o"])

        with torch.cuda.stream(stream):
            step()
        torch.cuda.synchronize()
        g = _capture(step, stream)
        state_bytes = B * Hv * dv * dk * 4
        io_bytes = 2 * B * T * Hk * dk * 2 + 2 * B * T * Hv * dv * 2 + 2 * B * T * Hv * 4
        per_layer = 2 * state_bytes + io_bytes
        resident = spec.layers * state_bytes
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                g.replay()
            n = max(steps, 3)
            if resident < 2 * 126 * 2 ** 20:
                ms = _timed_flushed(g.replay, n, stream, lambda: flush_buf.zero_()) / n
                l2 = "L2 flushed between timed steps (256 MB write outside the events)"
            else:
                ms = _timed_replays(g.replay, n, stream) / n
                l2 = "inputs larger than L2 (%.0f MB of state per step)" % (resident / 2 ** 20)
        us_layer = ms * 1e3 / spec.layers
        gbs = per_layer / (us_layer * 1e-6) / 1e9
        flops = 7.0 * B * T * Hv * dv * dk
        tflops = flops / (us_layer * 1e-6) / 1e12
        r = {"workload": "%s: B=%d sequences x T=%d tokens, Hk %d, Hv %d, dk %d, dv %d, %d layer%s" %
                         (name, B, T, Hk, Hv, dk, dv, spec.layers, "s" if spec.layers > 1 else ""),
             "tokens_per_s": B * T / (ms * 1e-3), "ms_per_step": ms, "us_per_layer": us_layer,
             "gpu_launches_per_step": spec.layers, "l2": l2,
             "algorithmic_bytes_per_layer": per_layer, "algorithmic_flops_per_layer": flops}
        if name == "prefill":
            r["roofline"] = {"bound": "alu", "achieved": tflops, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                             "frac": tflops / FP32_PEAK_TFLOPS,
                             "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1.965 GHz",
                             "note": "one token after another: 2048 dependent steps per state row"}
        else:
            r["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "peak_source": peaks["source"] + " hbm_gbs"}
        out[name] = r
        del layers, g
        torch.cuda.synchronize()
    return out


def expert_bytes(h: int, i: int, g: int = G) -> int:
    """Packed bytes of one expert: gate/up [2i, h] and down [h, i] 4-bit codes
    plus one bf16 (scale, bias) pair per group of g inputs."""
    return (2 * i * h + h * i) // 2 + (2 * i * (h // g) + h * (i // g)) * 4


def _timed_flushed(replay, n, stream, flush):
    """Device time (ms) of n calls of replay(), each bracketed by its own CUDA
    events on stream, with flush() (an L2-sized write) between them outside
    the events."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize()
    for s, e in ev:
        flush()
        s.record(stream)
        replay()
        e.record(stream)
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in ev)


def other_config_specs() -> dict:
    """The remaining synthetic workloads, each (layer spec, layer index): the
    T=8 small case (H 512, I 128), the Zipf-skewed T=512 layer and the
    T=16384 layer with half its tokens biased onto 8 hot experts."""
    import gen
    return {str(c): (gen.config(c), 0) for c in (0, 2, 4)}


def small_t_specs() -> dict:
    """Decode-layer shapes (H 2048, I 512) with a few tokens, as speculative
    decoding's verification batches: 2-8 tokens through the decode kernel
    (weights read = the union of the selected experts), and 16 tokens, past
    the crossover to the tensor-core kernel."""
    import gen
    return {"T%d" % t: (gen.config(1).with_T(t), 3) for t in (2, 4, 8, 16)}


def run_other_configs(device, steps, warmup, peaks, specs=None):
    """Report-only layer measurements of `specs` (default: other_config_specs()).
    Scatter mode, the default implementation path, L2 flushed between
    iterations.  Each reports layer tokens/s, the expert-FFN time, its HBM
    fraction on the bytes of the experts the routing activated (with the
    shared expert) and its bf16 tensor fraction."""
    import torch
    import gen
    from bit_dequant_expert_b200 import MOE_MODE_SCATTER
    from bit_dequant_expert_b200.layer import MoELayer, to_device
    import bit_dequant_expert_b200 as m
    stream = torch.cuda.Stream(device=device)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    out = {}
    for cid, (spec, layer_index) in (specs or other_config_specs()).items():
        lay = gen.make_layer(spec, layer_index)
        T, h, i = spec.T, spec.H, spec.I
        L = MoELayer(lay, max_tokens=T, device=device, mode=MOE_MODE_SCATTER)
        x = to_device(lay["x"], device)
        bias = lay["logit_bias"]
        stride = int(lay["bias_stride"])
        bias_t = None if bias is None else to_device(bias, device)
        del lay

        def fwd():
            L.forward(x, logit_bias=bias_t, bias_stride=stride)

        def ffn():
            L.expert_ffn(x, T)

        with torch.cuda.stream(stream):
            fwd()
        torch.cuda.synchronize()
        err = m.moe_get_device_error(L.ws)
        active = int((L.counts > 0).sum().item())
        g_fwd, g_ffn = _capture(fwd, stream), _capture(ffn, stream)
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                g_fwd.replay()
                g_ffn.replay()
            flush = lambda: flush_buf.zero_()
            ms = _timed_flushed(g_fwd.replay, steps, stream, flush) / steps
            ffn_ms = _timed_flushed(g_ffn.replay, steps, stream, flush) / steps
        rows = (K + 1) * T
        flops = 2.0 * rows * (2 * i * h + h * i)
        wbytes = (active + 1) * expert_bytes(h, i)
        out[cid] = {
            "workload": "%s (T=%d, layer %d)" % (spec.name, T, layer_index), "T": T,
            "value": T / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "ffn_ms": ffn_ms, "steps": steps, "device_error": err, "active_experts": active,
            "hbm_frac_active_weight_bytes": wbytes / (ffn_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "tensor_frac": flops / (ffn_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "algorithmic_flops": flops, "active_weight_bytes": wbytes,
            "gpu_launches_per_step": _launch_count(L, T),
            "l2": "flushed between timed iterations (256 MB write outside the events)"}
        del L, x, bias_t, g_fwd, g_ffn
        torch.cuda.synchronize()
    return out


def run_ncu_case(case, device, calls):
    """One layer for a profiler: route + permute, then `calls` launches of the kernel under study."""
    import torch
    import gen
    if case.startswith("gdn"):
        import bit_dequant_expert_b200 as m
        spec = gen.scan_config(1 if case == "gdn-decode" else 3)
        d = gen.make_scan(spec, 0)
        t = {}
        for n in ("q", "k", "v", "g", "beta", "S0"):
            a = np.ascontiguousarray(d[n])
            t[n] = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16
                    else torch.from_numpy(a)).to(device)
        o = torch.empty(spec.B, spec.T, spec.Hv, spec.dv, dtype=torch.bfloat16, device=device)
        for _ in range(calls):
            m.gdn_scan(spec.B, spec.T, spec.Hk, spec.Hv, spec.dk, spec.dv, t["q"], t["k"], t["v"], t["g"],
                       t["beta"], d["scale"], t["S0"], t["S0"], o)
        torch.cuda.synchronize()
        print(json.dumps({"ncu_case": case, "calls": calls}))
        return 0
    import bit_dequant_expert_b200 as m
    from bit_dequant_expert_b200 import MOE_MODE_PAIRS, MOE_MODE_SCATTER
    from bit_dequant_expert_b200.layer import MoELayer, to_device
    prefill = case.startswith("prefill")
    # split-t16: 16 tokens of the decode layer shape through the split path (the tensor-core
    # kernel for the shared expert, the decode kernel's row-list launch for the others)
    spec = gen.config(3) if prefill else gen.config(1).with_T(16) if case == "split-t16" else gen.config(1)
    lay = gen.make_layer(spec, 3 if case == "split-t16" else 0)
    T = spec.T
    L = MoELayer(lay, max_tokens=T, device=device,
                 mode=MOE_MODE_PAIRS if prefill else MOE_MODE_SCATTER)
    x = to_device(lay["x"], device)
    del lay
    L.route(x, T)
    L.permute(T)
    for _ in range(calls):
        if case in ("decode-layer", "prefill-layer"):
            L.forward(x)
        else:
            L.expert_ffn(x, T)
    torch.cuda.synchronize()
    print(json.dumps({"ncu_case": case, "calls": calls, "device_error": m.moe_get_device_error(L.ws)}))
    return 0


DECODE_WORKLOAD = "decode: T=1 x 40 distinct layers cycled (H 2048, I 512, E 256 top-8 + shared, G 64)"


def decode_config(world: int) -> dict:
    """The decode workload's config (the same for both arms)."""
    return {
        "workload": DECODE_WORKLOAD,
        "global_batch": world,
        "seq_len": 1,
        "parallelism": "replicas" if world > 1 else "single GPU",
        "l2": "inputs larger than L2 (18.2 GB of weights streamed per step; no flush)",
        "graph": "one CUDA graph per step (40 layers x moe_decode_layer: decode kernel + combine)",
    }


def decode_line(res: dict, ms: float, units: float, world: int, steps: int, warmup: int, peaks: dict) -> dict:
    """The JSON line of the decode measurement: `ms` is the slowest rank's
    time per step, `units` the layer passes all ranks made per step, `res`
    what run_decode measured."""
    return {
        "metric": METRIC,
        "value": units / (ms / 1e3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 (4-bit weights, fp32 accumulation)",
        "data": "synthetic (seeded; SplitMix64 layers shaped like the pages' model)",
        "config": decode_config(world),
        "decode_token_per_s": world / (ms / 1e3),
        "breakdown_us_per_layer": res["breakdown_us_per_layer"],
        "gpu_launches": res["gpu_launches"],
        "roofline": res["roofline"],
        "roofline_ffn": res["roofline_ffn"],
        "e2e": res["e2e"],
        "clocks": res["clocks"],
        "peaks": peaks,
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-prefill", action="store_true", help="skip the T=2048 prefill measurement")
    ap.add_argument("--no-gdn", action="store_true", help="skip the Gated DeltaNet scan measurement")
    ap.add_argument("--expert-parallel", action="store_true",
                    help="measure the expert-parallel layer (256/N experts per rank, T=2048 per rank, all-to-all "
                         "exchanges; its line replaces the decode line)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="measure only the T=2048 prefill layer (its line replaces the decode line)")
    ap.add_argument("--ncu-case", choices=("decode-ffn", "decode-layer", "prefill-ffn", "prefill-layer", "gdn-decode",
                                                   "gdn-prefill", "split-t16"),
                    help="a small case for a profiler capture: one synthetic layer, route + permute, then "
                         "--steps calls of the named kernel (decode: config 1 layer 0, T=1; prefill: "
                         "config 3, T=2048); prints the device error word and nothing timed")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle CPU baseline")
    ap.add_argument("--other-configs", choices=("on", "off", "only"), default="on",
                    help="report-only layer measurements of the T=8 (H 512), T=512 Zipf and T=16384 hot-expert "
                         "workloads, and of decode-layer shapes with 2-16 tokens: 'on' adds them to the line "
                         "(other_configs, small_t), 'only' prints just them")
    args = ap.parse_args(argv)
    warmup = max(args.warmup, 3)
    world, rank, local = dist_env()

    if args.impl == "reference":
        return run_reference(args, world, rank, warmup)

    import torch
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()

    if args.ncu_case:
        return run_ncu_case(args.ncu_case, device, max(args.steps, 1))

    if args.other_configs == "only":
        oc = run_other_configs(device, max(args.steps // 10, 5), warmup, peaks)
        st = run_other_configs(device, max(args.steps // 10, 5), warmup, peaks, small_t_specs())
        if rank == 0:
            print(json.dumps({"other_configs": oc, "small_t": st, "peaks": peaks}), flush=True)
        if world > 1:
            import torch.distributed as dist
            barrier(world)
            dist.destroy_process_group()
        return 0

    if args.expert_parallel:
        r = run_expert_parallel(device, max(args.steps // 10, 5), warmup, world, rank, peaks)
        ms, units = aggregate(r["ms_per_step"], r["T"], world)
        e2e_ms, _ = aggregate(r["e2e_ms"], r["T"], world)
        line = {"metric": "MoE expert-layer tokens/s (expert parallel, T=2048 per rank)",
                "value": units / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": max(args.steps // 10, 5),
                "warmup": warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16 (4-bit weights, fp32 accumulation)",
                "data": "synthetic (seeded; SplitMix64 layers shaped like the pages' model)",
                "config": {"workload": "prefill: T=2048 per rank, uniform router, 256/N experts per rank "
                                       "(H 2048, I 512, E 256 top-8 + shared, G 64)",
                           "global_batch": 2048 * world, "seq_len": 2048, "parallelism": "ep%d" % world,
                           "l2": "inputs larger than L2 (455.8 MB of packed weights per layer over all ranks)"},
                "e2e": {"value": units / (e2e_ms / 1e3), "unit": UNIT,
                        "h2d_bytes_per_step": r["bytes_per_step"]["h2d"],
                        "d2h_bytes_per_step": r["bytes_per_step"]["d2h"]},
                "rows_sent_per_rank_last_call": r["send_rows"], "device_errors": r["device_errors"],
                "peaks": peaks}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            barrier(world)
            dist.destroy_process_group()
        return 0

    if args.prefill_only:
        pre = run_prefill(device, max(args.steps, 1), warmup, world, peaks)
        ms, units = aggregate(pre["ms_per_step"], 2048, world)
        line = {"metric": "MoE expert-layer tokens/s (T=2048 prefill layer)", "value": units / (ms / 1e3),
                "unit": UNIT, "n_gpus": world, "steps": pre["steps"], "warmup": warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16 (4-bit weights, fp32 accumulation)",
                "data": "synthetic (seeded; SplitMix64 layers shaped like the pages' model)",
                "config": {"workload": pre["workload"], "global_batch": 2048 * world, "seq_len": 2048,
                           "parallelism": "replicas" if world > 1 else "single GPU", "l2": pre["l2"]},
                "roofline": pre["roofline"], "gpu_launches": pre["gpu_launches_per_step"] * pre["steps"],
                "breakdown_us": pre["breakdown_us"], "peaks": peaks}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            barrier(world)
            dist.destroy_process_group()
        return 0

    res = run_decode(device, args.steps, warmup, world, peaks)
    pre = None if args.no_prefill else run_prefill(device, max(args.steps // 10, 5), warmup, world, peaks)

    ms, units = aggregate(res["ms_per_step"], res["units_per_step"], world)
    line = decode_line(res, ms, units, world, args.steps, warmup, peaks)
    if args.other_configs == "on":
        line["other_configs"] = run_other_configs(device, max(args.steps // 10, 5), warmup, peaks)
        line["small_t"] = run_other_configs(device, max(args.steps // 10, 5), warmup, peaks, small_t_specs())
    if rank == 0 and world == 1:
        budget = args.cpu_budget
        layers_host = res.pop("_host_layers")
        rate, n, dt = time_oracle_decode(layers_host, budget)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": omp_threads(), "cpu": cpu_model(),
                                "kind": "oracle",
                                "sample": "%d layer passes (T=1) of the first decode layers, %.1f s" % (n, dt)}
        if "other_configs" in line:
            for cid, cpu in time_oracle_other_configs(budget / 4).items():
                line["other_configs"][cid]["cpu_baseline"] = cpu
    if not args.no_gdn:
        line["gdn_scan"] = run_gdn(device, max(args.steps // 10, 5), warmup, peaks)
    if pre is not None:
        # last key of the line, so that a reader keeping only the line's tail still sees it
        line["prefill_t2048"] = pre
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()
    return 0


def run_reference(args, world, rank, warmup):
    """The reference arm: the CPU oracle on this host's cores, same metric."""
    if rank != 0:
        return 0
    import gen
    spec = gen.config(1)
    layers = [gen.make_layer(spec, l) for l in range(3)]
    per_step = []
    total_t = time.perf_counter()
    for s in range(warmup + args.steps):
        t0 = time.perf_counter()
        # one bounded sample step: one layer pass of T = 1 (of the 40-layer workload)
        import oracle
        oracle.layer(layers[s % len(layers)])
        if s >= warmup:
            per_step.append(time.perf_counter() - t0)
        if time.perf_counter() - total_t > 150:
            break
    ms = 1e3 * float(np.mean(per_step)) if per_step else float("nan")
    value = 1e3 / ms
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": len(per_step),
        "warmup": warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic (seeded)",
        "config": decode_config(world),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": omp_threads(), "cpu": cpu_model(), "kind": "oracle",
                         "sample": "one layer pass (T=1) per step, layers 0-2 cycled"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
