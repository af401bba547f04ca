"""Benchmark of the BitNest nested W4/W8 linear layer on B200.

One step = the decode hot path over the seven Llama-3-8B-shaped projections
(q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096, down 4096x14336, group
128): for every projection the draft pass (activation quantise + W4A8 linear
at M = 1, hi plane only) and the verify pass (quantise + W8A8 linear at
M = 4 = gamma + 1, hi and lo planes); o_proj activations are quantised per
128-group.  Inputs are seeded synthetic tensors of those shapes, resident in
HBM.  The metric is HBM throughput: the algorithmic bytes the step must move
(weights, scales, activations, outputs) divided by the device time.

Also reported: the dominant kernel against the HBM roofline, an end-to-end
number with host buffers (activation upload and output download inside the
timed region), and the CPU oracle timed on a bounded sample of the same work.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
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
sys.path.insert(0, ROOT)

from w8_quantized_linear_b200 import synth  # noqa: E402

METRIC = "HBM GB/s and % of 8 TB/s for draft/target GEMV; int8 TOPS % peak at prefill"
UNIT = "GB/s"
N_COPIES = 4  # rotating weight copies: 4 x 218 MB of planes, far above the 126 MB L2
DECODE_M = {0: 1, 1: 4}  # draft at M = 1, target (verify) at M = gamma + 1 = 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def linear_bytes(mode, M, N, K):
    """Algorithmic bytes of one linear launch: planes read once (hi, or hi and
    lo), fp16 group scales, int8 activations and their fp32 scales, fp32 output."""
    G = K // 128
    planes = (1 if mode == 0 else 2) * N * K // 2
    return planes + 2 * N * G + M * K + 4 * M + 4 * M * N


def quant_bytes(M, K, act_group):
    """fp16 activations read; int8 codes and their fp32 scales written."""
    G = K // 128
    return 2 * M * K + M * K + 4 * (M if act_group == 0 else M * G)


def fused_bytes(mode, M, N, K, act_group):
    """Algorithmic bytes of one quantise + linear call (bitnest_quantize_linear
    without an xsum buffer: the layer forms the group sums itself): planes,
    fp16 group scales, fp16 activations read; int8 codes, their scales and
    the fp32 output written."""
    G = K // 128
    planes = (1 if mode == 0 else 2) * N * K // 2
    return planes + 2 * N * G + quant_bytes(M, K, act_group) + 4 * M * N


class ClockSampler:
    """NVML samples of SM clock and throttle reasons while the timed region runs."""

    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index, period=0.02):
        self.samples = []
        self.reasons = set()
        self.period = period
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = device_index
            if vis:
                ids = [v for v in vis.split(",") if v.strip()]
                if device_index < len(ids) and ids[device_index].strip().isdigit():
                    idx = int(ids[device_index])
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # no NVML: clocks are reported as unknown
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        return {
            "sm_mhz": statistics.median(self.samples) if self.samples else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": sorted(self.reasons),
            "samples": len(self.samples),
        }


def dominant_traffic(kernel_tag):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if that summary was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_tag]
        src = os.path.join(ROOT, rec["source"])
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if sha != rec["source_sha"]:
            return None
        return rec["bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


# ---------------------------------------------------------------- workload
# One decoder layer's projections as launched by an inference engine: q|k|v
# share their input and are one fused weight (N = 6144), likewise gate|up
# (N = 28672); o_proj takes per-128-group activation scales.
LAYER_GROUPS = [
    ("qkv", ("q_proj", "k_proj", "v_proj")),
    ("o", ("o_proj",)),
    ("gate_up", ("gate_proj", "up_proj")),
    ("down", ("down_proj",)),
]


def group_shape(members):
    N = sum(synth.LLAMA3_8B_PROJECTIONS[m][0] for m in members)
    K = synth.LLAMA3_8B_PROJECTIONS[members[0]][1]
    g = synth.LLAMA3_8B_PROJECTIONS[members[0]][2]
    return N, K, g


def step_host_inputs():
    """The decode step's seeded inputs on the host: per layer group its
    stacked nibble planes and scales, per (group, pass) its fp16 activations.
    Only the input generators; no arithmetic of the layer."""
    groups, acts = {}, {}
    for gi, (gname, members) in enumerate(LAYER_GROUPS):
        parts = []
        for m in members:
            N, K, _ = synth.LLAMA3_8B_PROJECTIONS[m]
            pid = synth.PROJ_IDS[m]
            parts.append((synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_HI, N, K),
                          synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_LO, N, K),
                          synth.group_scales(synth.SEED_SCALES + pid, N, K)))
        groups[gname] = tuple(np.concatenate([p[i] for p in parts], axis=0) if len(parts) > 1
                              else parts[0][i] for i in range(3))
        N, K, g = group_shape(members)
        for mode, M in DECODE_M.items():
            acts[gname, mode] = synth.activations(synth.SEED_ACTS + 10 * gi + 100 * mode, M, K)
    return groups, acts


def decode_step_bytes():
    """Algorithmic bytes of one decode step (both passes, all layer groups)."""
    tot = 0
    for _, members in LAYER_GROUPS:
        N, K, g = group_shape(members)
        for mode, M in DECODE_M.items():
            tot += fused_bytes(mode, M, N, K, g)
    return tot


class DecodeWorkload:
    """Weights (N_COPIES rotating copies of the fused layer weights, plus one
    unfused copy for per-projection timing), activations and outputs."""

    def __init__(self, device, n_copies=N_COPIES, overlap=True):
        import torch

        import w8_quantized_linear_b200 as bn

        self.bn = bn
        self.overlap = overlap
        self.dev = device
        self.projs = list(synth.LLAMA3_8B_PROJECTIONS.items())
        nib = {}
        for name, (N, K, _) in self.projs:
            pid = synth.PROJ_IDS[name]
            nib[name] = (synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_HI, N, K),
                         synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_LO, N, K),
                         synth.group_scales(synth.SEED_SCALES + pid, N, K))

        def planes(uh, ul, s):
            hi, lo = bn.pack_planes(torch.from_numpy(uh).to(device), torch.from_numpy(ul).to(device))
            return hi, lo, torch.from_numpy(s).to(device)

        self.single = {name: planes(*nib[name]) for name, _ in self.projs}
        del nib
        host_groups, host_acts = step_host_inputs()
        base = {gname: planes(*host_groups[gname]) for gname, _ in LAYER_GROUPS}
        del host_groups
        self.copies = [base] + [{k: tuple(t.clone() for t in v) for k, v in base.items()}
                                for _ in range(1, n_copies)]
        # per layer group and pass: activations and outputs, each a view of one
        # flat device buffer with a pinned host twin, so that the end-to-end
        # step moves its inputs up and its results down in one copy each
        # (every view starts on a 16-byte boundary: M K and M N are multiples of 8)
        shapes = []
        for gi, (gname, members) in enumerate(LAYER_GROUPS):
            N, K, g = group_shape(members)
            for mode, M in DECODE_M.items():
                shapes.append((gi, gname, mode, M, N, K, g))
        nx = sum(M * K for _, _, _, M, _, K, _ in shapes)
        ny = sum(M * N for _, _, _, M, N, _, _ in shapes)
        self.x_flat_host = torch.empty(nx, dtype=torch.float16).pin_memory()
        self.y_flat_host = torch.empty(ny, dtype=torch.float32).pin_memory()
        self.x_flat = torch.empty(nx, dtype=torch.float16, device=device)
        self.y_flat = torch.empty(ny, dtype=torch.float32, device=device)
        self.x, self.x_host, self.bufs = {}, {}, {}
        ox = oy = 0
        for gi, gname, mode, M, N, K, g in shapes:
            xh = self.x_flat_host[ox:ox + M * K].view(M, K)
            xh.copy_(torch.from_numpy(host_acts[gname, mode]))
            self.x_host[gname, mode] = xh
            self.x[gname, mode] = self.x_flat[ox:ox + M * K].view(M, K)
            b = self._bufs(M, N, K, g)
            b["y"] = self.y_flat[oy:oy + M * N].view(M, N)
            b["y_host"] = self.y_flat_host[oy:oy + M * N].view(M, N)
            self.bufs[gname, mode] = b
            ox += M * K
            oy += M * N
        self.x_flat.copy_(self.x_flat_host)
        # unfused per-projection buffers (kernel timing)
        self.pbufs = {}
        for name, (N, K, g) in self.projs:
            pid = synth.PROJ_IDS[name]
            for mode, M in DECODE_M.items():
                x = torch.from_numpy(synth.activations(synth.SEED_ACTS + pid + 100 * mode, M, K))
                self.pbufs[name, mode] = dict(self._bufs(M, N, K, g), x=x.to(device))
        torch.cuda.synchronize()

    def _bufs(self, M, N, K, g):
        import torch

        G = K // 128
        return dict(
            xq=torch.empty((M, K), dtype=torch.int8, device=self.dev),
            xs=torch.empty((M,) if g == 0 else (M, G), dtype=torch.float32, device=self.dev),
            y=torch.empty((M, N), dtype=torch.float32, device=self.dev),
            y_host=torch.empty((M, N), dtype=torch.float32).pin_memory(),
        )

    def step_bytes(self):
        return decode_step_bytes()

    def launches_per_step(self):
        # per layer group and pass, one bitnest_quantize_linear call: the
        # quantiser kernel and the layer kernel
        return 2 * len(DECODE_M) * len(LAYER_GROUPS)

    def io_bytes(self):
        h2d = sum(t.numel() * t.element_size() for t in self.x_host.values())
        d2h = sum(b["y_host"].numel() * 4 for b in self.bufs.values())
        return h2d, d2h

    def _path(self):
        return self.bn.PATH_AUTO | (self.bn.PATH_OVERLAP if self.overlap else 0)

    def run_step(self, copy, events=None, e2e=False):
        """Enqueue one step on the current stream: the draft pass then the
        verify pass, one quantise + linear call (bitnest_quantize_linear) per
        layer group.  `events`: per (group, mode) (start, end) CUDA events
        around the call."""
        bn = self.bn
        w = self.copies[copy]
        if e2e:  # the step's activations, all layer groups and passes, in one upload
            self.x_flat.copy_(self.x_flat_host, non_blocking=True)
        for mode in (0, 1):
            for gname, members in LAYER_GROUPS:
                _, _, g = group_shape(members)
                b = self.bufs[gname, mode]
                x = self.x[gname, mode]
                hi, lo, s = w[gname]
                if events is not None:
                    events[gname, mode][0].record()
                bn.quantize_linear(mode, hi, lo, s, x, g, out=b["y"],
                                   act_out=(b["xq"], b["xs"], None), path=self._path())
                if events is not None:
                    events[gname, mode][1].record()
        if e2e:  # and every output back in one download
            self.y_flat_host.copy_(self.y_flat, non_blocking=True)

    def step_results(self):
        """Host copies of the step's results, per (group, pass): output y,
        int8 activation codes and their fp32 scales."""
        import torch

        torch.cuda.synchronize()
        return {k: (b["y"].cpu().numpy(), b["xq"].cpu().numpy(), b["xs"].cpu().numpy())
                for k, b in self.bufs.items()}

    def run_projection(self, name, mode):
        """One unfused projection: quantise its own input and apply the layer."""
        bn = self.bn
        _, _, g = synth.LLAMA3_8B_PROJECTIONS[name]
        b = self.pbufs[name, mode]
        hi, lo, s = self.single[name]
        return lambda: bn.quantize_linear(mode, hi, lo, s, b["x"], g, out=b["y"],
                                          act_out=(b["xq"], b["xs"], None),
                                          path=self._path())


class EagerStep:
    """Stands in for a captured graph: replay() launches the step directly."""

    def __init__(self, fn):
        self.fn = fn

    def replay(self):
        self.fn()

    def reset(self):
        pass


def capture(fn, eager=False):
    import torch

    if eager:
        fn()
        torch.cuda.synchronize()
        return EagerStep(fn)

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm: first-launch host setup happens outside capture
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        fn()
    torch.cuda.synchronize()
    return g


def timed_replays(graphs, steps, barrier):
    import torch

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    start.record()
    for i in range(steps):
        graphs[i % len(graphs)].replay()
    end.record()
    torch.cuda.synchronize()
    barrier()
    return start.elapsed_time(end) / 1e3  # seconds


# ----------------------------------------------------------------- prefill
PREFILL_M = 2048


def measure_prefill(wl, reps=10):
    """Target W8A8 at M = 2048 through the seven projections on the tcgen05
    path.  Each launch is timed alone with CUDA events after an L2 flush
    (a 256 MB write); returns per-projection and total int8 TOPS."""
    import torch

    bn = wl.bn
    dev = wl.dev
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {}
    tot_ops = 0.0
    tot_t = 0.0
    for name, (N, K, g) in wl.projs:
        pid = synth.PROJ_IDS[name]
        x = torch.from_numpy(synth.activations(synth.SEED_ACTS + pid, PREFILL_M, K)).to(dev)
        xq, xs, xsum = bn.quantize_act(x, g)
        y = torch.empty((PREFILL_M, N), dtype=torch.float32, device=dev)
        hi, lo, sc = wl.single[name]
        bn.linear(1, hi, lo, sc, xq, xs, xsum, g, out=y)  # warm
        t = 0.0
        for _ in range(reps):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            bn.linear(1, hi, lo, sc, xq, xs, xsum, g, out=y)
            b.record()
            torch.cuda.synchronize()
            t += a.elapsed_time(b) / 1e3
        t /= reps
        ops = 2.0 * PREFILL_M * N * K
        res[name] = {"us": round(t * 1e6, 2), "TOPS": round(ops / t / 1e12, 1)}
        tot_ops += ops
        tot_t += t
        del x, xq, xs, xsum, y
    del flush
    return res, tot_ops, tot_t


# -------------------------------------------------------------- CPU oracle
def oracle_step_inputs():
    """The step's inputs as the oracle takes them: packed planes per group."""
    import oracle

    groups, acts = step_host_inputs()
    packed = {g: (oracle.pack_plane(uh), oracle.pack_plane(ul), s)
              for g, (uh, ul, s) in groups.items()}
    return packed, acts


def oracle_step(packed, acts):
    """One decode step by the oracle: per (group, pass) (y, codes, scales)."""
    import oracle

    outs = {}
    for gname, members in LAYER_GROUPS:
        N, K, g = group_shape(members)
        hi, lo, s = packed[gname]
        for mode in DECODE_M:
            q, xs = oracle.quantize(acts[gname, mode], g)
            outs[gname, mode] = (oracle.linear(mode, hi, lo if mode else None, s, q, xs, K, g),
                                 q, xs)
    return outs


def compare_step(outs, results, tol=1e-3):
    """The GPU step's results against the oracle's: activation codes and
    scales bit-exact, every output element within `tol` in the normalised
    error max |y - y_ref| / (|y_ref| + 1e-3 rms(y_ref)).  "ok" or the list
    of failures."""
    import oracle

    bad = []
    for key, (y_ref, q, xs) in outs.items():
        y, xq_gpu, xs_gpu = results[key]
        tag = f"{key[0]}/{'draft' if key[1] == 0 else 'target'}"
        if not (np.array_equal(xq_gpu, q) and np.array_equal(xs_gpu, xs)):
            bad.append(f"{tag}: activation codes differ")
        err = oracle.max_normalised_error(y, y_ref) if y.shape == y_ref.shape else float("inf")
        if not err <= tol:
            bad.append(f"{tag}: output error {err:.3g}")
    return "ok" if not bad else "FAILED: " + "; ".join(bad)


def cpu_baseline(results=None, budget_s=12.0, max_steps=None):
    """The oracle, as it stands, on the host cores: whole decode steps (every
    layer group, both passes, every output row) on the step's own seeded
    inputs, repeated until `budget_s` of CPU work (at least one step, at most
    `max_steps`).  Returns (seconds per step, threads, steps, self_check).

    With `results` (the GPU step's outputs, from DecodeWorkload.step_results)
    the first oracle step also checks them (compare_step)."""
    import oracle

    oracle.build()
    packed, acts = oracle_step_inputs()
    check = None
    times = []
    while True:
        t0 = time.perf_counter()
        outs = oracle_step(packed, acts)
        times.append(time.perf_counter() - t0)
        if results is not None and len(times) == 1:
            check = compare_step(outs, results)
        if sum(times) >= budget_s or (max_steps is not None and len(times) >= max_steps):
            break
    return statistics.median(times), oracle.num_threads(), len(times), check


def measure_decode(args, wl, barrier, max_over_ranks, world, hbm_peak, peak_kind):
    """The timed decode step (CUDA graphs over rotating weight copies), the
    end-to-end variant with host buffers, and per-launch kernel times."""
    import torch

    step_bytes = wl.step_bytes()
    eager = args.no_graph
    graphs = [capture(lambda c=c: wl.run_step(c), eager) for c in range(N_COPIES)]
    e2e_graphs = [capture(lambda c=c: wl.run_step(c, e2e=True), eager) for c in range(N_COPIES)]

    for i in range(args.warmup):
        graphs[i % N_COPIES].replay()
    torch.cuda.synchronize()

    with ClockSampler(torch.cuda.current_device()) as clocks:
        t = timed_replays(graphs, args.steps, barrier)
    t = max_over_ranks(t)
    ms_per_step = 1e3 * t / args.steps
    value = world * step_bytes * args.steps / t / 1e9

    # end to end: activations uploaded from pinned host memory and outputs read back
    for i in range(args.warmup):
        e2e_graphs[i % N_COPIES].replay()
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(timed_replays(e2e_graphs, args.steps, barrier))
    e2e_value = world * step_bytes * args.steps / t_e2e / 1e9
    h2d, d2h = wl.io_bytes()

    # dominant kernel: the verify (target, M = 4) GEMV.  Per-launch device
    # time from CUDA events recorded on the launching stream right around each
    # launch; a spin kernel first lets the host enqueue the whole sequence, so
    # no launch waits on the host between its two events.
    def ev_pairs():
        return {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for k in wl.bufs}

    events = ev_pairs()
    dur = {k: 0.0 for k in events}
    n_ev = max(8, min(args.steps, 200))
    for i in range(n_ev):
        torch.cuda._sleep(4_000_000)
        wl.run_step(i % N_COPIES, events=events)
        torch.cuda.synchronize()
        for k, (a, b) in events.items():
            dur[k] += a.elapsed_time(b) / 1e3
    per_group = {}
    for (gname, mode) in events:
        N, K, g = group_shape(dict(LAYER_GROUPS)[gname])
        d = dur[gname, mode] / n_ev
        b = fused_bytes(mode, DECODE_M[mode], N, K, g)
        per_group[f"{gname}/{'draft' if mode == 0 else 'target'}"] = {
            "N": N, "K": K, "us": round(d * 1e6, 3), "GB/s": round(b / d / 1e9, 1),
            "frac_hbm": round(b / d / 1e9 / hbm_peak, 3)}
    # the dominant launch: the fused gate|up verify (target, M = 4) layer
    dom_N, dom_K, dom_g = group_shape(dict(LAYER_GROUPS)["gate_up"])
    dom_bytes = fused_bytes(1, DECODE_M[1], dom_N, dom_K, dom_g)
    dom_time = dur["gate_up", 1] / n_ev
    achieved = dom_bytes / dom_time / 1e9
    # every projection on its own (unfused): one quantise + layer call per
    # launch, device time per call from a CUDA graph of back-to-back calls
    # over rotating weight copies (each call reads its weights from HBM)
    per_proj = {}
    for name, (N, K, g) in wl.projs:
        copies = weight_copies(wl, N, K, N * K // 2)
        for mode, M in DECODE_M.items():
            pb = wl.pbufs[name, mode]
            t = chained(lambda c: wl.bn.quantize_linear(mode, *copies[c], pb["x"], g, out=pb["y"],
                                                        act_out=(pb["xq"], pb["xs"], None),
                                                        path=wl._path()), copies, reps=5)
            b = fused_bytes(mode, M, N, K, g)
            per_proj[f"{name}/{'draft' if mode == 0 else 'target'}"] = {
                "us": round(t * 1e6, 3), "GB/s": round(b / t / 1e9, 1),
                "frac_hbm": round(b / t / 1e9 / hbm_peak, 3)}
        del copies
    roofline = {
        "bound": "hbm",
        "kernel": f"gemv_tma_kernel<TARGET, M=4>, fused gate|up weights (N={dom_N}, "
                  f"K={dom_K}); the timed call also runs its quantiser launch",
        "achieved": round(achieved, 1),
        "peak": hbm_peak,
        "unit": "GB/s",
        "frac": round(achieved / hbm_peak, 4),
        "peak_kind": f"{peak_kind} (copy bandwidth)",
        "traffic": dominant_traffic("gemv_target_m4_gate_up"),
        "algorithmic_bytes_per_launch": dom_bytes,
        "per_launch_in_step": per_group,
        "per_projection_unfused": per_proj,
        "per_projection_timing": "one quantise + layer call per projection, CUDA graph of "
                                 "back-to-back calls over rotating weight copies, per call",
    }
    for g in graphs + e2e_graphs:
        g.reset()
    return value, ms_per_step, clocks, e2e_value, h2d, d2h, roofline



# ------------------------------------------------------------- M sweep
SWEEP_M = (1, 2, 4, 8, 16, 32, 64, 128)
SWEEP_SHAPES = ("gate_proj", "down_proj")  # 14336 x 4096 and 4096 x 14336


def weight_copies(wl, N, K, nbytes, min_copies=3, max_copies=64):
    """Rotating copies of seeded [N, K] planes and scales, enough that between
    two reads of one copy the others push it out of the 126 MB L2."""
    import torch

    bn = wl.bn
    count = max(min_copies, min(max_copies, -(-160_000_000 // max(nbytes, 1)) + 1))
    uh = torch.from_numpy(synth.nibbles(synth.SEED_WEIGHTS + 50 + N, synth.STREAM_HI, N, K)).to(wl.dev)
    ul = torch.from_numpy(synth.nibbles(synth.SEED_WEIGHTS + 50 + N, synth.STREAM_LO, N, K)).to(wl.dev)
    sc = torch.from_numpy(synth.group_scales(synth.SEED_SCALES + 50 + N, N, K)).to(wl.dev)
    hi, lo = bn.pack_planes(uh, ul)
    del uh, ul
    return [(hi, lo, sc)] + [(hi.clone(), lo.clone(), sc.clone()) for _ in range(count - 1)]


def chained(fn_of_copy, copies, reps=8, per_copy=2):
    """Device time per launch of `fn_of_copy(c)`: a CUDA graph of
    len(copies) * per_copy launches cycling over the copies, CUDA events
    around each replay, median over `reps` replays."""
    import torch

    n = len(copies) * per_copy
    g = capture(lambda: [fn_of_copy(i % len(copies)) for i in range(n)])
    g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    ts = []
    for _ in range(reps):
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / 1e3 / n)
    g.reset()
    return statistics.median(ts)


def measure_sweep(wl, hbm_peak, reps=5):
    """Every M of the batch / verify sweep on the two MLP shapes, both modes:
    the path the library picks, device time per launch from a CUDA graph of
    back-to-back launches over rotating weight copies (each launch reads its
    weights from HBM; the time includes the gap between two launches but not
    the events' own cost), HBM throughput and int8 TOPS."""
    import torch

    bn = wl.bn
    dev = wl.dev
    res = {}
    torch.cuda._sleep(200_000_000)  # about 0.1 s of spinning: clocks up before the first case
    torch.cuda.synchronize()
    for name in SWEEP_SHAPES:
        N, K, g = synth.LLAMA3_8B_PROJECTIONS[name]
        pid = synth.PROJ_IDS[name]
        copies = weight_copies(wl, N, K, N * K // 2, min_copies=6)
        for M in SWEEP_M:
            x = torch.from_numpy(synth.activations(synth.SEED_ACTS + pid + 1000 * M, M, K)).to(dev)
            xq, xs, xsum = bn.quantize_act(x, g)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            for mode in (0, 1):
                path = bn.select_path(mode, M, N, K)
                # scratch for the tensor-core path's split K (few tiles, long K)
                nws = bn.linear_ws_bytes(mode, M, N, K)
                ws = bn.workspace(nws, dev) if nws else None
                t = chained(lambda c: bn.linear_ws(mode, *copies[c], xq, xs, xsum, ws, g, out=y),
                            copies, reps=reps)
                nb = linear_bytes(mode, M, N, K)
                label = "tcgen05 split-K" if nws else (
                    "gemv" if path == bn.PATH_GEMV else "tcgen05")
                res[f"{name}/{'draft' if mode == 0 else 'target'}/M={M}"] = {
                    "path": label,
                    "us": round(t * 1e6, 2), "GB/s": round(nb / t / 1e9, 1),
                    "frac_hbm": round(nb / t / 1e9 / hbm_peak, 3),
                    "TOPS": round(2.0 * M * N * K / t / 1e12, 2)}
            del x, xq, xs, xsum, y
        del copies
    return res


def measure_call_cost(wl, hbm_peak, reps=5):
    """Fixed cost per decode call: t = a + bytes / BW fitted (least squares)
    over K = 4096 layers of N = 1024, 4096, 14336 and 28672 rows, draft
    (M = 1) and target (M = 4), for the layer alone (`bitnest_linear` on
    quantised activations) and for the one-call quantise + layer entry
    (`bitnest_quantize_linear`, the decode step's call).  Device time per
    launch from CUDA graphs over rotating weight copies (`chained`)."""
    import torch

    bn = wl.bn
    dev = wl.dev
    K, g = 4096, 0
    P = bn.PATH_AUTO | bn.PATH_OVERLAP
    pts = {}
    for N in (1024, 4096, 14336, 28672):
        copies = weight_copies(wl, N, K, N * K // 2)
        for mode, M in DECODE_M.items():
            x = torch.from_numpy(synth.activations(synth.SEED_ACTS + 900 + M, M, K)).to(dev)
            xq, xs, _ = bn.quantize_act(x, g)
            ao = (torch.empty_like(xq), torch.empty_like(xs), None)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            t_lin = chained(lambda c: bn.linear(mode, *copies[c], xq, xs, None, g, out=y, path=P),
                            copies, reps=reps)
            t_ql = chained(lambda c: bn.quantize_linear(mode, *copies[c], x, g, out=y, act_out=ao,
                                                        path=P), copies, reps=reps)
            tag = "draft" if mode == 0 else "target"
            pts.setdefault(("layer", tag), []).append((linear_bytes(mode, M, N, K), t_lin, N))
            pts.setdefault(("quantise+layer", tag), []).append(
                (fused_bytes(mode, M, N, K, g), t_ql, N))
        del copies
    res = {}
    for (kind, tag), v in pts.items():
        xb = np.array([b for b, _, _ in v], np.float64)
        yt = np.array([t for _, t, _ in v], np.float64)
        slope, icpt = np.polyfit(xb, yt, 1)
        res[f"{kind}/{tag}"] = {
            "a_us": round(icpt * 1e6, 2), "BW_GB/s": round(1.0 / slope / 1e9, 1),
            "BW_frac_hbm": round(1.0 / slope / 1e9 / hbm_peak, 3),
            "points": {f"N={n}": {"MB": round(b / 1e6, 2), "us": round(t * 1e6, 2),
                                  "frac_hbm": round(b / t / 1e9 / hbm_peak, 3)}
                       for b, t, n in v}}
    return {"workload": "decode calls on K = 4096 layers (N = 1024 .. 28672), draft M = 1, "
                        "target M = 4; fit t = a + bytes / BW",
            "timing": "CUDA graph of back-to-back calls over rotating weight copies, per call",
            "per_kind": res}


# ------------------------------------------- down_proj input: R4 rotation
def measure_hadamard(wl, hbm_peak, reps=10, chain=20):
    """bitnest_hadamard_quantize_act (x H / sqrt(K) + per-token int8) on the
    down_proj input (K = 14336) next to the plain quantiser, at the decode
    batches and the prefill batch.  Device time per launch: a CUDA graph of
    `chain` launches back to back (the decode-size rows stay in L2, as they
    would coming from the preceding kernel), CUDA events around each replay."""
    import torch

    bn = wl.bn
    N, K, _ = synth.LLAMA3_8B_PROJECTIONS["down_proj"]
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    res = {}
    for M in (1, 4, PREFILL_M):
        x = torch.from_numpy(synth.activations(synth.SEED_ACTS + 500 + M, M, K)).to(wl.dev)
        out = (torch.empty((M, K), dtype=torch.int8, device=wl.dev),
               torch.empty((M,), dtype=torch.float32, device=wl.dev),
               torch.empty((M, K // 128), dtype=torch.int32, device=wl.dev))
        nbytes = 2 * M * K + M * K + 4 * M + 4 * M * (K // 128)
        n = chain if M < PREFILL_M else 4
        for name, fn in (("rotate+quantise", lambda: bn.hadamard_quantize_act(x, out=out)),
                         ("quantise", lambda: bn.quantize_act(x, 0, out=out))):
            g = capture(lambda: [fn() for _ in range(n)])
            g.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                a.record()
                g.replay()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) / 1e3 / n)
            g.reset()
            t = statistics.median(ts)
            res[f"{name}/M={M}"] = {"us": round(t * 1e6, 2), "GB/s": round(nbytes / t / 1e9, 1),
                                    "frac_hbm": round(nbytes / t / 1e9 / hbm_peak, 3)}
        del x, out
    return {"workload": "down_proj input (K = 14336 = 28 x 512): online Hadamard rotation "
                        "fused with per-token int8 quantisation, vs the quantiser alone",
            "timing": f"CUDA graph of {chain} launches (4 at M = {PREFILL_M}), per launch",
            "per_case": res}


def attention_bytes(mode, H, Hkv, T, D=128):
    """Algorithmic bytes of one decode-attention launch: the K and V hi planes
    (and lo planes for the target) and their fp16 row scales, the fp16 query,
    the fp32 output."""
    rows = T * Hkv
    planes = (1 if mode == 0 else 2) * 2 * rows * (D // 2)
    return planes + 2 * 2 * rows + 2 * H * D + 4 * H * D


def measure_attention(wl, hbm_peak, reps=10, chain=20):
    """bitnest_nested_attention for one Llama-3-8B decode token (32 query
    heads, 8 KV heads, head_dim 128) over caches of 2048 and 8192 tokens
    (seeded synthetic K / V packed with bitnest_pack_weights), draft (KV4) and
    target (KV8).  Device time per launch: a CUDA graph of `chain` launches
    back to back, CUDA events around its replay (so the per-launch time
    includes the gap between two launches, not the events' own cost)."""
    import torch

    bn = wl.bn
    H, Hkv, D = 32, 8, 128
    gen = torch.Generator(device=wl.dev)
    gen.manual_seed(synth.SEED_ACTS + 700)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    res = {}
    for T in (2048, 8192):
        kv = [torch.randn((T * Hkv, D), generator=gen, device=wl.dev).half() for _ in range(2)]
        kp, vp = bn.pack_weights(kv[0]), bn.pack_weights(kv[1])
        q = torch.randn((H, D), generator=gen, device=wl.dev).half()
        out = torch.empty((H, D), dtype=torch.float32, device=wl.dev)
        for mode in (0, 1):
            g = capture(lambda: [bn.nested_attention(mode, q, kp, vp, Hkv, out=out)
                                 for _ in range(chain)])
            g.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                a.record()
                g.replay()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) / 1e3 / chain)
            g.reset()
            t = statistics.median(ts)
            nb = attention_bytes(mode, H, Hkv, T, D)
            res[f"{'draft' if mode == 0 else 'target'}/T={T}"] = {
                "us": round(t * 1e6, 2), "GB/s": round(nb / t / 1e9, 1),
                "frac_hbm": round(nb / t / 1e9 / hbm_peak, 3)}
        del kv, kp, vp
    return {"workload": "decode attention of one token over a nested KV cache (H=32, Hkv=8, "
                        "D=128), draft reads KV4 (hi planes), target KV8 (hi + lo)",
            "timing": f"CUDA graph of {chain} launches, median of {reps} replays, per launch",
            "per_case": res}


# ------------------------------------------------ packer from fp weights
def measure_pack(wl, hbm_peak, reps=5):
    """bitnest_pack_weights on the seven projections' shapes (seeded
    synthetic fp16 weights, N(0, 0.02^2)): one launch per projection after
    a 256 MB L2 flush.  Bytes: fp16 weights read, both planes and the fp16
    scales written."""
    import torch

    bn = wl.bn
    dev = wl.dev
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(synth.SEED_WEIGHTS)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    res, tot_b, tot_t = {}, 0, 0.0
    for name, (N, K, _) in wl.projs:
        w = (torch.randn((N, K), generator=gen, device=dev, dtype=torch.float32) * 0.02).half()
        out = bn.pack_weights(w)
        t = 0.0
        for _ in range(reps):
            flush.fill_(1)
            a.record()
            bn.pack_weights(w, out=out)
            b.record()
            torch.cuda.synchronize()
            t += a.elapsed_time(b) / 1e3
        t /= reps
        nbytes = 2 * N * K + N * K + 2 * N * (K // 128)
        res[name] = {"us": round(t * 1e6, 2), "GB/s": round(nbytes / t / 1e9, 1),
                     "frac_hbm": round(nbytes / t / 1e9 / hbm_peak, 3)}
        tot_b += nbytes
        tot_t += t
        del w, out
    del flush
    return {"workload": "fp16 weights of the 7 Llama-3-8B-shaped projections -> planes + "
                        "scales, one launch each after an L2 flush",
            "GB/s": round(tot_b / tot_t / 1e9, 1), "frac_hbm": round(tot_b / tot_t / 1e9 / hbm_peak, 3),
            "us_total": round(tot_t * 1e6, 1), "per_projection": res}


# --------------------------------------------------------- decode round
ROUND_LAYERS = 32
ROUND_DRAFT_PASSES = 3  # gamma = 3 draft tokens, then one verify pass at M = gamma + 1


def round_bytes():
    """Algorithmic bytes of one speculative decode round over the 32 layers."""
    per = {}
    for mode, M in DECODE_M.items():
        per[mode] = sum(fused_bytes(mode, M, *group_shape(m)) for _, m in LAYER_GROUPS)
    return ROUND_LAYERS * (ROUND_DRAFT_PASSES * per[0] + per[1])


def measure_round(wl, hbm_peak, reps=10):
    """One speculative decode round on 32 layers of Llama-3-8B-shaped nested
    weights (3.5 GB hi + 3.5 GB lo planes): three draft passes at M = 1, then
    the verify pass at M = 4, every layer's four quantise + linear pairs, as
    one CUDA graph.  The layer weights are drawn on the device by torch's
    seeded generator (uniform plane bytes = uniform nibbles; scales
    1e-4 + 0.005 |N(0,1)| in fp16); they are only timed, never checked."""
    import torch

    bn = wl.bn
    dev = wl.dev
    gen = torch.Generator(device=dev)
    gen.manual_seed(6000)
    layers = []
    for _ in range(ROUND_LAYERS):
        lw = {}
        for gname, members in LAYER_GROUPS:
            N, K, _ = group_shape(members)
            hi = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=gen)
            lo = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=gen)
            z = torch.randn((N, K // 128), device=dev, generator=gen)
            lw[gname] = (hi, lo, (1e-4 + 0.005 * z.abs()).half())
        layers.append(lw)
    path = bn.PATH_AUTO | (bn.PATH_OVERLAP if wl.overlap else 0)

    def one_round():
        for p in range(ROUND_DRAFT_PASSES + 1):
            mode = 1 if p == ROUND_DRAFT_PASSES else 0
            for lw in layers:
                for gname, members in LAYER_GROUPS:
                    _, _, g = group_shape(members)
                    b = wl.bufs[gname, mode]
                    hi, lo, s = lw[gname]
                    bn.quantize_linear(mode, hi, lo, s, wl.x[gname, mode], g, out=b["y"],
                                       act_out=(b["xq"], b["xs"], None), path=path)

    graph = capture(one_round)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    t = timed_replays([graph], reps, lambda: None) / reps
    graph.reset()
    del layers
    torch.cuda.empty_cache()
    nb = round_bytes()
    launches = (ROUND_DRAFT_PASSES + 1) * ROUND_LAYERS * len(LAYER_GROUPS)
    return {
        "workload": "speculative round: 32 layers x 7 projections, 3 draft passes (M=1) + "
                    "1 verify pass (M=4), one quantise + linear kernel per layer group, one CUDA graph",
        "us_per_round": round(t * 1e6, 1),
        "GB_per_round": round(nb / 1e9, 3),
        "GB_per_token_full_acceptance": round(nb / 1e9 / (ROUND_DRAFT_PASSES + 1), 3),
        "GB/s": round(nb / t / 1e9, 1),
        "frac_hbm": round(nb / t / 1e9 / hbm_peak, 3),
        "launches_per_round": launches,
        "rounds_timed": reps,
    }


# ------------------------------------------ speculative decoding rounds
SPEC_DIM, SPEC_LAYERS, SPEC_VOCAB, SPEC_GAMMA = 4096, 4, 8192, 3


def measure_speculative(wl, hbm_peak, replays=40):
    """Speculative rounds (gamma = 3) against the target's own greedy
    decoding on a synthetic nested model (dim 4096, 4 layers, vocabulary
    8192; planes and scales packed by bitnest_pack_weights from seeded
    N(0, 0.02^2) fp16 weights, so the draft is close to the target).  One
    round and one greedy step are each captured as a CUDA graph (the
    sequence and its length stay on the device) and replayed; CUDA events."""
    import torch

    bn = wl.bn
    dev = wl.dev
    d, L, V, gamma = SPEC_DIM, SPEC_LAYERS, SPEC_VOCAB, SPEC_GAMMA
    gen = torch.Generator(device=dev)
    gen.manual_seed(synth.SEED_WEIGHTS + 900)

    def packed(rows):
        w = (0.02 * torch.randn((rows, d), generator=gen, device=dev)).half()
        return bn.pack_weights(w)

    model = bn.SpecModel(torch.randn((V, d), generator=gen, device=dev).half(),
                         [packed(d) for _ in range(L)], packed(V))
    cap = 2 + (replays + 4) * (gamma + 1)

    def state(g):
        seq = torch.zeros((cap,), dtype=torch.int32, device=dev)
        seq[:2] = torch.tensor([1, 2], dtype=torch.int32)
        return (seq, torch.tensor([2], dtype=torch.int32, device=dev),
                torch.zeros(4, dtype=torch.int32, device=dev),
                torch.empty(bn.spec_work_bytes(V, d, g), dtype=torch.uint8, device=dev))

    res = {}
    for name, g, fn in (("speculative", gamma, lambda st: bn.spec_rounds(model, gamma, 1, *st)),
                        ("target_greedy", 0, lambda st: bn.spec_greedy(model, 1, *st))):
        st = state(g)
        graph = capture(lambda: fn(st))  # one round (or step) already ran while warming
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        st[2].zero_()
        torch.cuda.synchronize()
        a.record()
        for _ in range(replays):
            graph.replay()
        b.record()
        torch.cuda.synchronize()
        t = a.elapsed_time(b) / 1e3
        rounds, appended, accepted, overflow = (int(v) for v in st[2].tolist())
        graph.reset()
        res[name] = {"us_per_call": round(t / replays * 1e6, 2),
                     "tokens_per_s": round(appended / t, 1),
                     "tokens_per_call": round(appended / replays, 3)}
        if g:
            res[name]["acceptance"] = round(accepted / max(1, rounds * gamma), 4)
        if overflow:
            res[name]["error"] = "sequence capacity exceeded"
    res["speedup_vs_target_greedy"] = round(res["speculative"]["tokens_per_s"] /
                                            res["target_greedy"]["tokens_per_s"], 3)
    del model
    return {"workload": f"synthetic nested model: dim {d}, {L} layers, vocabulary {V}, "
                        f"gamma {gamma}; one round / one greedy step per CUDA graph replay",
            **res}


# ------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="bitnest", choices=["bitnest", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch the layer kernels without programmatic dependent launch "
                         "(ncu cannot replay such launches inside a captured graph)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step's kernels directly instead of replaying a CUDA graph "
                         "(for profilers that cannot replay the captured kernel nodes)")
    ap.add_argument("--workload", default="all",
                    choices=["all", "decode", "prefill", "sweep", "cost", "round", "pack",
                             "hadamard", "attention", "spec"],
                    help="all: the decode step line with the prefill, M-sweep and "
                         "decode-round objects; otherwise only that part (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.no_overlap:
        os.environ["BITNEST_PDL"] = "0"  # read by the library at its first launch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl_name = "llama3-8b-decode-projections"

    if args.impl == "reference":
        run_reference(args, rank, world, wl_name)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=device)

    barrier, max_over_ranks = dist_helpers(world, device)

    wl = DecodeWorkload(device, overlap=not args.no_overlap)
    step_bytes = wl.step_bytes()
    hbm_peak, bf16_peak, peak_kind = load_peaks()
    dec = None
    if args.workload in ("all", "decode"):
        dec = measure_decode(args, wl, barrier, max_over_ranks, world, hbm_peak, peak_kind)
        step_results = wl.step_results()
    sweep = rnd = cost = None
    if args.workload in ("all", "sweep"):
        sweep = measure_sweep(wl, hbm_peak, reps=5 if args.workload == "all" else 2)
    if args.workload in ("all", "cost"):
        cost = measure_call_cost(wl, hbm_peak, reps=5 if args.workload == "all" else 3)
    if args.workload in ("all", "round"):
        rnd = measure_round(wl, hbm_peak, reps=10 if args.workload == "all" else 3)
    pack = None
    if args.workload in ("all", "pack"):
        pack = measure_pack(wl, hbm_peak)
    had = None
    if args.workload in ("all", "hadamard"):
        had = measure_hadamard(wl, hbm_peak)
    prefill = None
    if args.workload in ("all", "prefill"):
        pre, pre_ops, pre_t = measure_prefill(wl, reps=10 if args.workload == "all" else 3)
        int8_peak = 2.0 * bf16_peak  # dense int8 : dense bf16 = 2 : 1 (nominal 4.5 : 2.25 PFLOP/s)
        pre_tops = pre_ops / pre_t / 1e12
        prefill = {
            "workload": f"target W8A8, M={PREFILL_M}, 7 Llama-3-8B-shaped projections, tcgen05 kind::i8",
            "TOPS": round(pre_tops, 1),
            "us_total": round(pre_t * 1e6, 1),
            "roofline": {"bound": "tensor", "achieved": round(pre_tops, 1),
                         "peak": round(int8_peak, 1), "unit": "TOPS",
                         "frac": round(pre_tops / int8_peak, 4),
                         "peak_kind": f"{peak_kind} bf16 x 2 (dense int8 : bf16 nominal ratio)"},
            "per_projection": pre,
            "l2": "flushed (256 MB write) before every timed launch",
        }
    spec_res = None
    if args.workload in ("all", "spec"):
        try:
            spec_res = measure_speculative(wl, hbm_peak)
        except Exception as e:  # noqa: BLE001
            spec_res = {"error": f"{type(e).__name__}: {e}"}
    att = None
    if args.workload in ("all", "attention"):
        # an auxiliary row, measured last: its failure must not cost the rest
        try:
            att = measure_attention(wl, hbm_peak)
        except Exception as e:  # noqa: BLE001
            att = {"error": f"{type(e).__name__}: {e}"}
    if dec is None:
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            part = {"prefill": prefill, "m_sweep": sweep, "decode_call_cost": cost,
                    "decode_round": rnd,
                    "pack_from_weights": pack, "down_proj_input_rotation": had,
                    "nested_kv_attention": att, "speculative_rounds": spec_res}
            print(json.dumps({"metric": METRIC, "workload": f"{args.workload} only",
                              **{k: v for k, v in part.items() if v is not None}}), flush=True)
        return
    value, ms_per_step, clocks, e2e_value, h2d, d2h, roofline = dec

    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8 x u8/u4 -> int32, fp32 epilogue",
        "data": "synthetic (seeded SplitMix64: uniform nibbles, fp16 scales, N(0,1) activations with 4 x20 outliers)",
        "config": step_config(wl_name, world),
        "timing": ("direct launches" if args.no_graph else "CUDA graph per step")
                  + ", CUDA events on the launching stream, max over ranks",
        "clocks": clocks.summary(),
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "every step: all activations uploaded from pinned host memory in one copy, all outputs read back in one copy; weights resident"},
        "gpu_launches": wl.launches_per_step() * args.steps,
        "roofline": roofline,
    }
    if prefill is not None:
        out["prefill"] = prefill
    if sweep is not None:
        out["m_sweep"] = {"workload": "M in {1..128} x gate_proj 14336x4096 / down_proj "
                                      "4096x14336 x draft / target",
                          "timing": "CUDA graph of back-to-back launches over six rotating "
                                    "weight copies (weights read from HBM), per launch",
                          "per_case": sweep}
    if cost is not None:
        out["decode_call_cost"] = cost
    if rnd is not None:
        out["decode_round"] = rnd
    if pack is not None:
        out["pack_from_weights"] = pack
    if had is not None:
        out["down_proj_input_rotation"] = had
    if att is not None:
        out["nested_kv_attention"] = att
    if spec_res is not None:
        out["speculative_rounds"] = spec_res
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, cores, n_steps, check = cpu_baseline(results=step_results)
        out["cpu_baseline"] = {
            "value": round(step_bytes / t_cpu / 1e9, 4), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{n_steps} whole decode steps on the step's own inputs (every layer "
                      "group, both passes, every output row), median step time",
        }
        out["self_check"] = check
    else:
        out["self_check"] = "not run (no oracle leg on this rank or run)"
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def step_config(wl_name, world):
    """The workload of one step (the same for both arms)."""
    return {
        "workload": wl_name,
        "projections": {k: list(v[:2]) for k, v in synth.LLAMA3_8B_PROJECTIONS.items()},
        "launches": "per pass: one quantise + linear call for q|k|v (fused, N=6144), o (per-group "
                    "activation scales), gate|up (fused, N=28672), down",
        "passes": "draft W4A8 M=1 then verify W8A8 M=4 (gamma+1)",
        "group": 128,
        "bytes_per_step": decode_step_bytes(),
        "l2": f"inputs larger than L2: {N_COPIES} rotating copies of the layer weights "
              f"({N_COPIES * sum(v[0] * v[1] for v in synth.LLAMA3_8B_PROJECTIONS.values()) / 1e6:.0f}"
              " MB of planes)",
        "parallelism": "replicas" if world > 1 else "single",
    }


def dist_helpers(world, device):
    """barrier() and max_over_ranks(v) over the default process group (any
    backend: CUDA tensors for nccl, CPU tensors for gloo); no-ops alone."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def run_reference(args, rank, world, wl_name):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    step_bytes = decode_step_bytes()
    steps = min(args.steps, 60)  # whole oracle steps: about 0.7 s each on 16 threads
    cpu_baseline(budget_s=0.0, max_steps=1)  # warm-up (first-touch of the inputs)
    t, cores, n, _ = cpu_baseline(budget_s=float("inf"), max_steps=steps)
    times = [t] * n
    value = step_bytes / t / 1e9
    out = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": len(times), "warmup": args.warmup, "ms_per_step": round(1e3 * t, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int64 sums, fp64 output", "data": "synthetic",
        "config": step_config(wl_name, world),
        "timing": "host wall clock of the oracle, median over the steps",
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} whole decode steps (every layer group, both passes, "
                                   "every output row), median step time"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
