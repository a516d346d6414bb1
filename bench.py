#!/usr/bin/env python
"""Throughput of the sparse noisy top-k MoE layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral|decode|nano|fine|toy]
                    [--impl ours|reference]

One step = one moe_forward call (router, dispatch, expert FFN, combine) over
one batch of the workload's synthetic tokens, inputs resident in HBM.  Under
torchrun every rank runs its own independent batch (data-parallel replicas,
weak scaling, no collective on the data path); the time is the max over ranks.
Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle instead
(rank 0 only, bounded samples of the same workload).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "MoE layer tokens/sec at 1 B200; % of bf16 tensor peak (prefill) / HBM BW (decode)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="mixtral", choices=["mixtral", "decode", "nano", "fine", "toy"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the secondary decode measurement")
    ap.add_argument("--only", action="store_true", help="measure only --workload (no secondary workloads)")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward measurement")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (small cases for profiling); implies --only")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.tokens is not None:
        a.only = True
    return a


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ ranks
class Dist:
    def __init__(self, backend="nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float, device=None) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.barrier()
            self.pg.destroy_process_group()


def aggregate(tokens_per_rank: int, steps: int, world: int, max_seconds: float) -> dict:
    """Whole-job throughput from the slowest rank's device time."""
    total = tokens_per_rank * steps * world
    return {"value": total / max_seconds, "ms_per_step": 1e3 * max_seconds / steps}


# ------------------------------------------------------------------ clocks
_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
            0x10: "sync_boost", 0x100: "display_clock_setting"}


class ClockSampler:
    """Reads SM clocks and clock-event reasons through NVML every 20 ms (read only)."""

    def __init__(self, torch_device):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            props = torch.cuda.get_device_properties(torch_device)
            bus = getattr(props, "pci_bus_id", None)
            if bus is not None:
                busid = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(busid.encode())
            else:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((sm, r))
            except Exception:
                pass
            self._stop.wait(0.02)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, r in self.samples:
            for bit, name in _REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ algorithmic work
def ffn_flops(R: int, d: int, d_ff: int) -> float:
    """Expert GEMMs: up (R x d x d_ff) and down (R x d_ff x d), 2 flops per MAC."""
    return 4.0 * R * d * d_ff


def ffn_bytes(counts, d: int, d_ff: int, elem: int) -> float:
    """Least HBM traffic of the expert FFN: every touched expert's W_up and
    W_down once, the gathered rows read once, the hidden rows written and read
    once, the expert outputs written once."""
    R = int(sum(counts))
    touched = sum(1 for c in counts if c > 0)
    return elem * (touched * 2.0 * d * d_ff + R * d + 2.0 * R * d_ff + R * d)


def ncu_traffic(kernel_tag: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel source (its hash matches); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    src = os.path.join(ROOT, "sparse_mixture_experts_noisy_b200", "csrc", "gemm_tc.cu")
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        for line in open(path):
            parts = line.split()
            if len(parts) >= 3 and parts[0] == kernel_tag and parts[1] == h:
                return float(parts[2])
    except OSError:
        pass
    return None


# ------------------------------------------------------------------ oracle (CPU) timing
def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_tokens_for(wl, seconds: float, nthreads: int) -> int:
    """Tokens of a sub-batch the oracle finishes in about `seconds`: the router
    runs on one thread (d*E double multiply-adds per token), the expert FFN on
    `nthreads` (k*2*d*d_ff per token), about 1 ns each."""
    per_token = (wl.d * wl.E + wl.k * 2.0 * wl.d * wl.d_ff / max(1, nthreads)) * 1.0e-9
    return max(1, min(wl.N, int(seconds / max(per_token, 1e-12))))


class OracleSteps:
    """The CPU oracle as the layer's reference implementation, on bounded
    samples of the workload.  One step is the oracle's whole layer (router
    logits, noise, KeepTopK, softmax, slot assignment against the sub-batch's
    own capacity, expert FFN, combine) on a contiguous sub-batch of n tokens of
    the workload's batch; successive steps take successive sub-batches.  Every
    second of it is timed; nothing is extrapolated."""

    def __init__(self, inp, wl, n, nthreads):
        self.inp, self.wl, self.n, self.nthreads = inp, wl, n, nthreads
        self.off = 0

    def step(self) -> float:
        import oracle
        inp, wl = self.inp, self.wl
        n = self.n
        if self.off + n > wl.N:
            self.off = 0
        sl = slice(self.off, self.off + n)
        noise = inp.noise[sl] if inp.noise is not None else None
        t0 = time.perf_counter()
        oracle.forward(inp.x[sl], inp.W_g, inp.b_g, noise, wl.sigma, wl.k, wl.cf, inp.W_up, inp.W_down,
                       nthreads=self.nthreads)
        dt = time.perf_counter() - t0
        self.off += n
        return dt

    def describe(self) -> str:
        wl = self.wl
        whole = "the whole batch" if self.n == wl.N else f"contiguous {self.n}-token sub-batches of the {wl.N}-token batch"
        return (f"oracle layer forward (logits, routing, slots with the sub-batch's own capacity, expert FFN, "
                f"combine) on {whole}; FFN and combine on {self.nthreads} threads, the rest on one")


def oracle_timed(inp, wl, seconds: float, nthreads: int, steps: int = 1, warmup: int = 1):
    """Times `steps` oracle steps after `warmup` (the first warm-up step also
    calibrates the sub-batch size to about `seconds` per step).
    Returns (OracleSteps, total timed seconds, tokens timed)."""
    n0 = oracle_tokens_for(wl, seconds, nthreads)
    probe = OracleSteps(inp, wl, max(1, min(n0, max(1, n0 // 8))), nthreads)
    t = probe.step()
    n = max(1, min(wl.N, int(probe.n * seconds / max(t, 1e-6))))
    run = OracleSteps(inp, wl, n, nthreads)
    for _ in range(max(0, warmup - 1)):
        run.step()
    total = sum(run.step() for _ in range(steps))
    return run, total, n * steps


def run_reference(args):
    from sparse_mixture_experts_noisy_b200.synth import WORKLOADS, make_inputs
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    inp = make_inputs(wl, args.seed)
    nthreads = max(1, min(cpu_cores(), 64))
    # each step about 1.5 s of CPU work, so --steps 20 --warmup 5 ends within a minute or so
    run, total, tokens = oracle_timed(inp, wl, 1.5, nthreads, steps=args.steps, warmup=args.warmup)
    value = tokens / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                             "sample": run.describe(), "tokens_per_step": run.n},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            # not a measurement: the time a whole batch would take at the measured rate
            "extrapolated_whole_batch_ms": 1e3 * total / tokens * wl.N}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, extra=None):
    weights = 2 * wl.E * wl.d * wl.d_ff * (2 if wl.dtype == "bf16" else 4)
    c = {"workload": wl.name, "N": wl.N, "d": wl.d, "E": wl.E, "d_ff": wl.d_ff, "k": wl.k,
         "capacity_factor": wl.cf if math.isfinite(wl.cf) else "inf", "sigma": wl.sigma,
         "router_bias_e0": wl.bias0, "storage": wl.dtype,
         "l2": ("inputs larger than L2 (expert weights %.2f GB)" % (weights / 1e9)) if weights > L2_BYTES
         else "L2 flushed between timed steps (256 MiB write)"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------ GPU arm
def to_dev(a, torch):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def time_steps(fn, steps, torch, flush=None):
    """Per-step CUDA events on the current stream; returns total seconds."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush()
        starts[i].record()
        fn()
        ends[i].record()
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / 1e3


def measure_layer(wl, inp_dev, steps, warmup, dist, torch, moe, flush_needed):
    """moe_forward replayed from a CUDA graph (one graph launch per step)."""
    x, W_g, b_g, noise, W_up, W_down = inp_dev
    layer = moe.MoELayer(W_g, W_up, W_down, wl.k, wl.cf, b_g=b_g, sigma=wl.sigma, max_tokens=wl.N)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=x.device) if flush_needed else None
    flush = (lambda: flush_buf.fill_(1)) if flush_needed else None
    graphed = moe.GraphedForward(layer, x, noise)
    y = graphed.y
    run = graphed.replay
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(x.device)
    with clk:
        sec = time_steps(run, steps, torch, flush)
    torch.cuda.synchronize()
    dist.barrier()
    code, word = moe.check_status(layer.workspace)
    if code != 0:
        raise RuntimeError(f"kernel status {code} (0x{word:08x}) after the timed region")
    return graphed, y, sec, clk.summary()


def measure_ffn(wl, inp_dev, steps, torch, moe, flush=None):
    """The dominant kernels alone: the expert FFN (tcgen05 grouped GEMMs) on the
    batch's gathered rows, back to back on the current stream (the L2 flushed
    between calls when `flush` is given)."""
    x, W_g, b_g, noise, W_up, W_down = inp_dev
    topk, gates, _ = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma, want_logits=False)
    dsp = moe.moe_dispatch(topk, x, wl.E, wl.cf)
    xg, offs, cnt = dsp["x_gathered"], dsp["offsets"], dsp["counts"]
    rows, d = xg.shape
    dt = moe.MOE_BF16 if xg.dtype == torch.bfloat16 else moe.MOE_F32
    ws = moe.new_workspace(moe.load_library().moe_expert_ffn_workspace_size(rows, d, wl.E, wl.d_ff, dt),
                           x.device)
    out = torch.empty_like(xg)
    run = lambda: moe.moe_expert_ffn(xg, offs, cnt, W_up, W_down, ws=ws, out=out)  # noqa: E731
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    sec = time_steps(run, steps, torch, flush)
    code, word = moe.check_status(ws)
    if code != 0:
        raise RuntimeError(f"kernel status {code} (0x{word:08x}) after the expert FFN timing")
    counts = cnt.cpu().numpy().tolist()
    return sec / steps, counts


def measure_e2e(graphed, wl, inp, steps, torch, moe):
    """Through the public API with host buffers (moe.HostPipeline): every step
    copies that step's pinned x (and eps) in, runs the layer and copies y back
    to pinned host memory; the copies of neighbouring steps overlap the
    forward.  Time = all steps from the first copy in to the last copy out."""
    bf = inp.x.dtype == np.uint16
    x_h = torch.from_numpy(inp.x.view(np.int16) if bf else inp.x).pin_memory()
    x_h = x_h.view(torch.bfloat16) if bf else x_h
    n_h = torch.from_numpy(inp.noise).pin_memory() if inp.noise is not None else None
    y_h = [torch.empty(x_h.shape, dtype=x_h.dtype).pin_memory() for _ in range(2)]
    x_d = x_h.to("cuda")
    n_d = n_h.to("cuda") if n_h is not None else None
    pipe = moe.HostPipeline(graphed.layer, x_d, n_d)
    del x_d, n_d
    for i in range(3):
        pipe.submit(x_h, y_h[i & 1], n_h)
    pipe.synchronize()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(steps):
        pipe.submit(x_h, y_h[i & 1], n_h)
    pipe.synchronize()
    sec = time.perf_counter() - t0
    h2d = x_h.numel() * x_h.element_size() + (n_h.numel() * n_h.element_size() if n_h is not None else 0)
    d2h = y_h[0].numel() * y_h[0].element_size()
    return sec / steps, h2d, d2h


def roofline_entry(kind, achieved, peak, unit, traffic, kernel, peak_src, extra=None):
    e = {"bound": kind, "achieved": achieved, "peak": peak, "unit": unit,
         "frac": (achieved / peak) if peak else None,
         "traffic": traffic, "kernel": kernel, "peak_source": peak_src}
    if extra:
        e.update(extra)
    return e


def ffn_kernel_name(wl, moe):
    tc = wl.dtype == "bf16" and wl.d % 8 == 0 and wl.d_ff % 8 == 0
    if not tc:
        return "simt_gemm_kernel (fp32 CUDA cores, up + down)"
    if moe.gathered_rows(wl.N, wl.E, wl.k, wl.cf) <= 256:
        return "tc_gemm_kernel, weight-row tiles (up + down) + reduce_parts_kernel"
    if os.environ.get("MOE_TC_PAIR", "1") != "0":
        return "tc2_gemm_kernel, CTA pairs (up + down launches of one moe_expert_ffn call)"
    return "tc_gemm_kernel (up + down launches of one moe_expert_ffn call)"


def measure_workload(wl, inp_dev, steps, warmup, dist, dev, torch, moe, peaks, peak_src, ffn_steps):
    """Device time of the graphed layer over `steps` steps (max over ranks),
    the expert FFN alone for the roofline, and the clocks seen meanwhile."""
    weights_bytes = 2 * wl.E * wl.d * wl.d_ff * (2 if wl.dtype == "bf16" else 4)
    flush_needed = weights_bytes <= L2_BYTES
    graphed, _, sec, clocks = measure_layer(wl, inp_dev, steps, warmup, dist, torch, moe, flush_needed)
    max_sec = dist.max(sec, device=dev)
    agg = aggregate(wl.N, steps, dist.world, max_sec)
    step_s = max_sec / steps
    elem = 2 if wl.dtype == "bf16" else 4
    kernel = ffn_kernel_name(wl, moe)
    flush = None
    if flush_needed:
        buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        flush = lambda: buf.fill_(1)  # noqa: E731
    ffn_sec, counts = measure_ffn(wl, inp_dev, ffn_steps, torch, moe, flush)
    R = int(sum(counts))
    decode_plan = "weight-row" in kernel
    if wl.dtype != "bf16":
        # fp32 storage: CUDA-core FFMA; a handful of tokens is launch-latency bound
        fl = ffn_flops(R, wl.d, wl.d_ff)
        roof = roofline_entry("latency", step_s * 1e6, None, "us", None, kernel, None,
                              {"ffn_us_per_call": ffn_sec * 1e6, "algorithmic_flops": fl, "kept_rows": R,
                               "note": "fp32 toy layer: the step is a few kernel launches, no roofline applies"})
    elif decode_plan:
        byt = ffn_bytes(counts, wl.d, wl.d_ff, elem)
        layer_bytes = byt + wl.N * wl.d * elem * 2 + wl.E * wl.d * 4
        roof = roofline_entry("hbm", byt / ffn_sec / 1e9, peaks["hbm_gbs"], "GB/s", ncu_traffic("decode"),
                              kernel, peak_src + " (copy)",
                              {"algorithmic_bytes": byt, "ms_per_call": ffn_sec * 1e3,
                               "whole_layer_gbs": layer_bytes / step_s / 1e9,
                               "whole_layer_frac": layer_bytes / step_s / 1e9 / peaks["hbm_gbs"],
                               "whole_layer_frac_of_8tbs": layer_bytes / step_s / 8e12})
    else:
        fl = ffn_flops(R, wl.d, wl.d_ff)
        roof = roofline_entry("tensor", fl / ffn_sec / 1e12, peaks["bf16_tflops"], "TFLOP/s",
                              ncu_traffic("prefill_" + wl.name), kernel, peak_src + " burst",
                              {"frac_of_sustained": fl / ffn_sec / 1e12 / peaks["bf16_tflops_sustained"],
                               "algorithmic_flops": fl, "kept_rows": R, "ms_per_call": ffn_sec * 1e3,
                               "whole_layer_frac": fl / step_s / 1e12 / peaks["bf16_tflops"]})
    router = None
    if wl.dtype == "bf16":
        # the router alone (moe_forward's pre-split path), against the copy bandwidth
        # replayed from a CUDA graph, so the time is the GPU's, not the host's launch path
        rws = moe.route_workspace(wl.d, wl.E, dev)
        x, W_g, b_g, noise = inp_dev[:4]
        rcall = lambda: moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma,  # noqa: E731
                                      want_logits=False, status=rws)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            rcall()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        # tokens larger than L2: 20 calls back to back in one graph (one call
        # is shorter than the host's launch path); else one call per replay
        # with the L2 flushed between replays
        per_graph = 20 if wl.N * wl.d * elem > L2_BYTES else 1
        rgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(rgraph):
            for _ in range(per_graph):
                rcall()
        for _ in range(3):
            rgraph.replay()
        torch.cuda.synchronize()
        rsteps = max(10, min(steps, 100))
        rsec = time_steps(rgraph.replay, rsteps, torch, None if per_graph > 1 else flush) / (rsteps * per_graph)
        rbytes = wl.N * wl.d * elem + (wl.N * wl.E * 4 if noise is not None else 0) + wl.N * wl.k * 8
        router = {"us_per_call": rsec * 1e6, "calls_per_graph": per_graph, "algorithmic_bytes": rbytes,
                  "gbs": rbytes / rsec / 1e9,
                  "frac": rbytes / rsec / 1e9 / peaks["hbm_gbs"], "peak_source": peak_src + " (copy)"}
    out = {"workload": wl.name, "value": agg["value"], "unit": UNIT, "ms_per_step": agg["ms_per_step"],
           "steps": steps, "config": workload_config(wl), "roofline": roof, "clocks": clocks, "router": router,
           "gpu_launches": moe.forward_launches(wl.N, wl.d, wl.E, wl.d_ff, wl.k, wl.cf, inp_dev[0].dtype) * steps}
    if decode_plan and not moe.set_fused_small_batch(None):
        # the same layer as one cooperative launch (opt-in), for comparison
        moe.set_fused_small_batch(True)
        try:
            if moe.forward_launches(wl.N, wl.d, wl.E, wl.d_ff, wl.k, wl.cf, inp_dev[0].dtype) == 1:
                fsteps = max(20, min(steps, 300))
                fg, _, fsec, fclk = measure_layer(wl, inp_dev, fsteps, warmup, dist, torch, moe, flush_needed)
                fsec = dist.max(fsec, device=dev)
                del fg
                out["single_launch"] = {"what": "decode_fused_kernel (moe_set_fused_small_batch(1))",
                                        "ms_per_step": 1e3 * fsec / fsteps,
                                        "value": wl.N * dist.world * fsteps / fsec, "unit": UNIT,
                                        "steps": fsteps, "clocks": fclk}
        finally:
            moe.set_fused_small_batch(False)
    return out, graphed


def measure_backward(wl, inp_dev, steps, dist, dev, torch, moe, peaks, peak_src, seed):
    """The backward of the layer (moe_backward) for the routing of one staged
    forward, on the forward's kept activations: its four expert GEMMs are
    2 R d d_ff flops each.  Timed with CUDA events over back-to-back calls."""
    from sparse_mixture_experts_noisy_b200.synth import f32_to_bf16_bits, normal_f32
    x, W_g, b_g, noise, W_up, W_down = inp_dev
    topk, gates, _ = moe.moe_route(x, W_g, wl.k, b_g=b_g, noise=noise, sigma=wl.sigma, want_logits=False)
    dsp = moe.moe_dispatch(topk, x, wl.E, wl.cf)
    out, H = moe.moe_expert_ffn_train(dsp["x_gathered"], dsp["offsets"], dsp["counts"], W_up, W_down)
    dyh = normal_f32(seed + 5, (wl.N, wl.d), 1.0)
    dy = to_dev(f32_to_bf16_bits(dyh) if wl.dtype == "bf16" else dyh, torch)
    args = (x, W_g, W_up, W_down, wl.k, topk, gates, dsp["slot"], dsp["offsets"], dsp["counts"], dsp["x_gathered"], H,
            out, dy)
    g = moe.moe_backward(*args)
    ws = g["ws"]
    run = lambda: moe.moe_backward(*args, ws=ws)  # noqa: E731
    for _ in range(2):
        run()
    torch.cuda.synchronize()
    dist.barrier()
    clk = ClockSampler(dev)
    with clk:
        sec = time_steps(run, steps, torch)
    code, word = moe.check_status(ws)
    if code != 0:
        raise RuntimeError(f"kernel status {code} (0x{word:08x}) after the backward timing")
    sec = dist.max(sec, device=dev)
    R = int(dsp["counts"].sum().item())
    fl = 2.0 * ffn_flops(R, wl.d, wl.d_ff)
    return {"workload": wl.name, "what": "moe_backward: dx, dW_g, db_g, dW_up, dW_down for one routed batch",
            "value": wl.N * dist.world * steps / sec, "unit": UNIT, "ms_per_step": 1e3 * sec / steps, "steps": steps,
            "roofline": roofline_entry("tensor", fl / (sec / steps) / 1e12, peaks["bf16_tflops"], "TFLOP/s", None,
                                       "whole backward (four expert GEMMs on the tensor cores + per-token kernels)",
                                       peak_src + " burst", {"algorithmic_flops": fl, "kept_rows": R}),
            "clocks": clk.summary()}


# timed steps of the secondary workloads, whatever --steps is: enough that the
# timed region lasts about half a second and the clock sampler sees 20 samples
SECONDARY_STEPS = {"decode": 1500, "nano": 2500, "fine": 200, "toy": 5000}


def run_ours(args):
    import torch
    from sparse_mixture_experts_noisy_b200 import moe
    from sparse_mixture_experts_noisy_b200.synth import WORKLOADS, make_inputs, make_noise, make_x

    dist = Dist("nccl")
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    moe.load_library()
    peaks, peak_src = load_peaks()

    def inputs(name, weights=True):
        wl = WORKLOADS[name]
        if args.tokens is not None and name == args.workload:
            wl = wl.with_(N=args.tokens)
        # replicas of one model: the same weights on every rank, each rank its own tokens
        inp = make_inputs(wl, args.seed, weights=weights)
        if dist.rank > 0:
            inp.x = make_x(wl, args.seed + 7919 * dist.rank)
            inp.noise = make_noise(wl, args.seed + 7919 * dist.rank)
        return wl, inp

    wl, inp = inputs(args.workload)
    inp_dev = tuple(to_dev(a, torch) for a in (inp.x, inp.W_g, inp.b_g, inp.noise, inp.W_up, inp.W_down))
    main, graphed = measure_workload(wl, inp_dev, args.steps, args.warmup, dist, dev, torch, moe, peaks, peak_src,
                                     max(10, min(args.steps, 200)))

    # end to end through the public API with host buffers
    e2e_steps = max(5, min(args.steps, 50))
    e2e_sec, h2d, d2h = measure_e2e(graphed, wl, inp, e2e_steps, torch, moe)
    e2e_sec = dist.max(e2e_sec, device=dev)

    line = {"metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": workload_config(wl, {"parallelism": f"replicas x{dist.world}" if dist.world > 1 else "1 GPU",
                                           "seed": args.seed}),
            "roofline": main["roofline"],
            "e2e": {"value": wl.N * dist.world / e2e_sec, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": main["gpu_launches"],
            "clocks": main["clocks"],
            "router": main["router"]}
    if main.get("single_launch"):
        line["single_launch"] = main["single_launch"]
    del graphed

    if wl.dtype == "bf16" and not args.no_backward:
        line["backward"] = measure_backward(wl, inp_dev, max(10, min(args.steps, 50)), dist, dev, torch, moe, peaks,
                                            peak_src, args.seed)
        torch.cuda.empty_cache()

    # every other workload, each with its own timed region, roofline and clocks
    if args.workload == "mixtral" and not args.only:
        for name in ("decode", "nano", "fine", "toy"):
            if name == "decode" and args.no_decode:
                continue
            if name == "decode":
                # same weight shapes and seeds as the Mixtral-shaped layer: reuse them
                swl, sinp = inputs("decode", weights=False)
                sdev = (to_dev(sinp.x, torch), inp_dev[1], None, None, inp_dev[4], inp_dev[5])
            else:
                swl, sinp = inputs(name)
                sdev = tuple(to_dev(a, torch) for a in (sinp.x, sinp.W_g, sinp.b_g, sinp.noise, sinp.W_up,
                                                        sinp.W_down))
            steps = SECONDARY_STEPS[name]
            obj, g = measure_workload(swl, sdev, steps, args.warmup, dist, dev, torch, moe, peaks, peak_src,
                                      max(20, min(steps, 200)))
            del g, sdev
            obj.pop("config")
            line[name] = obj
            torch.cuda.empty_cache()

    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        nthreads = max(1, min(cpu_cores(), 64))
        run, total, tokens = oracle_timed(inp, wl, args.cpu_seconds, nthreads, steps=1, warmup=1)
        line["cpu_baseline"] = {"value": tokens / total, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                                "sample": run.describe() + f" ({run.n} tokens, {total:.1f} s timed)"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
