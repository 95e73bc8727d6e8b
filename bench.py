"""Benchmark of the W8A8 int8-dynamic linear path on B200.

One step = one pass of the hot path over one batch: dynamic per-token int8
quantisation of the activations, the int8 x int8 -> int32 tensor-core GEMM
against pre-packed int8 weights, and the dequantising bf16 epilogue
(w8a8_linear), on the square 512 x 4096 x 4096 projection with bias and an
all-zero row.  Weights are packed once before timing (load time).

Prints ONE JSON line (rank 0).  ``value`` is whole-job int8 TOPS (2*M*N*K per
step, summed over ranks, divided by the max-over-ranks device time).  Inputs
rotate over enough buffer sets to exceed the 126 MB L2, and each set's step is
replayed from a CUDA graph so host launch overhead stays out of the device
timing.  Also reported: the dominant kernel's roofline (GEMM alone, CUDA
events on its stream), an end-to-end figure through the public API with
host buffers, the oracle's CPU throughput, SM clocks sampled during the timed
region, and a sweep over the other workloads.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--no-sweep] [--workload NAME]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

from w8a8_int8_dynamic_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

MAIN_WORKLOAD = "square_512x4096x4096"
# where the raw nvidia-smi clock samples go (--clocks-dir); the JSON line
# carries their summary either way
CLOCKS_DIR = os.path.join(tempfile.gettempdir(), "w8a8_bench_clocks")
L2_BYTES = 126 * 1024 * 1024
SPEC_INT8_TOPS = 4500.0


# ----------------------------------------------------------------------------- peaks
def load_peaks():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# the sources the dominant kernel is compiled from (a change voids the record)
TRAFFIC_SOURCES = ("gemm.cu", "gemm_common.cuh", "act.cuh", "ptx.cuh")


def recorded_traffic(workload):
    """DRAM bytes per launch of the GEMM from the committed ncu capture, or
    None when there is none or the kernel sources changed since it was taken."""
    import hashlib
    path = os.path.join(HERE, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(workload)
    if not rec:
        return None
    csrc = os.path.join(HERE, "w8a8_int8_dynamic_b200", "csrc")
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    if h.hexdigest()[:16] != rec.get("source_sha256_16"):
        return None
    return rec.get("gemm_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, tag: str = ""):
        self.index = index
        self.tag = tag
        self.proc = None
        self.path = None

    def start(self):
        os.makedirs(CLOCKS_DIR, exist_ok=True)
        self.path = os.path.join(CLOCKS_DIR, f"clocks_rank{self.index}{self.tag}.csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [t.strip() for t in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[2], parts[3:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names[1:], r[3][1:]):
                if v.lower() == "active":
                    reasons.add(n)
        loaded = [r[0] for r in rows if r[0] > 500] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ----------------------------------------------------------------------------- helpers
def smi_index(device):
    return torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" in os.environ else device.index or 0


def bf16_dev(a_u16: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).to(device).view(torch.bfloat16)


def algorithmic(wl, M=None):
    M = wl.M if M is None else M
    N, K = wl.N, wl.K
    bias = 2 * N if wl.bias else 0
    ops = 2 * M * N * K
    gemm_bytes = M * K + N * K + 2 * M * N + 4 * M + 4 * N + bias
    quant_bytes = 3 * M * K + 4 * M
    fused_bytes = 2 * M * K + N * K + 2 * M * N + 4 * N + bias
    return ops, gemm_bytes, quant_bytes, fused_bytes


class LayerSets:
    """``nsets`` independent copies of a workload's tensors on the device."""

    def __init__(self, w8, wl, nsets, device, M=None):
        inp = make_inputs(wl, M)
        self.M, self.N, self.K = inp.x.shape[0], wl.N, wl.K
        self.sets = []
        x0 = bf16_dev(inp.x, device)
        w0 = torch.from_numpy(inp.w).to(device)
        packed0 = w8.pack_weight(w0)
        del w0
        ws0 = torch.from_numpy(inp.w_scale).to(device)
        b0 = None if inp.bias is None else bf16_dev(inp.bias, device)
        wsb = w8.linear_workspace_bytes(self.M, self.N, self.K)
        mmws = w8.scaled_mm_workspace_bytes(self.M, self.N, self.K)
        for i in range(nsets):
            s = {
                "x": x0 if i == 0 else x0.clone(),
                "packed": packed0 if i == 0 else packed0.clone(),
                "w_scale": ws0 if i == 0 else ws0.clone(),
                "bias": None if b0 is None else (b0 if i == 0 else b0.clone()),
                "y": torch.empty((self.M, self.N), dtype=torch.bfloat16, device=device),
                "ws": torch.empty((wsb,), dtype=torch.uint8, device=device),
                "mmws": torch.empty((max(mmws, 16),), dtype=torch.uint8, device=device)
                if mmws else None,
            }
            s["q"], s["a_scale"] = w8.quant_act(s["x"])
            self.sets.append(s)
        torch.cuda.synchronize()

    def set_bytes(self):
        s = self.sets[0]
        return sum(t.numel() * t.element_size() for k, t in s.items()
                   if isinstance(t, torch.Tensor))


def sets_needed(w8, wl, M=None):
    """Input sets to rotate over so that every timed loop -- the layer, the
    GEMM alone, the quantisation alone -- touches more than L2 (x 1.5)
    between two uses of the same set.  A quantisation too small to exceed L2
    even over 16 sets (it is latency-bound then) does not count."""
    probe_M = wl.M if M is None else M
    M, N, K = probe_M, wl.N, wl.K
    per = (M * K * 3 + N * K + 2 * M * N + 8 * N + w8.linear_workspace_bytes(M, N, K))
    footprints = [per, M * K + N * K + 2 * M * N]  # the layer; the GEMM alone (q, W, y)
    if 16 * 3 * M * K > 1.5 * L2_BYTES:
        footprints.append(3 * M * K)  # the quantisation alone (x, q)
    smallest = min(footprints)
    n = 1
    while n * smallest <= 1.5 * L2_BYTES and n < 16:
        n += 1
    return n, per


def capture(fns, stream):
    """One CUDA graph that runs the callables in order (consecutive steps)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for fn in fns:
            fn()
    return g


class GraphLoop:
    """Runs `fns` (one per rotated input set) cyclically, `per_graph` calls per
    graph replay, so that the device sees back-to-back kernels and host
    launch overhead stays out of the timing.  A step count that is not a
    multiple of `per_graph` ends with one graph of the remaining steps,
    captured beforehand by `prepare` (otherwise one replay per step)."""

    def __init__(self, fns, stream, per_graph=64):
        self.fns = list(fns)
        self.n = len(fns)
        self.per_graph = max(self.n, per_graph - per_graph % self.n)
        self.stream = stream
        self.graph = capture([fns[i % self.n] for i in range(self.per_graph)], stream)
        self.single = [capture([fn], stream) for fn in fns]
        self.tail = {}  # steps % per_graph -> graph of that many steps from set 0

    def prepare(self, steps):
        """Capture the tail graph that `run(steps)` will need, and replay it
        once: a graph's first replay uploads it (about 2 us a kernel node),
        which must not land in a timed region.  Call outside any timed
        region."""
        rest = steps % self.per_graph
        if rest and rest not in self.tail:
            g = capture([self.fns[i % self.n] for i in range(rest)], self.stream)
            with torch.cuda.stream(self.stream):
                g.replay()
            self.tail[rest] = g

    def run(self, steps):
        full, rest = divmod(steps, self.per_graph)
        for _ in range(full):
            self.graph.replay()
        if rest in self.tail:
            self.tail[rest].replay()
        else:
            for i in range(rest):
                self.single[i % self.n].replay()


def time_loop(loop, steps, stream):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        loop.run(steps)
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3  # seconds


# ----------------------------------------------------------------------------- our arm
def run_workload(w8, wl, steps, warmup, device, stream, M=None, with_quant=True,
                 gemm_clock_tag=None):
    nsets, _ = sets_needed(w8, wl, M)
    ls = LayerSets(w8, wl, nsets, device, M)
    steps_fns, mm_fns, q_fns = [], [], []
    for s in ls.sets:
        def step(s=s):
            w8.linear(s["x"], s["packed"], s["w_scale"], s["bias"], ls.N, out=s["y"],
                      workspace=s["ws"], stream=stream)
        def mm(s=s):
            w8.scaled_mm(s["q"], s["a_scale"], s["packed"], s["w_scale"], s["bias"], ls.N,
                         out=s["y"], workspace=s["mmws"], stream=stream)
        def qa(s=s):
            w8.quant_act(s["x"], q=s["q"], a_scale=s["a_scale"], stream=stream)
        steps_fns.append(step)
        mm_fns.append(mm)
        q_fns.append(qa)
    with torch.cuda.stream(stream):
        for f in steps_fns[:1] + mm_fns[:1] + q_fns[:1]:
            f()  # warm the launch path (attributes, tensor maps) before capture
    torch.cuda.synchronize()
    c0 = w8.launch_count()
    capture([steps_fns[0]], stream)
    per_step = w8.launch_count() - c0
    layer_loop = GraphLoop(steps_fns, stream)
    mm_loop = GraphLoop(mm_fns, stream)
    q_loop = GraphLoop(q_fns, stream)
    for loop in (layer_loop, mm_loop, q_loop):
        loop.prepare(steps)
    torch.cuda.synchronize()
    assert w8.poll_status() == 0
    for loop in (layer_loop, mm_loop, q_loop):
        time_loop(loop, max(warmup, 3) * loop.per_graph, stream)
    res = {"launches_per_step": per_step, "nsets": nsets, "set_bytes": ls.set_bytes(),
           "M": ls.M, "N": ls.N, "K": ls.K}
    res["t_step"] = time_loop(layer_loop, steps, stream) / steps
    res["t_gemm"] = time_loop(mm_loop, steps, stream) / steps
    if gemm_clock_tag is not None:
        # the GEMM alone again, long enough (>= 0.6 s) for the clock sampler:
        # a tensor-bound loop may run under the power cap
        per = mm_loop.per_graph
        n = max(steps, int(0.6 / res["t_gemm"]) // per * per)
        cs = ClockSampler(smi_index(device), tag=gemm_clock_tag)
        cs.start()
        res["t_gemm_long"] = time_loop(mm_loop, n, stream) / n
        res["gemm_clock"] = cs.stop()
    if with_quant:
        res["t_quant"] = time_loop(q_loop, steps, stream) / steps
    assert w8.poll_status() == 0, "device-side timeout during the benchmark"
    return ls, layer_loop, res


def run_ours(args, rank, world, device):
    import w8a8_int8_dynamic_b200 as w8
    w8.lib()
    peaks = load_peaks()
    int8_peak = 2.0 * peaks["bf16_tflops"]  # nominal int8 : bf16 dense rate = 2
    stream = torch.cuda.Stream(device=device)
    wl = WORKLOADS[args.workload]
    ops, gemm_bytes, quant_bytes, fused_bytes = algorithmic(wl)

    ls, layer_loop, base = run_workload(w8, wl, 2000, args.warmup, device, stream)
    layer_loop.prepare(args.steps)
    torch.cuda.synchronize()
    # ---- the timed region: exactly K steps, barrier + sync on both sides
    sampler = ClockSampler(smi_index(device))
    sampler.start()
    time_loop(layer_loop, args.warmup, stream)  # W untimed warm-up steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        layer_loop.run(args.steps)
        end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    elapsed = start.elapsed_time(end) / 1e3
    clocks = sampler.stop()
    assert w8.poll_status() == 0, "device-side timeout during the timed region"
    t_max = elapsed
    if world > 1:
        t = torch.tensor([elapsed], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        t_max = float(t.item())
    value = ops * args.steps * world / t_max / 1e12
    ms_per_step = t_max / args.steps * 1e3

    # ---- dominant kernel (the GEMM) alone, CUDA events on its stream
    gemm_tops = ops / base["t_gemm"] / 1e12
    roofline = {"bound": "tensor", "achieved": round(gemm_tops, 2), "peak": round(int8_peak, 1),
                "unit": "TOPS", "frac": round(gemm_tops / int8_peak, 4), "traffic": None,
                "kernel": w8.gemm_kernel_name(wl.M, wl.N, wl.K),
                "peak_note": f"int8 = 2 x {peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s",
                "frac_vs_spec_4500": round(gemm_tops / SPEC_INT8_TOPS, 4),
                "gemm_us": round(base["t_gemm"] * 1e6, 3),
                "quant_us": round(base["t_quant"] * 1e6, 3),
                "quant_gbs": round(quant_bytes / base["t_quant"] / 1e9, 1),
                "quant_frac_hbm": round(quant_bytes / base["t_quant"] / 1e9 / peaks["hbm_gbs"], 4)}
    roofline["traffic"] = recorded_traffic(args.workload)

    # ---- end to end through the public API, host buffers
    e2e = run_e2e(w8, ls, args, stream, ops)

    out = {
        "metric": "W8A8 quant+scaled-GEMM TOPS and % of int8 roofline on one B200",
        "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8 x int8 -> int32, bf16 in/out",
        "data": "synthetic (seeded; N(0,1) activations with 1% outlier channels x10, "
                "int8 weights uniform [-127,127], fp32 scales, bf16 bias)",
        "config": {"workload": args.workload, "M": wl.M, "N": wl.N, "K": wl.K,
                   "step": "w8a8_linear = quant kernel + tcgen05 GEMM/epilogue (2 launches, PDL)",
                   "l2": f"rotating {base['nsets']} input sets of {base['set_bytes'] / 2**20:.1f} MiB "
                         f"(> 126 MB L2)",
                   "launch": "CUDA graphs of 64 consecutive steps over the rotated sets",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "fused_frac_of_roofline": round(max(ops / (int8_peak * 1e12),
                                            fused_bytes / (peaks["hbm_gbs"] * 1e9)) / (t_max / args.steps),
                                        4),
        "e2e": e2e,
        "gpu_launches": int(base["launches_per_step"] * args.steps),
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_seconds)
    if not args.no_sweep:
        out["sweep"] = sweep(w8, args, device, stream, peaks, int8_peak)
        out["mlp_chain"] = mlp_chain(w8, device, stream)
    return out


def run_e2e(w8, ls, args, stream, ops):
    """Public API, host buffers: per step H2D of x from pinned memory, the
    layer call, D2H of y into pinned memory, all inside the timed region.
    Steps are pipelined the way a serving loop would run them: the upload of
    step i+1, the layer of step i and the download of step i-1 overlap on
    three streams (PCIe is full duplex), with three device buffer sets."""
    s0 = ls.sets[0]
    M, N, K = ls.M, ls.N, ls.K
    dev = s0["x"].device
    nhost, ndev = 4, 3
    xs = [s0["x"].cpu().pin_memory() for _ in range(nhost)]
    ys = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(nhost)]
    xd = [torch.empty_like(s0["x"]) for _ in range(ndev)]
    yd = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(ndev)]
    layer_args = (s0["packed"], s0["w_scale"], s0["bias"], N)
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    comp = stream
    ev_in = [torch.cuda.Event() for _ in range(ndev)]
    ev_done = [torch.cuda.Event() for _ in range(ndev)]
    ev_out = [torch.cuda.Event() for _ in range(ndev)]

    def step(i, first):
        b = i % ndev
        if not first[b]:
            up.wait_event(ev_done[b])        # x[b] free: the layer that read it is done
        with torch.cuda.stream(up):
            xd[b].copy_(xs[i % nhost], non_blocking=True)
            ev_in[b].record(up)
        comp.wait_event(ev_in[b])
        if not first[b]:
            comp.wait_event(ev_out[b])       # y[b] free: its download is done
        w8.linear(xd[b], *layer_args, out=yd[b], workspace=s0["ws"], stream=comp)
        ev_done[b].record(comp)
        down.wait_event(ev_done[b])
        with torch.cuda.stream(down):
            ys[i % nhost].copy_(yd[b], non_blocking=True)
            ev_out[b].record(down)
        first[b] = False

    steps = max(10, min(args.steps, 2000))
    first = [True] * ndev
    for i in range(3):
        step(i, first)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(up)
    comp.wait_event(start)
    down.wait_event(start)
    for i in range(steps):
        step(i, first)
    comp.wait_stream(down)
    comp.wait_stream(up)
    end.record(comp)
    end.synchronize()
    t = start.elapsed_time(end) / 1e3 / steps
    # the last step's output must have arrived
    assert torch.equal(ys[(steps - 1) % nhost].to(dev), yd[(steps - 1) % ndev])
    return {"value": round(ops / t / 1e12, 3), "unit": "TOPS", "h2d_bytes_per_step": M * K * 2,
            "d2h_bytes_per_step": M * N * 2, "steps": steps, "ms_per_step": round(t * 1e3, 4),
            "pipelining": "H2D of step i+1, layer of step i and D2H of step i-1 on three streams",
            "api": "w8a8_int8_dynamic_b200.linear (ctypes -> w8a8_linear)"}


def sweep(w8, args, device, stream, peaks, int8_peak):
    out = {}
    names = ["small_64x128x256", "square_512x4096x4096", "fused_qkv_512x12288x4096",
             "dit_mlp_up_4096x12288x3072", "dit_mlp_down_4096x3072x12288",
             "decode_m1_27648x5120", "decode_m4_27648x5120", "decode_m16_27648x5120"]
    for name in names:
        wl = WORKLOADS[name]
        ops, gemm_bytes, quant_bytes, fused_bytes = algorithmic(wl)
        steps = 256 if wl.M * wl.N * wl.K > 1e11 else 2048
        bound = "tensor" if ops / (int8_peak * 1e12) >= gemm_bytes / (peaks["hbm_gbs"] * 1e9) else "hbm"
        ls, loop, r = run_workload(w8, wl, steps, 3, device, stream,
                                   gemm_clock_tag=("_gemm_" + name) if bound == "tensor" else None)
        t_roof_gemm = max(ops / (int8_peak * 1e12), gemm_bytes / (peaks["hbm_gbs"] * 1e9))
        t_roof_fused = max(ops / (int8_peak * 1e12), fused_bytes / (peaks["hbm_gbs"] * 1e9))
        out[name] = {
            "M": wl.M, "N": wl.N, "K": wl.K, "bound": bound,
            "step_us": round(r["t_step"] * 1e6, 3), "gemm_us": round(r["t_gemm"] * 1e6, 3),
            "quant_us": round(r["t_quant"] * 1e6, 3),
            "step_tops": round(ops / r["t_step"] / 1e12, 2),
            "gemm_tops": round(ops / r["t_gemm"] / 1e12, 2),
            "gemm_gbs": round(gemm_bytes / r["t_gemm"] / 1e9, 1),
            "gemm_frac_roofline": round(t_roof_gemm / r["t_gemm"], 4),
            "gemm_frac_spec_int8": round(ops / r["t_gemm"] / 1e12 / SPEC_INT8_TOPS, 4),
            "quant_gbs": round(quant_bytes / r["t_quant"] / 1e9, 1),
            "quant_frac_hbm": round(quant_bytes / r["t_quant"] / 1e9 / peaks["hbm_gbs"], 4),
            "step_frac_roofline": round(t_roof_fused / r["t_step"], 4),
            "l2_sets": r["nsets"],
            "kernel": w8.gemm_kernel_name(wl.M, wl.N, wl.K),
        }
        if "gemm_clock" in r:
            # a long GEMM loop with its clocks: under the power cap the
            # sustained bf16 rate (x 2 for int8) is the ceiling it can reach
            sustained = 2.0 * peaks["bf16_tflops_sustained"]
            tops_long = ops / r["t_gemm_long"] / 1e12
            out[name]["gemm_long_loop"] = {
                "us": round(r["t_gemm_long"] * 1e6, 3), "tops": round(tops_long, 1),
                "sm_mhz": r["gemm_clock"]["sm_mhz"], "reasons": r["gemm_clock"]["reasons"],
                "frac_of_sustained": round(tops_long / sustained, 4),
                "sustained_peak_tops": round(sustained, 1)}
        del ls, loop
        torch.cuda.empty_cache()
    return out


def mlp_chain(w8, device, stream, steps=128, nsets=2):
    """The DiT MLP block (4096 tokens, 3072 -> 12288 -> 3072): the two W8A8
    layers with the GELU between them, unfused (layer, GELU kernel, layer)
    and with the GELU in the up-projection's epilogue."""
    up_wl = WORKLOADS["dit_mlp_up_4096x12288x3072"]
    dn_wl = WORKLOADS["dit_mlp_down_4096x3072x12288"]
    up, dn = make_inputs(up_wl), make_inputs(dn_wl)
    M, H, D = up_wl.M, up_wl.N, up_wl.K
    sets = []
    for i in range(nsets):
        s = {"x": bf16_dev(up.x, device),
             "pu": w8.pack_weight(torch.from_numpy(up.w).to(device)),
             "su": torch.from_numpy(up.w_scale).to(device), "bu": bf16_dev(up.bias, device),
             "pd": w8.pack_weight(torch.from_numpy(dn.w).to(device)),
             "sd": torch.from_numpy(dn.w_scale).to(device), "bd": bf16_dev(dn.bias, device),
             "h": torch.empty((M, H), dtype=torch.bfloat16, device=device),
             "g": torch.empty((M, H), dtype=torch.bfloat16, device=device),
             "y": torch.empty((M, D), dtype=torch.bfloat16, device=device),
             "wsu": torch.empty((w8.linear_workspace_bytes(M, H, D),), dtype=torch.uint8,
                                device=device),
             "wsd": torch.empty((w8.linear_workspace_bytes(M, D, H),), dtype=torch.uint8,
                                device=device)}
        sets.append(s)
    def unfused(s):
        w8.linear(s["x"], s["pu"], s["su"], s["bu"], H, out=s["h"], workspace=s["wsu"], stream=stream)
        w8.gelu_tanh(s["h"], out=s["g"], stream=stream)
        w8.linear(s["g"], s["pd"], s["sd"], s["bd"], D, out=s["y"], workspace=s["wsd"], stream=stream)
    def fused(s):
        w8.linear(s["x"], s["pu"], s["su"], s["bu"], H, out=s["g"], workspace=s["wsu"],
                  stream=stream, act=w8.ACT_GELU_TANH)
        w8.linear(s["g"], s["pd"], s["sd"], s["bd"], D, out=s["y"], workspace=s["wsd"], stream=stream)
    def up_only(s, act):
        w8.linear(s["x"], s["pu"], s["su"], s["bu"], H, out=s["g"], workspace=s["wsu"],
                  stream=stream, act=act)
    loops = {
        "unfused": GraphLoop([lambda s=s: unfused(s) for s in sets], stream, per_graph=8),
        "fused": GraphLoop([lambda s=s: fused(s) for s in sets], stream, per_graph=8),
        "up_layer": GraphLoop([lambda s=s: up_only(s, w8.ACT_NONE) for s in sets], stream, 16),
        "up_layer_gelu": GraphLoop([lambda s=s: up_only(s, w8.ACT_GELU_TANH) for s in sets],
                                   stream, 16),
        "gelu_kernel": GraphLoop([lambda s=s: w8.gelu_tanh(s["h"], out=s["g"], stream=stream)
                                  for s in sets], stream, 16),
    }
    torch.cuda.synchronize()
    for lp in loops.values():
        time_loop(lp, 3 * lp.per_graph, stream)
    ops = 2 * (2 * M * H * D)
    out = {"tokens": M, "dims": [D, H, D]}
    for name, lp in loops.items():
        # long enough (>= 0.6 s) for the clock sampler to see the loop
        t0 = time_loop(lp, lp.per_graph, stream) / lp.per_graph
        n = max(steps, int(0.6 / t0) // lp.per_graph * lp.per_graph)
        cs = ClockSampler(smi_index(device), tag="_mlp_" + name)
        cs.start()
        t = time_loop(lp, n, stream) / n
        clk = cs.stop()
        out[name + "_us"] = round(t * 1e6, 2)
        out[name + "_sm_mhz"] = clk["sm_mhz"]
        if clk["reasons"]:
            out[name + "_clock_reasons"] = clk["reasons"]
    for name in ("unfused", "fused"):
        out[name + "_tops"] = round(ops / (out[name + "_us"] * 1e-6) / 1e12, 1)
    assert w8.poll_status() == 0
    del sets, loops
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- CPU oracle
def cpu_baseline(wl, budget_s=12.0):
    """The oracle as it stands, on the host cores: whole layers of the same
    workload, repeated until about budget_s seconds have elapsed."""
    import oracle
    inp = make_inputs(wl)
    ops = 2 * wl.M * wl.N * wl.K
    oracle.linear(inp.x[:8], inp.w[:64], inp.w_scale[:64], None if inp.bias is None else inp.bias[:64])
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.linear(inp.x, inp.w, inp.w_scale, inp.bias)
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= 50:
            break
    t = (time.perf_counter() - t0) / reps
    return {"value": round(ops / t / 1e12, 5), "unit": "TOPS", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{reps} full {wl.name} layers (quant + int32 GEMM + epilogue), "
                      f"{t:.3f} s each, OpenMP over rows"}


def run_reference(args):
    wl = WORKLOADS[args.workload]
    import oracle
    inp = make_inputs(wl)
    ops = 2 * wl.M * wl.N * wl.K
    # bounded sample per step: a slice of rows of the same workload
    rows = max(1, min(wl.M, int(args.ref_rows)))
    x = inp.x[:rows]
    for _ in range(args.warmup):
        oracle.linear(x, inp.w, inp.w_scale, inp.bias)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear(x, inp.w, inp.w_scale, inp.bias)
    t = (time.perf_counter() - t0) / args.steps
    sample_ops = 2 * rows * wl.N * wl.K
    value = sample_ops / t / 1e12
    return {
        "metric": "W8A8 quant+scaled-GEMM TOPS and % of int8 roofline on one B200",
        "impl": "reference", "value": round(value, 5), "unit": "TOPS", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 x int8 -> int32, bf16 in/out", "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "M": wl.M, "N": wl.N, "K": wl.K,
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 5), "unit": "TOPS", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} of {wl.M} rows of {wl.name} per step "
                                   f"({sample_ops / ops:.3f} of a layer)"},
        "e2e": {"value": round(value, 5), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main
def main():
    global CLOCKS_DIR
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=MAIN_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--clocks-dir", default=None,
                    help="directory for the raw clock samples (default: a temporary one)")
    args = ap.parse_args()
    if args.clocks_dir:
        CLOCKS_DIR = os.path.abspath(args.clocks_dir)
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        out = run_ours(args, rank, world, device)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
