"""Benchmark of the W8A8 int8-dynamic linear path on B200.

One step = one pass of the hot path over one batch.  The default step is the
DiT transformer-block MLP at image-token scale (4096 tokens): the
up-projection 3072 -> 12288 with GELU(tanh) in its epilogue, then the
row-parallel down-projection 12288 -> 3072 fed its bf16 output.  Each layer
is w8a8_linear: dynamic per-token int8 quantisation of its input, the
int8 x int8 -> int32 tensor-core GEMM against weights packed once before
timing (load time), and the dequantising bf16 epilogue.  ``--workload NAME``
times a single layer of another workload instead.

Prints ONE JSON line (rank 0).  ``value`` is whole-job int8 TOPS (2*M*N*K of
every layer of every step, summed over ranks, divided by the max-over-ranks
device time).  Inputs rotate over enough buffer sets to exceed the 126 MB L2
between two uses, and consecutive steps are replayed from CUDA graphs so host
launch overhead stays out of the device timing.  Also reported: the dominant
kernel's roofline (the GEMM, timed alone with CUDA events on its stream), an
end-to-end figure through the public API with host buffers, the oracle's CPU
throughput, SM clocks sampled during the timed region, and a compact sweep
over the other workloads.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--no-sweep] [--no-cpu-baseline]
  python bench.py --profile MODE --workload NAME [--reps R]
      runs one workload's kernels R times as separate launches, without
      graphs, for ncu (MODE: layer, gemm, quant, gelu, block)
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

ACT_NONE, ACT_GELU = 0, 1  # w8a8_act
# A chain of layers, each fed the previous one's output: (layer workload,
# epilogue activation, whether the layer also forms the next layer's codes).
# A layer that does runs w8a8_linear_act_quant, and the next one then runs
# the scaled GEMM on those codes; any other layer runs w8a8_linear_act.
# The DiT MLP block: the up-projection with GELU in its epilogue, then the
# down-projection.  (The variant with the down-projection's quantisation
# fused into the up-projection is measured beside it: block_variants.)
BLOCK = "dit_mlp_block_4096x3072x12288"
CHAINS = {BLOCK: (("dit_mlp_up_4096x12288x3072", ACT_GELU, False),
                  ("dit_mlp_down_4096x3072x12288", ACT_NONE, False))}
BLOCK_FUSED_QUANT = (("dit_mlp_up_4096x12288x3072", ACT_GELU, True),
                     ("dit_mlp_down_4096x3072x12288", ACT_NONE, False))
MAIN_WORKLOAD = BLOCK
METRIC = "W8A8 quant+scaled-GEMM TOPS and % of int8 roofline on one B200"
# where the raw nvidia-smi clock samples go (--clocks-dir); the JSON line
# carries their summary either way
CLOCKS_DIR = os.path.join(tempfile.gettempdir(), "w8a8_bench_clocks")
L2_BYTES = 126 * 1024 * 1024
SPEC_INT8_TOPS = 4500.0


def chain_of(name):
    """The layers of a workload name: a chain, or one plain layer."""
    if name in CHAINS:
        return CHAINS[name]
    return ((name, ACT_NONE, False),)


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


# the sources each GEMM kernel is compiled from (a change voids its record)
_GEMM_HEADERS = ("gemm_common.cuh", "act.cuh", "f32x2.cuh", "quant_common.cuh", "ptx.cuh")
TRAFFIC_SOURCES = {
    "gemm_kernel": ("gemm.cu",) + _GEMM_HEADERS,
    "gemm2sm_kernel": ("gemm2sm.cu",) + _GEMM_HEADERS,
    "decode_kernel": ("decode.cu",) + _GEMM_HEADERS,
}


def code_text(src):
    """C / CUDA source with its comments removed and every run of whitespace
    made one space: what the compiler sees, so that an edit of comments or
    layout alone does not void a recorded measurement."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":  # string or character literal, copied whole
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def sources_hash(kernel):
    """First 16 hex digits of the sha256 of the code text (code_text) of a
    kernel family's sources, in TRAFFIC_SOURCES order, one line each."""
    import hashlib
    csrc = os.path.join(HERE, "w8a8_int8_dynamic_b200", "csrc")
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES[kernel]:
        src = open(os.path.join(csrc, f), encoding="utf-8").read()
        h.update((code_text(src) + "\n").encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per launch of a workload's GEMM from the committed ncu
    capture, or None when there is none or the kernel's sources changed
    since it was taken."""
    path = os.path.join(HERE, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(workload)
    if not rec or rec.get("kernel_family") not in TRAFFIC_SOURCES:
        return None
    if sources_hash(rec["kernel_family"]) != rec.get("source_sha256_16"):
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


def algorithmic(M, N, K, bias):
    """2MNK ops; GEMM bytes MK + NK + 2MN + scales (+ bias); quantisation
    bytes 3MK + 4M; the layer's bytes without the int8 round trip of q."""
    b = 2 * N if bias else 0
    ops = 2 * M * N * K
    gemm_bytes = M * K + N * K + 2 * M * N + 4 * M + 4 * N + b
    quant_bytes = 3 * M * K + 4 * M
    fused_bytes = 2 * M * K + N * K + 2 * M * N + 4 * N + b
    return ops, gemm_bytes, quant_bytes, fused_bytes


def chain_shapes(names, M=None):
    """(M, N, K, bias) of each layer of a chain."""
    out = []
    for name, *_ in names:
        wl = WORKLOADS[name]
        out.append((wl.M if M is None else M, wl.N, wl.K, wl.bias))
    return out


def footprints(shapes, layer_ws):
    """Bytes each timed loop touches per input set: the whole step, each
    layer's GEMM alone (q, W, y) and each layer's quantisation alone (x, q).
    A quantisation too small to exceed L2 even over 16 sets (it is
    latency-bound then) does not count."""
    step = sum(3 * M * K + N * K + 2 * M * N + 8 * N + ws
               for (M, N, K, _), ws in zip(shapes, layer_ws))
    fp = {"step": step}
    for i, (M, N, K, _) in enumerate(shapes):
        fp[f"gemm{i}"] = M * K + N * K + 2 * M * N
        if 16 * 3 * M * K > 1.5 * L2_BYTES:
            fp[f"quant{i}"] = 3 * M * K
    return fp


def sets_needed(fp):
    """Input sets to rotate over so that every timed loop touches more than
    L2 (x 1.5) between two uses of the same set (at most 16)."""
    smallest = min(fp.values())
    n = 1
    while n * smallest <= 1.5 * L2_BYTES and n < 16:
        n += 1
    return n


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


def per_graph_for(t_step_estimate):
    """Steps per captured graph: about 1 ms of work, between 4 and 64."""
    return int(min(64, max(4, 1e-3 / max(t_step_estimate, 1e-7))))


# ----------------------------------------------------------------------------- chains
class Layer:
    """One W8A8 layer of one input set on the device."""

    def __init__(self, w8, wl, act, inp, device, clone_of=None, fuse_next=False):
        self.wl, self.act, self.fuse_next = wl, act, fuse_next
        self.from_codes = False  # set by the chain: the previous layer forms its codes
        self.M, self.N, self.K = inp.x.shape[0], wl.N, wl.K
        if clone_of is None:
            self.packed = w8.pack_weight(torch.from_numpy(inp.w).to(device))
            self.w_scale = torch.from_numpy(inp.w_scale).to(device)
            self.bias = None if inp.bias is None else bf16_dev(inp.bias, device)
        else:
            self.packed = clone_of.packed.clone()
            self.w_scale = clone_of.w_scale.clone()
            self.bias = None if clone_of.bias is None else clone_of.bias.clone()
        M, N, K = self.M, self.N, self.K
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty((w8.linear_workspace_bytes(M, N, K),), dtype=torch.uint8,
                              device=device)
        mm = w8.scaled_mm_workspace_bytes(M, N, K)
        self.mmws = torch.empty((mm,), dtype=torch.uint8, device=device) if mm else None
        self.q = torch.empty((M, K), dtype=torch.int8, device=device)
        self.a = torch.empty((M,), dtype=torch.float32, device=device)
        self.aqws = (torch.empty((w8.linear_act_quant_workspace_bytes(M, N, K),),
                                 dtype=torch.uint8, device=device) if fuse_next else None)


class ChainSets:
    """``nsets`` independent copies of a chain's tensors on the device (the
    first layer's input x, every layer's packed weight, scales, bias, output
    and workspaces)."""

    def __init__(self, w8, names, nsets, device, M=None):
        self.names = names
        inps = [make_inputs(WORKLOADS[n], M) for n, *_ in names]
        self.M = inps[0].x.shape[0]
        x0 = bf16_dev(inps[0].x, device)
        self.sets = []
        for i in range(nsets):
            first = self.sets[0] if self.sets else None
            layers = [Layer(w8, WORKLOADS[n], act, inp, device,
                            None if first is None else first["layers"][j], fuse)
                      for j, ((n, act, fuse), inp) in enumerate(zip(names, inps))]
            for prev, L in zip(layers, layers[1:]):
                L.from_codes = prev.fuse_next
            self.sets.append({"x": x0 if i == 0 else x0.clone(), "layers": layers})
        del inps
        torch.cuda.synchronize()

    def inputs(self, s):
        """The input tensor of each layer of set s."""
        return [s["x"]] + [L.y for L in s["layers"][:-1]]

    def set_bytes(self):
        s = self.sets[0]
        n = s["x"].numel() * 2
        for L in s["layers"]:
            for t in (L.packed, L.w_scale, L.bias, L.y, L.ws, L.mmws, L.q, L.a, L.aqws):
                if t is not None:
                    n += t.numel() * t.element_size()
        return n


def run_chain(w8, cs, s, stream):
    x = s["x"]
    layers = s["layers"]
    for i, L in enumerate(layers):
        if L.from_codes:
            # codes and scales formed by the previous layer
            w8.scaled_mm(L.q, L.a, L.packed, L.w_scale, L.bias, L.N, out=L.y,
                         workspace=L.mmws, stream=stream, act=L.act)
        elif L.fuse_next:
            nxt = layers[i + 1]
            w8.linear_act_quant(x, L.packed, L.w_scale, L.bias, L.N, out=L.y, q_next=nxt.q,
                                a_scale_next=nxt.a, workspace=L.aqws, stream=stream, act=L.act)
        else:
            w8.linear(x, L.packed, L.w_scale, L.bias, L.N, out=L.y, workspace=L.ws, stream=stream,
                      act=L.act)
        x = L.y


def measure_chain(w8, names, steps, warmup, device, stream, with_layers=True, M=None,
                  long_gemm_clock=False, warm_gemm=False):
    """Times the chain step, and (with_layers) each layer's GEMM alone and
    quantisation alone, each over rotated input sets in CUDA graphs."""
    shapes = chain_shapes(names, M)
    ws_bytes = [w8.linear_workspace_bytes(m, n, k) for m, n, k, _ in shapes]
    nsets = sets_needed(footprints(shapes, ws_bytes))
    cs = ChainSets(w8, names, nsets, device, M)
    with torch.cuda.stream(stream):
        for s in cs.sets:
            run_chain(w8, cs, s, stream)  # warm the launch path; layer inputs exist
        for s in cs.sets:
            for L, x in zip(s["layers"], cs.inputs(s)):
                w8.quant_act(x, q=L.q, a_scale=L.a, stream=stream)
    torch.cuda.synchronize()
    c0 = w8.launch_count()
    capture([lambda: run_chain(w8, cs, cs.sets[0], stream)], stream)
    per_step = w8.launch_count() - c0
    ops = [algorithmic(*sh)[0] for sh in shapes]
    est = sum(ops) / 2.0e15
    step_loop = GraphLoop([lambda s=s: run_chain(w8, cs, s, stream) for s in cs.sets], stream,
                          per_graph_for(est))
    loops = {"step": step_loop}
    if with_layers:
        for i in range(len(names)):
            def mm(s, i=i):
                L = s["layers"][i]
                w8.scaled_mm(L.q, L.a, L.packed, L.w_scale, L.bias, L.N, out=L.y,
                             workspace=L.mmws, stream=stream, act=L.act)

            def qa(s, i=i):
                L = s["layers"][i]
                w8.quant_act(cs.inputs(s)[i], q=L.q, a_scale=L.a, stream=stream)
            # (each callable binds this layer's functions: the loops' tail
            # graphs are captured after this loop has moved on)
            loops[f"gemm{i}"] = GraphLoop([lambda s=s, f=mm: f(s) for s in cs.sets], stream,
                                          per_graph_for(ops[i] / 2.0e15))
            loops[f"quant{i}"] = GraphLoop([lambda s=s, f=qa: f(s) for s in cs.sets], stream,
                                           per_graph_for(3e-6))
            if warm_gemm:
                # the same set over and over: operands resident in L2 when they fit
                loops[f"gemm{i}_warm"] = GraphLoop([lambda f=mm: f(cs.sets[0])], stream,
                                                   per_graph_for(ops[i] / 2.0e15))
    for lp in loops.values():
        lp.prepare(steps)
    torch.cuda.synchronize()
    assert w8.poll_status() == 0
    for lp in loops.values():
        time_loop(lp, max(warmup, 3) * lp.per_graph, stream)
    res = {"launches_per_step": per_step, "nsets": nsets, "set_bytes": cs.set_bytes(),
           "shapes": shapes, "ops": ops}
    for k, lp in loops.items():
        res["t_" + k] = time_loop(lp, steps, stream) / steps
    if long_gemm_clock:
        # each GEMM again, long enough (>= 0.6 s) for the clock sampler: a
        # tensor-bound loop may run under the power cap
        for i in range(len(names)):
            lp = loops[f"gemm{i}"]
            n = max(steps, int(0.6 / res[f"t_gemm{i}"]) // lp.per_graph * lp.per_graph)
            cs_ = ClockSampler(smi_index(device), tag=f"_gemm{i}")
            cs_.start()
            res[f"t_gemm{i}_long"] = time_loop(lp, n, stream) / n
            res[f"gemm{i}_clock"] = cs_.stop()
    assert w8.poll_status() == 0, "device-side timeout during the benchmark"
    return cs, step_loop, res


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, device):
    import w8a8_int8_dynamic_b200 as w8
    w8.lib()
    peaks = load_peaks()
    int8_peak = 2.0 * peaks["bf16_tflops"]  # nominal int8 : bf16 dense rate = 2
    stream = torch.cuda.Stream(device=device)
    names = chain_of(args.workload)

    cs, step_loop, base = measure_chain(w8, names, 2000 if len(names) == 1 else 400,
                                        args.warmup, device, stream, long_gemm_clock=True)
    shapes, ops_l = base["shapes"], base["ops"]
    ops = sum(ops_l)
    step_loop.prepare(args.steps)
    torch.cuda.synchronize()
    # ---- the timed region: exactly K steps, barrier + sync on both sides
    sampler = ClockSampler(smi_index(device))
    sampler.start()
    time_loop(step_loop, args.warmup, stream)  # W untimed warm-up steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        step_loop.run(args.steps)
        end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    elapsed = start.elapsed_time(end) / 1e3
    clocks = sampler.stop()
    assert w8.poll_status() == 0, "device-side timeout during the timed region"
    t_max = max_over_ranks(elapsed, world, device)
    value = whole_job_tops(ops, args.steps, world, t_max)
    ms_per_step = t_max / args.steps * 1e3
    per_graph = step_loop.per_graph

    # ---- dominant kernel: the GEMM of every layer, each timed alone (without
    # the fused quantisation); the algorithmic ops of one launch over the mean
    # launch duration
    t_g = [base[f"t_gemm{i}"] for i in range(len(names))]
    gemm_tops = ops / sum(t_g) / 1e12
    # the int8 tensor-core rate with no memory traffic, measured here now
    with torch.cuda.stream(stream):
        mma_ceiling = w8.selftest_int8_mma_rate(20000, stream=stream)
    kernels = [w8.gemm_kernel_name(M, N, K) for M, N, K, _ in shapes]
    traffic = [recorded_traffic(n) for n, *_ in names]
    roofline = {
        "bound": "tensor", "achieved": round(gemm_tops, 1), "peak": round(int8_peak, 1),
        "unit": "TOPS", "frac": round(gemm_tops / int8_peak, 4),
        "traffic": None if None in traffic else int(sum(traffic) / len(traffic)),
        "kernel": kernels[0].split(" (")[0] if len(set(kernels)) == 1 else kernels,
        "peak_note": f"2 x {peaks['source']} bf16 burst",
        "frac_vs_spec_4500": round(gemm_tops / SPEC_INT8_TOPS, 4),
        "frac_vs_mma_ceiling": round(gemm_tops / mma_ceiling, 4),
        "mma_ceiling": round(mma_ceiling, 1),
        "ops_per_launch": ops_l[0] if len(set(ops_l)) == 1 else ops_l,
        "gemm_us": [round(t * 1e6, 2) for t in t_g],
        "quant_us": [round(base[f"t_quant{i}"] * 1e6, 2) for i in range(len(names))],
        "quant_frac_hbm": [round(algorithmic(*sh)[2] / base[f"t_quant{i}"] / 1e9 /
                                 peaks["hbm_gbs"], 4) for i, sh in enumerate(shapes)],
    }
    sustained = 2.0 * peaks["bf16_tflops_sustained"]
    t_long = [base[f"t_gemm{i}_long"] for i in range(len(names))]
    clk = [base[f"gemm{i}_clock"] for i in range(len(names))]
    roofline["long_loop"] = {
        "frac_of_sustained": round(ops / sum(t_long) / 1e12 / sustained, 4),
        "sustained_peak": round(sustained, 1),
        "sm_mhz": [c["sm_mhz"] for c in clk],
        "reasons": sorted({r for c in clk for r in c["reasons"]})}
    t_roof = 0.0
    for sh in shapes:
        o, _, _, fused = algorithmic(*sh)
        t_roof += max(o / (int8_peak * 1e12), fused / (peaks["hbm_gbs"] * 1e9))

    # ---- end to end through the public API, host buffers
    e2e = run_e2e(w8, cs, args, stream, ops, world, device)
    del cs, step_loop
    torch.cuda.empty_cache()

    first = WORKLOADS[names[0][0]]
    out = {
        "metric": METRIC,
        "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8 x int8 -> int32, bf16 in/out",
        "data": "synthetic, seeded (workloads.py recipe)",
        "config": {"workload": args.workload, "M": first.M if len(names) > 1 else shapes[0][0],
                   "layers": [f"{M}x{N}x{K}" + ("+gelu" if a else "") + ("+quant_next" if f else "")
                              for (M, N, K, _), (_, a, f) in zip(shapes, names)],
                   "step": step_description(names),
                   "l2": f"{base['nsets']} rotated input sets of "
                         f"{base['set_bytes'] / 2**20:.0f} MiB (> 126 MB L2)",
                   "launch": f"CUDA graphs of {per_graph} steps",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "step_frac_of_roofline": round(t_roof / (t_max / args.steps), 4),
        "e2e": e2e,
        "gpu_launches": int(base["launches_per_step"] * args.steps),
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:  # the oracle, at N = 1 only
        out["cpu_baseline"] = cpu_baseline(names, budget_s=args.cpu_seconds)
    if not args.no_sweep:
        out["sweep_cols"] = SWEEP_COLS
        out["sweep"] = sweep(w8, args, device, stream, peaks, int8_peak)
        if args.workload == BLOCK:
            out["block_variants_us"] = block_variants(w8, device, stream)
    return out


def step_description(names):
    if len(names) == 1:
        return "w8a8_linear: quant kernel + tcgen05 GEMM/epilogue (PDL)"
    if names[0][2]:
        return ("w8a8_linear_act_quant (quant, GEMM+GELU+codes of its output) + "
                "w8a8_scaled_mm on those codes")
    return (f"{len(names)} x w8a8_linear_act (quant kernel + tcgen05 GEMM/epilogue, PDL), "
            "GELU in the first epilogue")


def max_over_ranks(elapsed, world, device):
    """The slowest rank's time: every rank takes part (one all-reduce)."""
    if world == 1:
        return elapsed
    t = torch.tensor([elapsed], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_step, steps, world, t_max):
    """Replicas: every rank runs `steps` steps; the job's throughput is all
    ranks' work over the slowest rank's time."""
    return ops_per_step * steps * world / t_max / 1e12


def e2e_record(ops_per_step, steps, elapsed, world, device, h2d_bytes, d2h_bytes):
    """The end-to-end leg as a whole-job figure, like `value`: every rank's
    steps over the slowest rank's time, and the bytes all ranks copy a step
    (replicas: each rank moves its own)."""
    t_max = max_over_ranks(elapsed, world, device)
    return {"value": round(whole_job_tops(ops_per_step, steps, world, t_max), 2),
            "unit": "TOPS", "h2d_bytes_per_step": h2d_bytes * world,
            "d2h_bytes_per_step": d2h_bytes * world, "steps": steps,
            "ms_per_step": round(t_max / steps * 1e3, 4)}


# host <-> device copies of a step, each in this many cudaMemcpyAsync pieces:
# two halves let the two directions interleave on PCIe (DiT MLP block, 25 MB
# each way: 0.533 ms a step against 0.573 ms with whole copies; the copies
# alone take 0.532 ms; 8 or more pieces cost more host time than they save)
E2E_PIECES = 2


def run_e2e(w8, cs, args, stream, ops, world=1, device=None):
    """Public API, host buffers: per step H2D of the first layer's input from
    pinned memory, the layers, D2H of the last layer's output into pinned
    memory, all inside the timed region.  Steps are pipelined the way a
    serving loop would run them: the upload of step i+1, the layers of step
    i and the download of step i-1 overlap on three streams (PCIe is full
    duplex), with three device buffer sets.  Every pinned host buffer is
    used once before timing (a pinned buffer's first copy is slow), and at
    least 50 steps are timed so that filling and draining the pipeline
    (about one step) weighs little."""
    s0 = cs.sets[0]
    ndev = min(3, len(cs.sets))
    nhost = 4
    dev = s0["x"].device
    x_shape = tuple(s0["x"].shape)
    y_shape = tuple(s0["layers"][-1].y.shape)
    xs = [s0["x"].cpu().pin_memory() for _ in range(nhost)]
    ys = [torch.empty(y_shape, dtype=torch.bfloat16).pin_memory() for _ in range(nhost)]
    dsets = [cs.sets[i] for i in range(ndev)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    comp = stream
    ev_in = [torch.cuda.Event() for _ in range(ndev)]
    ev_done = [torch.cuda.Event() for _ in range(ndev)]
    ev_out = [torch.cuda.Event() for _ in range(ndev)]

    def copy(dst, src):
        a, b = dst.view(-1), src.view(-1)
        n = a.numel()
        for j in range(E2E_PIECES):
            lo, hi = n * j // E2E_PIECES, n * (j + 1) // E2E_PIECES
            a[lo:hi].copy_(b[lo:hi], non_blocking=True)

    def step(i, first):
        b = i % ndev
        d = dsets[b]
        if not first[b]:
            up.wait_event(ev_done[b])        # x[b] free: the layers that read it are done
        with torch.cuda.stream(up):
            copy(d["x"], xs[i % nhost])
            ev_in[b].record(up)
        comp.wait_event(ev_in[b])
        if not first[b]:
            comp.wait_event(ev_out[b])       # y[b] free: its download is done
        run_chain(w8, cs, d, comp)
        ev_done[b].record(comp)
        down.wait_event(ev_done[b])
        with torch.cuda.stream(down):
            copy(ys[i % nhost], d["layers"][-1].y)
            ev_out[b].record(down)
        first[b] = False

    steps = max(50, min(args.steps, 200))
    first = [True] * ndev
    for i in range(max(nhost, ndev)):
        step(i, first)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
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
    elapsed = start.elapsed_time(end) / 1e3
    # the last step's output must have arrived
    last = dsets[(steps - 1) % ndev]["layers"][-1].y
    assert torch.equal(ys[(steps - 1) % nhost].to(dev), last)
    xb = int(np.prod(x_shape)) * 2
    yb = int(np.prod(y_shape)) * 2
    rec = e2e_record(ops, steps, elapsed, world, device, xb, yb)
    rec["overlap"] = f"H2D i+1 | layers i | D2H i-1, 3 streams, copies in {E2E_PIECES} pieces"
    rec["api"] = "+".join(sorted({"w8a8_linear_act_quant" if L.fuse_next else
                                  "w8a8_scaled_mm" if L.from_codes else "w8a8_linear_act"
                                  for L in s0["layers"]}))
    return rec


# compact sweep rows: one list per workload, columns named once
SWEEP_COLS = ["kernel", "step_us", "gemm_us", "quant_us", "gemm_frac", "quant_frac_hbm",
              "step_frac", "gemm_us_warm"]
SWEEP = ["small_64x128x256", "square_512x4096x4096", "fused_qkv_512x12288x4096",
         "dit_mlp_up_4096x12288x3072", "dit_mlp_down_4096x3072x12288",
         "decode_m1_27648x5120", "decode_m4_27648x5120", "decode_m16_27648x5120"]


def short_kernel(name):
    """'gemm2sm_kernel<256, 3> (...)' -> 'pair256'."""
    if name.startswith("decode"):
        return "decode"
    if name.startswith("gemm2sm"):
        return "pair" + name.split("<")[1].split(",")[0]
    return "1sm" + name.split("<")[1].split(",")[0]


def sweep_steps(ops, gemm_bytes, int8_peak_tops, hbm_gbs, work_s=25e-3):
    """Steps of a sweep loop: about `work_s` of work (a layer estimated at 0.6
    of the int8 peak or 0.8 of HBM, whichever is slower), 100 to 2000 steps,
    so that each loop finishes before the power cap settles, like the burst
    peak it is read against (the headline's long loops give the sustained
    figure)."""
    t_est = max(ops / (int8_peak_tops * 1e12 * 0.6), gemm_bytes / (hbm_gbs * 1e9 * 0.8))
    return int(min(2000, max(100, work_s / t_est)))


def sweep(w8, args, device, stream, peaks, int8_peak):
    """Every workload as one layer: step (quant + GEMM), GEMM alone (cold
    operands; warm too where they fit L2), quantisation alone.  gemm_frac is
    t_roof / t for the GEMM (tensor or HBM bound, whichever is slower),
    quant_frac_hbm the quantisation's fraction of HBM bandwidth, step_frac the
    layer's fraction of its roofline."""
    out = {}
    for name in SWEEP:
        wl = WORKLOADS[name]
        ops, gemm_bytes, quant_bytes, fused_bytes = algorithmic(wl.M, wl.N, wl.K, wl.bias)
        steps = sweep_steps(ops, gemm_bytes, int8_peak, peaks["hbm_gbs"])
        warm = wl.N * wl.K + wl.M * wl.K + 2 * wl.M * wl.N < L2_BYTES // 2
        cs, loop, r = measure_chain(w8, chain_of(name), steps, 3, device, stream,
                                    warm_gemm=warm)
        t_roof_gemm = max(ops / (int8_peak * 1e12), gemm_bytes / (peaks["hbm_gbs"] * 1e9))
        t_roof_step = max(ops / (int8_peak * 1e12), fused_bytes / (peaks["hbm_gbs"] * 1e9))
        row = [short_kernel(w8.gemm_kernel_name(wl.M, wl.N, wl.K)),
               round(r["t_step"] * 1e6, 2), round(r["t_gemm0"] * 1e6, 2),
               round(r["t_quant0"] * 1e6, 2), round(t_roof_gemm / r["t_gemm0"], 3),
               round(quant_bytes / r["t_quant0"] / 1e9 / peaks["hbm_gbs"], 3),
               round(t_roof_step / r["t_step"], 3)]
        if warm:
            row.append(round(r["t_gemm0_warm"] * 1e6, 2))
        out[name] = row
        del cs, loop
        torch.cuda.empty_cache()
    return out


def block_variants(w8, device, stream, nsets=4, steps=64):
    """The DiT MLP block in three forms, same inputs and loop, microseconds a
    step: "layers" -- the headline step's two w8a8_linear_act calls;
    "fused_quant" -- the down-projection's quantisation fused into the
    up-projection (w8a8_linear_act_quant), then the scaled GEMM on its codes;
    "unfused" -- layer, GELU kernel, layer."""
    cs = ChainSets(w8, BLOCK_FUSED_QUANT, nsets, device)
    gs = [torch.empty_like(s["layers"][0].y) for s in cs.sets]

    def layers(s, g):
        Lu, Ld = s["layers"]
        w8.linear(s["x"], Lu.packed, Lu.w_scale, Lu.bias, Lu.N, out=Lu.y, workspace=Lu.ws,
                  stream=stream, act=Lu.act)
        w8.linear(Lu.y, Ld.packed, Ld.w_scale, Ld.bias, Ld.N, out=Ld.y, workspace=Ld.ws,
                  stream=stream)

    def fused_quant(s, g):
        run_chain(w8, cs, s, stream)

    def unfused(s, g):
        Lu, Ld = s["layers"]
        w8.linear(s["x"], Lu.packed, Lu.w_scale, Lu.bias, Lu.N, out=Lu.y, workspace=Lu.ws,
                  stream=stream)
        w8.gelu_tanh(Lu.y, out=g, stream=stream)
        w8.linear(g, Ld.packed, Ld.w_scale, Ld.bias, Ld.N, out=Ld.y, workspace=Ld.ws,
                  stream=stream)
    out = {}
    for name, fn in (("layers", layers), ("fused_quant", fused_quant), ("unfused", unfused)):
        lp = GraphLoop([lambda s=s, g=g, f=fn: f(s, g) for s, g in zip(cs.sets, gs)], stream, 4)
        lp.prepare(steps)
        time_loop(lp, 3 * lp.per_graph, stream)
        out[name] = round(time_loop(lp, steps, stream) / steps * 1e6, 2)
        del lp
    assert w8.poll_status() == 0
    del cs, gs
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- CPU oracle
def oracle_chain(oracle, names, x, inps):
    """The chain through the oracle: each layer, then GELU where it has one
    (the codes a layer forms for the next are the next layer's own)."""
    for (name, act, _), inp in zip(names, inps):
        x = oracle.linear(x, inp.w, inp.w_scale, inp.bias)[0]
        if act == ACT_GELU:
            x = oracle.gelu_tanh(x)
    return x


def cpu_baseline(names, budget_s=12.0):
    """The oracle as it stands, on the host cores: whole steps of the same
    workload (every layer at full size), repeated until about budget_s
    seconds have elapsed; plus single-thread figures for the three smaller
    workloads (a row sample of each)."""
    import oracle
    inps = [make_inputs(WORKLOADS[n]) for n, *_ in names]
    ops = sum(algorithmic(*sh)[0] for sh in chain_shapes(names))
    oracle_chain(oracle, names, inps[0].x[:4], inps)  # load and touch
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle_chain(oracle, names, inps[0].x, inps)
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= 50:
            break
    t = (time.perf_counter() - t0) / reps
    cores = oracle.num_threads()
    single = {}
    oracle.set_num_threads(1)
    try:
        for name, rows in (("small_64x128x256", 64), ("square_512x4096x4096", 32),
                           ("fused_qkv_512x12288x4096", 16)):
            wl = WORKLOADS[name]
            inp = make_inputs(wl)
            x = inp.x[:rows]
            t1 = time.perf_counter()
            oracle.linear(x, inp.w, inp.w_scale, inp.bias)
            dt = time.perf_counter() - t1
            single[name] = [round(2 * rows * wl.N * wl.K / dt / 1e12, 5), rows]
    finally:
        oracle.set_num_threads(cores)
    del inps
    return {"value": round(ops / t / 1e12, 5), "unit": "TOPS", "cores": cores,
            "kind": "oracle",
            "sample": f"{reps} whole step(s) of {len(names)} full layer(s), {t:.2f} s each",
            "single_thread_tops_rows": single}


def run_reference(args):
    """The oracle, as it stands, on the host cores: each step a bounded
    sample of the same workload (its first rows through every layer)."""
    import oracle
    names = chain_of(args.workload)
    inps = [make_inputs(WORKLOADS[n]) for n, *_ in names]
    shapes = chain_shapes(names)
    M = shapes[0][0]
    rows = max(1, min(M, int(args.ref_rows)))
    x = inps[0].x[:rows]
    for _ in range(args.warmup):
        oracle_chain(oracle, names, x, inps)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_chain(oracle, names, x, inps)
    t = (time.perf_counter() - t0) / args.steps
    sample_ops = sum(2 * rows * N * K for _, N, K, _ in shapes)
    full_ops = sum(algorithmic(*sh)[0] for sh in shapes)
    value = sample_ops / t / 1e12
    return {
        "metric": METRIC, "impl": "reference", "value": round(value, 5), "unit": "TOPS",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8 x int8 -> int32, bf16 in/out",
        "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "M": M,
                   "layers": [f"{m}x{n}x{k}" for m, n, k, _ in shapes],
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 5), "unit": "TOPS", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} of {M} rows through every layer per step "
                                   f"({sample_ops / full_ops:.4f} of a step)"},
        "e2e": {"value": round(value, 5), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- profiling
def run_profile(args):
    """A workload's kernels as separate launches (no graphs), so that ncu can
    select them with -k / -s / -c.  MODE layer: w8a8_linear; gemm: the
    quantisation then the GEMM alone; quant: the quantisation; gelu: the
    GELU kernel over the layer's output shape; block: the chain."""
    import w8a8_int8_dynamic_b200 as w8
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    names = chain_of(args.workload)
    cs = ChainSets(w8, names, 1, device)
    s = cs.sets[0]
    mode = args.profile
    L0 = s["layers"][0]
    g_in = None
    if mode == "gelu":
        g_in = torch.randn(L0.M, L0.N, device=device,
                           generator=torch.Generator(device).manual_seed(0)).to(torch.bfloat16)
    for _ in range(args.reps):
        if mode in ("block", "layer"):
            run_chain(w8, cs, s, stream)
        elif mode == "gelu":
            w8.gelu_tanh(g_in, out=L0.y)
        else:
            for L, x in zip(s["layers"], cs.inputs(s)):
                w8.quant_act(x, q=L.q, a_scale=L.a)
                if mode == "gemm":
                    w8.scaled_mm(L.q, L.a, L.packed, L.w_scale, L.bias, L.N, out=L.y,
                                 workspace=L.mmws, act=L.act)
    torch.cuda.synchronize()
    st = w8.poll_status()
    if st != 0:
        raise SystemExit(f"device status {st}")
    print("done", args.workload, mode, args.reps)


# ----------------------------------------------------------------------------- main
def main():
    global CLOCKS_DIR
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=MAIN_WORKLOAD, choices=list(CHAINS) + list(WORKLOADS))
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=5.0)
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--profile", choices=["layer", "gemm", "quant", "gelu", "block"], default=None)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--clocks-dir", default=None,
                    help="directory for the raw clock samples (default: a temporary one)")
    args = ap.parse_args()
    if args.clocks_dir:
        CLOCKS_DIR = os.path.abspath(args.clocks_dir)
    args.warmup = max(args.warmup, 3)

    if args.profile:
        run_profile(args)
        return 0

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
            print(json.dumps(out, separators=(",", ":")), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
