"""Run one workload's kernels a few times, for profiling under ncu.

    python -m w8a8_int8_dynamic_b200.profile_driver <workload> <reps> [gemm|decode|quant|linear|gelu]

Draws the workload's seeded inputs, packs the weights, then launches the
quantisation and the GEMM `reps` times (no CUDA graphs, so each kernel is a
separate launch that ncu can select with -k / -s / -c).
"""
import sys

import numpy as np
import torch

import w8a8_int8_dynamic_b200 as w8
from w8a8_int8_dynamic_b200.workloads import WORKLOADS, make_inputs


def main(argv):
    name, reps = argv[1], int(argv[2])
    mode = argv[3] if len(argv) > 3 else "gemm"
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    x = torch.from_numpy(inp.x.view(np.int16)).cuda().view(torch.bfloat16)
    packed = w8.pack_weight(torch.from_numpy(inp.w).cuda())
    ws = torch.from_numpy(inp.w_scale).cuda()
    b = None if inp.bias is None else torch.from_numpy(inp.bias.view(np.int16)).cuda().view(torch.bfloat16)
    q, a = w8.quant_act(x)
    mmws = torch.empty(max(16, w8.scaled_mm_workspace_bytes(wl.M, wl.N, wl.K)), dtype=torch.uint8,
                       device="cuda")
    y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device="cuda")
    layer_ws = torch.empty(w8.linear_workspace_bytes(wl.M, wl.N, wl.K), dtype=torch.uint8, device="cuda")
    g_in = None
    if mode == "gelu":  # the GELU kernel over an [M, N] activation (the MLP's up output)
        g_in = torch.randn(wl.M, wl.N, device="cuda",
                           generator=torch.Generator("cuda").manual_seed(0)).to(torch.bfloat16)
    for _ in range(reps):
        if mode == "gelu":
            w8.gelu_tanh(g_in, out=y)
        elif mode == "linear":
            w8.linear(x, packed, ws, b, wl.N, out=y, workspace=layer_ws)
        else:
            w8.quant_act(x, q=q, a_scale=a)
            if mode != "quant":
                w8.scaled_mm(q, a, packed, ws, b, wl.N, out=y, workspace=mmws)
    torch.cuda.synchronize()
    st = w8.poll_status()
    if st != 0:
        raise SystemExit(f"device status {st}")
    print("done", name, mode, reps)


if __name__ == "__main__":
    main(sys.argv)
