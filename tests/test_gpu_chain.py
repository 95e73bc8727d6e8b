"""Layers in a chain: each layer's input is the previous layer's output, the
calls queued back to back on one stream with one shared workspace.

The quantisation kernel is a programmatic dependent launch and the decode
kernel releases the next kernel of the stream early, so the next layer's
kernels can be resident while the previous layer still runs.  The bar: every
layer's output bit-identical to the oracle applied layer by layer, both for
eager calls and for a CUDA graph of the chain replayed several times.
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_int8_dynamic_b200 as w8
from gpu_util import assert_bf16_close, dev, dev_bf16, host_u16, require_gpu
from w8a8_int8_dynamic_b200.workloads import random_case

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    w8.set_path(w8.PATH_AUTO)
    yield
    w8.set_path(w8.PATH_AUTO)
    assert w8.poll_status() == 0, "a kernel reported a device-side timeout"


def _chain_case(M, D, L, seed):
    x0 = random_case(seed, M, D, D, bias=True, n_outliers=D // 64).x
    layers = [random_case(seed + 101 * (l + 1), M, D, D, bias=True) for l in range(L)]
    ys, x = [], x0
    for inp in layers:
        y, *_ = oracle.linear(x, inp.w, inp.w_scale, inp.bias)
        ys.append(y)
        x = y
    return x0, layers, ys


@pytest.mark.parametrize("M", [1, 4, 16, 300])
def test_layer_chain_matches_oracle(M):
    D, L = 1024, 4
    x0, layers, ys_ref = _chain_case(M, D, L, 11 + M)
    packed = [w8.pack_weight(dev(inp.w)) for inp in layers]
    w_scale = [dev(inp.w_scale) for inp in layers]
    bias = [dev_bf16(inp.bias) for inp in layers]
    x = dev_bf16(x0)
    ys = [torch.empty((M, D), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    ws = torch.empty((w8.linear_workspace_bytes(M, D, D),), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def chain():
        inp = x
        for l in range(L):
            w8.linear(inp, packed[l], w_scale[l], bias[l], D, out=ys[l], workspace=ws, stream=stream)
            inp = ys[l]

    with torch.cuda.stream(stream):
        chain()
    stream.synchronize()
    for l in range(L):
        assert np.array_equal(host_u16(ys[l]), ys_ref[l]), f"eager chain, layer {l}"

    for y in ys:
        y.fill_(0)
    with torch.cuda.stream(stream):
        chain()  # warm the launch path before capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            chain()
        for y in ys:
            y.fill_(0)
        for _ in range(3):
            g.replay()
    stream.synchronize()
    for l in range(L):
        assert np.array_equal(host_u16(ys[l]), ys_ref[l]), f"graph replay, layer {l}"
    del g


def test_quant_after_decode_reads_its_output():
    """A standalone quantisation queued right behind a decode GEMM that
    released it early must still see that GEMM's output."""
    M, D = 4, 2064
    inp = random_case(5, M, D, D, bias=True)
    y_ref, *_ = oracle.linear(inp.x, inp.w, inp.w_scale, inp.bias)
    q2_ref, s2_ref = oracle.quant_act(y_ref)
    ws = torch.empty((w8.linear_workspace_bytes(M, D, D),), dtype=torch.uint8, device="cuda")
    y = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    packed = w8.pack_weight(dev(inp.w))
    for _ in range(5):
        y.fill_(0)
        w8.linear(dev_bf16(inp.x), packed, dev(inp.w_scale), dev_bf16(inp.bias), D, out=y,
                  workspace=ws)
        q2, s2 = w8.quant_act(y)
        torch.cuda.synchronize()
        assert np.array_equal(q2.cpu().numpy(), q2_ref)
        assert np.array_equal(s2.cpu().numpy(), s2_ref)


@pytest.mark.parametrize("M", [4, 300])
def test_mlp_block_chain(M):
    """The MLP pattern: up-projection with the GELU epilogue, then the
    down-projection on its output, queued back to back (the down-projection's
    quantisation waits on the device for the up-projection).  The up output
    is within one bf16 ulp of the oracle's GELU chain; the down-projection is
    checked bit for bit against the oracle fed the GPU's own GELU output (the
    two sides' GELU may differ by an ulp)."""
    D, H = 1024, 2064
    up = random_case(21 + M, M, H, D, bias=True, n_outliers=D // 64)
    dn = random_case(22 + M, M, D, H, bias=True)
    y_up_ref, *_ = oracle.linear(up.x, up.w, up.w_scale, up.bias)
    g_ref = oracle.gelu_tanh(y_up_ref)
    ws_up = torch.empty((w8.linear_workspace_bytes(M, H, D),), dtype=torch.uint8, device="cuda")
    ws_dn = torch.empty((w8.linear_workspace_bytes(M, D, H),), dtype=torch.uint8, device="cuda")
    p_up, p_dn = w8.pack_weight(dev(up.w)), w8.pack_weight(dev(dn.w))
    x = dev_bf16(up.x)
    g = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        g.fill_(0)
        y.fill_(0)
        w8.linear(x, p_up, dev(up.w_scale), dev_bf16(up.bias), H, out=g, workspace=ws_up,
                  act=w8.ACT_GELU_TANH)
        w8.linear(g, p_dn, dev(dn.w_scale), dev_bf16(dn.bias), D, out=y, workspace=ws_dn)
        torch.cuda.synchronize()
        g_h = host_u16(g)
        assert_bf16_close(g_h, g_ref, max_ulp=1, what="gelu chain")
        y_ref, *_ = oracle.linear(g_h, dn.w, dn.w_scale, dn.bias)
        assert np.array_equal(host_u16(y), y_ref)
