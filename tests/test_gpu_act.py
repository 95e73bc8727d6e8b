"""GELU(tanh) fused into the GEMM epilogue (the MLP up-projection followed by
its activation, without the bf16 round trip of the projection's output).

Bar: the fused output is bit-identical to the unfused GPU chain (layer, then
the standalone GELU kernel), on every GEMM kernel, and within one bf16 ulp of
the oracle's chain (the oracle's GELU is evaluated in double).
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_int8_dynamic_b200 as w8
from gpu_util import assert_bf16_close, dev, dev_bf16, host_u16, require_gpu
from w8a8_int8_dynamic_b200.workloads import WORKLOADS, make_inputs, random_case

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    w8.set_path(w8.PATH_AUTO)
    yield
    w8.set_path(w8.PATH_AUTO)
    assert w8.poll_status() == 0, "a kernel reported a device-side timeout"


def _case(M, N, K, bias, seed):
    inp = random_case(seed, M, N, K, bias=bias, n_outliers=K // 64, zero_row=True)
    q_ref, s_ref = oracle.quant_act(inp.x)
    y_ref = oracle.epilogue(oracle.gemm_i32(q_ref, inp.w), s_ref, inp.w_scale, inp.bias)
    return inp, q_ref, s_ref, y_ref


@pytest.mark.parametrize("bias", [False, True])
@pytest.mark.parametrize("path", [w8.PATH_LARGE_BN128, w8.PATH_LARGE_BN256, w8.PATH_LARGE_PAIR,
                                  w8.PATH_LARGE_PAIR128])
@pytest.mark.parametrize("M,N,K", [(64, 128, 256), (129, 392, 400), (300, 1000, 528),
                                   (512, 1024, 4096), (700, 520, 144)])
def test_scaled_mm_gelu_fused_equals_chain(M, N, K, path, bias):
    w8.set_path(path)
    inp, q_ref, s_ref, y_ref = _case(M, N, K, bias, M * 3 + N + K)
    b = None if inp.bias is None else dev_bf16(inp.bias)
    args = (dev(q_ref), dev(s_ref), w8.pack_weight(dev(inp.w)), dev(inp.w_scale), b, N)
    y = w8.scaled_mm(*args)
    g_chain = w8.gelu_tanh(y)
    g_fused = w8.scaled_mm(*args, act=w8.ACT_GELU_TANH)
    torch.cuda.synchronize()
    assert np.array_equal(host_u16(y), y_ref)
    assert torch.equal(g_fused, g_chain), "fused GELU differs from layer + GELU kernel"
    assert_bf16_close(host_u16(g_fused), oracle.gelu_tanh(y_ref), max_ulp=1, what="gelu")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_gelu_fused_equals_chain(M):
    N, K = 2056, 1040
    inp, q_ref, s_ref, y_ref = _case(M, N, K, True, 77 + M)
    ws = torch.empty((w8.scaled_mm_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    args = (dev(q_ref), dev(s_ref), w8.pack_weight(dev(inp.w)), dev(inp.w_scale),
            dev_bf16(inp.bias), N)
    y = w8.scaled_mm(*args, workspace=ws)
    g_chain = w8.gelu_tanh(y)
    g_fused = w8.scaled_mm(*args, workspace=ws, act=w8.ACT_GELU_TANH)
    torch.cuda.synchronize()
    assert np.array_equal(host_u16(y), y_ref)
    assert torch.equal(g_fused, g_chain)
    assert_bf16_close(host_u16(g_fused), oracle.gelu_tanh(y_ref), max_ulp=1, what="gelu")


@pytest.mark.parametrize("M", [3, 200])
def test_linear_gelu_matches_oracle_chain(M):
    N, K = 776, 1296
    inp, _, _, _ = _case(M, N, K, True, 5 + M)
    y_ref, *_ = oracle.linear(inp.x, inp.w, inp.w_scale, inp.bias)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias), act=w8.ACT_GELU_TANH)
    g = layer(dev_bf16(inp.x))
    torch.cuda.synchronize()
    assert_bf16_close(host_u16(g), oracle.gelu_tanh(y_ref), max_ulp=1, what="gelu")


def test_dit_mlp_up_fused_gelu_full_size():
    """The 4096 x 12288 x 3072 up-projection: fused output bit-identical to
    the unfused chain over all 50M elements."""
    up = make_inputs(WORKLOADS["dit_mlp_up_4096x12288x3072"])
    x = dev_bf16(up.x)
    plain = w8.W8A8Linear(dev(up.w), dev(up.w_scale), dev_bf16(up.bias))
    fused = w8.W8A8Linear(dev(up.w), dev(up.w_scale), dev_bf16(up.bias), act=w8.ACT_GELU_TANH)
    g_chain = w8.gelu_tanh(plain(x))
    g_fused = fused(x)
    torch.cuda.synchronize()
    assert torch.equal(g_fused, g_chain)


def test_gelu_epilogue_on_half_tiles():
    """A shape whose last round of 256 x 256 pair tiles runs as 256 x 128
    halves (99 tiles on 74 pairs; the last tile ragged in M and N): the GELU
    epilogue on the halves equals the layer followed by the GELU kernel, bit
    for bit, and the oracle's chain within one bf16 ulp."""
    M, N, K = 600, 8200, 400
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    tiles = ((M + 255) // 256) * ((N + 255) // 256)
    if not (tiles > pairs and 0 < tiles % pairs <= pairs // 2):
        pytest.skip(f"{tiles} tiles on {pairs} SM pairs leave no short last round")
    inp, q_ref, s_ref, y_ref = _case(M, N, K, True, 41)
    args = (dev(q_ref), dev(s_ref), w8.pack_weight(dev(inp.w)), dev(inp.w_scale),
            dev_bf16(inp.bias), N)
    y = w8.scaled_mm(*args)
    g_chain = w8.gelu_tanh(y)
    g_fused = w8.scaled_mm(*args, act=w8.ACT_GELU_TANH)
    torch.cuda.synchronize()
    assert np.array_equal(host_u16(y), y_ref)
    assert torch.equal(g_fused, g_chain)
    assert_bf16_close(host_u16(g_fused), oracle.gelu_tanh(y_ref), max_ulp=1, what="gelu")


def test_act_rejects_unknown_value():
    inp, q_ref, s_ref, _ = _case(64, 128, 256, False, 1)
    with pytest.raises(w8.W8A8Error):
        w8.scaled_mm(dev(q_ref), dev(s_ref), w8.pack_weight(dev(inp.w)), dev(inp.w_scale), None,
                     128, act=2)
