"""Full-size parity on the five workloads, in the launch configuration the
benchmark times (w8a8_linear: quantisation + GEMM, weights packed once).

Every workload is compared in full, element by element: codes, scales,
bf16 outputs, and for the DiT MLP pair also the int32 accumulators (the
oracle forms a 309 GOP layer in a few seconds on the host cores).
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_int8_dynamic_b200 as w8
from gpu_util import assert_bf16_close, dev, dev_bf16, host_u16, require_gpu
from w8a8_int8_dynamic_b200.workloads import WORKLOADS, bf16_bits_to_f32, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    w8.set_path(w8.PATH_AUTO)
    yield
    assert w8.poll_status() == 0


def _run_layer(inp):
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale),
                          None if inp.bias is None else dev_bf16(inp.bias))
    x = dev_bf16(inp.x)
    y = layer(x)
    q, s = w8.quant_act(x)
    torch.cuda.synchronize()
    return layer, x, y, q, s


@pytest.mark.parametrize("name", ["small_64x128x256", "square_512x4096x4096",
                                  "fused_qkv_512x12288x4096", "decode_m1_27648x5120",
                                  "decode_m4_27648x5120", "decode_m16_27648x5120"])
def test_workload_full_parity(name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    _, _, y, q, s = _run_layer(inp)
    y_ref, q_ref, s_ref, _ = oracle.linear(inp.x, inp.w, inp.w_scale, inp.bias)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    y_h = host_u16(y)
    assert_bf16_close(y_h, y_ref)
    assert np.array_equal(y_h, y_ref)
    if wl.zero_row:
        yrow = bf16_bits_to_f32(y_h[-1])
        bias = bf16_bits_to_f32(inp.bias) if inp.bias is not None else 0.0
        assert np.array_equal(yrow, np.asarray(bias, np.float32) + np.zeros_like(yrow))


def test_workload_decode_paths_agree():
    """The weight-streaming kernel and the large-M kernel give the same bits."""
    inp = make_inputs(WORKLOADS["decode_m16_27648x5120"])
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale))
    x = dev_bf16(inp.x)
    w8.set_path(w8.PATH_SMALL)
    y_small = layer(x).clone()
    w8.set_path(w8.PATH_LARGE)
    y_large = layer(x).clone()
    w8.set_path(w8.PATH_AUTO)
    assert torch.equal(y_small, y_large)


def test_dit_mlp_chain_full():
    """The DiT MLP block at full size, every element against the oracle: the
    4096 x 12288 x 3072 up-projection (codes, scales, int32 accumulators and
    bf16 outputs), the same layer with the GELU in its epilogue (within one
    bf16 ulp of the oracle's GELU of the oracle's output, and bit-identical
    to the layer followed by the GELU kernel), and the row-parallel
    4096 x 3072 x 12288 down-projection fed the GPU's own GELU output on both
    sides.  Layers run as the benchmark runs them (w8a8_linear /
    w8a8_linear_act, automatic kernel choice)."""
    up = make_inputs(WORKLOADS["dit_mlp_up_4096x12288x3072"])
    down = make_inputs(WORKLOADS["dit_mlp_down_4096x3072x12288"])
    l_up = w8.W8A8Linear(dev(up.w), dev(up.w_scale), dev_bf16(up.bias))
    l_up_gelu = w8.W8A8Linear(dev(up.w), dev(up.w_scale), dev_bf16(up.bias), act=w8.ACT_GELU_TANH)
    l_down = w8.W8A8Linear(dev(down.w), dev(down.w_scale), dev_bf16(down.bias))
    x = dev_bf16(up.x)
    h = l_up(x)
    g_fused = l_up_gelu(x)
    g = w8.gelu_tanh(h)
    y = l_down(g_fused)
    qg, sg = w8.quant_act(x)
    acc_g = w8.scaled_mm_i32(qg, l_up.packed, 12288)
    torch.cuda.synchronize()

    # up-projection: everything, element by element
    h_ref, q_ref, s_ref, acc_ref = oracle.linear(up.x, up.w, up.w_scale, up.bias)
    assert np.array_equal(qg.cpu().numpy(), q_ref)
    assert np.array_equal(sg.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(acc_g.cpu().numpy(), acc_ref)
    del acc_g, acc_ref
    h_h = host_u16(h)
    assert_bf16_close(h_h, h_ref)
    assert np.array_equal(h_h, h_ref), "up-projection: expected bit-exact bf16"

    # GELU in the epilogue: the chain's bits, and within 1 ulp of the oracle
    assert torch.equal(g_fused, g), "GELU epilogue differs from layer + GELU kernel"
    g_h = host_u16(g_fused)
    assert_bf16_close(g_h, oracle.gelu_tanh(h_ref), max_ulp=1, what="gelu epilogue")

    # row-parallel down-projection on the GPU's GELU output
    qd, sd = w8.quant_act(g_fused)
    acc_d = w8.scaled_mm_i32(qd, l_down.packed, 3072)
    torch.cuda.synchronize()
    y_ref, q_dn, s_dn, acc_dn = oracle.linear(g_h, down.w, down.w_scale, down.bias)
    assert np.array_equal(qd.cpu().numpy(), q_dn)
    assert np.array_equal(sd.cpu().numpy().view(np.uint32), s_dn.view(np.uint32))
    assert np.array_equal(acc_d.cpu().numpy(), acc_dn)
    y_h = host_u16(y)
    assert_bf16_close(y_h, y_ref)
    assert np.array_equal(y_h, y_ref), "down-projection: expected bit-exact bf16"


@pytest.mark.parametrize("name", ["small_64x128x256", "square_512x4096x4096",
                                  "fused_qkv_512x12288x4096"])
def test_rel_l2_reproduces_page_figure(name):
    """0.17% rel-L2 against the fp32 product of the dequantised operands
    ("Issue 5 probe", Round two, kernel-path verification)."""
    inp = make_inputs(WORKLOADS[name])
    _, _, y, q, s = _run_layer(inp)
    rows = slice(None) if inp.x.shape[0] <= 64 else slice(0, 64)
    yf = bf16_bits_to_f32(host_u16(y)[rows]).astype(np.float64)
    qh = q.cpu().numpy()[rows].astype(np.float64) * s.cpu().numpy()[rows, None].astype(np.float64)
    wdq = inp.w.astype(np.float64) * inp.w_scale[:, None].astype(np.float64)
    bias = 0.0 if inp.bias is None else bf16_bits_to_f32(inp.bias).astype(np.float64)
    ref = qh @ wdq.T + bias
    err = np.linalg.norm(yf - ref) / np.linalg.norm(ref)
    assert 0.0010 <= err <= 0.0025, err


def test_dit_mlp_block_fused_quant_full():
    """The benchmark's step at full size: the up-projection with GELU in its
    epilogue and the down-projection's quantisation fused in
    (w8a8_linear_act_quant), then the down-projection as a scaled GEMM on
    those codes.  The same bits as the two layers run one after the other,
    with the codes and scales equal to the oracle's quantisation of the GPU's
    GELU output, in full."""
    up = make_inputs(WORKLOADS["dit_mlp_up_4096x12288x3072"])
    down = make_inputs(WORKLOADS["dit_mlp_down_4096x3072x12288"])
    l_up = w8.W8A8Linear(dev(up.w), dev(up.w_scale), dev_bf16(up.bias), act=w8.ACT_GELU_TANH)
    l_down = w8.W8A8Linear(dev(down.w), dev(down.w_scale), dev_bf16(down.bias))
    x = dev_bf16(up.x)
    g, q, s = w8.linear_act_quant(x, l_up.packed, l_up.w_scale, l_up.bias, 12288,
                                  act=w8.ACT_GELU_TANH)
    y = w8.scaled_mm(q, s, l_down.packed, l_down.w_scale, l_down.bias, 3072)
    g_ref = l_up(x)
    y_ref = l_down(g_ref)
    torch.cuda.synchronize()
    assert torch.equal(g, g_ref)
    assert torch.equal(y, y_ref)
    q_o, s_o = oracle.quant_act(host_u16(g))
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))
