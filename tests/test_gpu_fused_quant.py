"""The next layer's quantisation fused with a layer (w8a8_linear_act_quant):
y and the codes and scales of y must equal, bit for bit, the layer followed
by the quantisation kernel, and the codes must equal the oracle's
quantisation of the GPU's y.  Every large-M kernel (the row maxima folded in
its epilogue, the codes kernel following its row blocks), the small-M path,
zero rows, scales below 1e-30, workspace of random bytes reused over calls,
and CUDA graph replays with new inputs (the completion words reused with
the same tag)."""
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


def _check(inp, N, act, y, q, s, y_layer=None):
    """y bit-equal to the plain layer (and to the oracle, GELU within 1 ulp);
    q and s bit-equal to the oracle's quantisation of the GPU's y."""
    y_h = host_u16(y)
    y_ref = oracle.linear(inp.x, inp.w, inp.w_scale, inp.bias)[0]
    if act == w8.ACT_GELU_TANH:
        assert_bf16_close(y_h, oracle.gelu_tanh(y_ref), max_ulp=1, what="gelu")
    else:
        assert np.array_equal(y_h, y_ref)
    if y_layer is not None:
        assert torch.equal(y, y_layer), "y differs from w8a8_linear_act"
    q_ref, s_ref = oracle.quant_act(y_h)
    assert np.array_equal(q.cpu().numpy(), q_ref), "codes differ from the oracle"
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), "scales differ"


@pytest.mark.parametrize("act", [w8.ACT_NONE, w8.ACT_GELU_TANH])
@pytest.mark.parametrize("path", [w8.PATH_AUTO, w8.PATH_LARGE_BN128, w8.PATH_LARGE_BN256,
                                  w8.PATH_LARGE_PAIR, w8.PATH_LARGE_PAIR128])
@pytest.mark.parametrize("M,N,K", [(129, 400, 400), (300, 1008, 528), (513, 4096, 1024),
                                   (1000, 2064, 1040), (256, 12288, 512)])
def test_act_quant_matches_layer_then_quant(M, N, K, path, act):
    w8.set_path(path)
    inp = random_case(M * 11 + N + K, M, N, K, bias=True, n_outliers=K // 64, zero_row=True)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias), act=act)
    x = dev_bf16(inp.x)
    y_layer = layer(x)
    y, q, s = w8.linear_act_quant(x, layer.packed, layer.w_scale, layer.bias, N, act=act)
    q2, s2 = w8.quant_act(y)
    torch.cuda.synchronize()
    assert torch.equal(q, q2) and torch.equal(s, s2), "differs from w8a8_quant_act of y"
    _check(inp, N, act, y, q, s, y_layer)


@pytest.mark.parametrize("M,N,K", [(1, 272, 400), (4, 2064, 1040), (16, 4096, 4096), (17, 528, 272)])
def test_act_quant_small_m(M, N, K):
    inp = random_case(M + N + K, M, N, K, bias=True, n_outliers=K // 64)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias))
    y, q, s = w8.linear_act_quant(dev_bf16(inp.x), layer.packed, layer.w_scale, layer.bias, N)
    torch.cuda.synchronize()
    _check(inp, N, w8.ACT_NONE, y, q, s)


def test_act_quant_zero_rows_and_tiny_scales():
    """Rows of zeros (no bias) give scale 0 and codes 0; a layer whose
    outputs are all below 1.3e-28 (row scales below 1e-30) takes the IEEE
    quotient for its codes."""
    M, N, K = 640, 1024, 512
    inp = random_case(5, M, N, K, bias=False, zero_row=True)
    inp.x[::7] = 0
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale))
    y, q, s = w8.linear_act_quant(dev_bf16(inp.x), layer.packed, layer.w_scale, None, N)
    torch.cuda.synchronize()
    assert (s.cpu().numpy()[::7] == 0).all() and (q.cpu().numpy()[::7] == 0).all()
    _check(inp, N, w8.ACT_NONE, y, q, s)
    inp.w_scale[:] = (inp.w_scale * np.float32(1e-32)).astype(np.float32)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale))
    y, q, s = w8.linear_act_quant(dev_bf16(inp.x), layer.packed, layer.w_scale, None, N)
    torch.cuda.synchronize()
    sh = s.cpu().numpy()
    assert (sh[sh > 0] < 1e-30).all() and (sh > 0).sum() > M // 2
    _check(inp, N, w8.ACT_NONE, y, q, s)


@pytest.mark.parametrize("path", [w8.PATH_AUTO, w8.PATH_LARGE_BN128])
def test_act_quant_garbage_workspace_repeated(path):
    """The workspace starts as random bytes (stale tags and counts in every
    word) and serves four calls with new activations; it is scrambled again
    between two of them."""
    w8.set_path(path)
    M, N, K = 1000, 2064, 1040
    inp = random_case(21, M, N, K, bias=True, n_outliers=K // 64)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias), act=w8.ACT_GELU_TANH)
    ws = torch.randint(0, 256, (w8.linear_act_quant_workspace_bytes(M, N, K),),
                       dtype=torch.uint8, device="cuda")
    for i in range(4):
        inp_i = random_case(600 + i, M, N, K, bias=True, n_outliers=K // 64)
        inp_i.w, inp_i.w_scale, inp_i.bias = inp.w, inp.w_scale, inp.bias
        x = dev_bf16(inp_i.x)
        y, q, s = w8.linear_act_quant(x, layer.packed, layer.w_scale, layer.bias, N,
                                      workspace=ws, act=w8.ACT_GELU_TANH)
        torch.cuda.synchronize()
        _check(inp_i, N, w8.ACT_GELU_TANH, y, q, s, layer(x))
        if i == 1:
            ws.random_(0, 256)


@pytest.mark.parametrize("M,N,K", [(1000, 2064, 1040), (600, 8208, 400)])
def test_act_quant_cuda_graph_replay_with_new_inputs(M, N, K):
    """A captured call replays with the tag it was captured with: the last
    CTA of each call must leave the completion words cleared.  Three replays
    with new inputs copied into the captured buffers, each bit-exact."""
    inp = random_case(33, M, N, K, bias=True, n_outliers=K // 64)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias))
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((M, N), dtype=torch.int8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    ws = torch.empty((w8.linear_act_quant_workspace_bytes(M, N, K),), dtype=torch.uint8,
                     device="cuda")

    def call():
        w8.linear_act_quant(x, layer.packed, layer.w_scale, layer.bias, N, out=y, q_next=q,
                            a_scale_next=s, workspace=ws)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        x.copy_(dev_bf16(inp.x))
        call()  # warm the launch path before capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call()
    torch.cuda.synchronize()
    for i in range(3):
        inp_i = random_case(700 + i, M, N, K, bias=True, n_outliers=K // 64)
        inp_i.w, inp_i.w_scale, inp_i.bias = inp.w, inp.w_scale, inp.bias
        x.copy_(dev_bf16(inp_i.x))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert w8.poll_status() == 0
        _check(inp_i, N, w8.ACT_NONE, y, q, s)
    del g


def test_act_quant_feeds_next_layer():
    """Two layers: the first with the next layer's quantisation fused in, the
    second a scaled GEMM on those codes; the same bits as two w8a8_linear
    calls."""
    M, H, D = 700, 2048, 1024
    up = random_case(41, M, H, D, bias=True, n_outliers=D // 64)
    dn = random_case(42, M, D, H, bias=True)
    l_up = w8.W8A8Linear(dev(up.w), dev(up.w_scale), dev_bf16(up.bias), act=w8.ACT_GELU_TANH)
    l_dn = w8.W8A8Linear(dev(dn.w), dev(dn.w_scale), dev_bf16(dn.bias))
    x = dev_bf16(up.x)
    g, q, s = w8.linear_act_quant(x, l_up.packed, l_up.w_scale, l_up.bias, H,
                                  act=w8.ACT_GELU_TANH)
    y = w8.scaled_mm(q, s, l_dn.packed, l_dn.w_scale, l_dn.bias, D)
    y_ref = l_dn(l_up(x))
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    y_o = oracle.linear(host_u16(g), dn.w, dn.w_scale, dn.bias)[0]
    assert np.array_equal(host_u16(y), y_o)
