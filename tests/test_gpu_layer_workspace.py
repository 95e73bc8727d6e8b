"""The whole layer (w8a8_linear) on a caller's workspace that starts as
random bytes, is scrambled between calls, is shared by two layers of
different shapes, and sits under CUDA graph replays: every large-M kernel,
ragged last row blocks, a pair tile whose second half lies past M, and
8192 / 8193 rows -- each output bit-exact with the oracle (GELU within one
bf16 ulp).
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_int8_dynamic_b200 as w8
from gpu_util import assert_bf16_close, dev, dev_bf16, host_u16, require_gpu
from w8a8_int8_dynamic_b200.workloads import random_case

pytestmark = pytest.mark.gpu

PATHS = [w8.PATH_AUTO, w8.PATH_LARGE_BN128, w8.PATH_LARGE_BN256, w8.PATH_LARGE_PAIR,
         w8.PATH_LARGE_PAIR128]


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    w8.set_path(w8.PATH_AUTO)
    yield
    w8.set_path(w8.PATH_AUTO)
    assert w8.poll_status() == 0, "a kernel reported a device-side timeout"


def _expect(xi, inp, act):
    y_ref = oracle.linear(xi, inp.w, inp.w_scale, inp.bias)[0]
    return oracle.gelu_tanh(y_ref) if act == w8.ACT_GELU_TANH else y_ref


def _compare(y, y_ref, act, what):
    if act == w8.ACT_GELU_TANH:
        assert_bf16_close(host_u16(y), y_ref, max_ulp=1, what=what)
    else:
        assert np.array_equal(host_u16(y), y_ref), what


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("M,N,K", [(17, 272, 192), (129, 400, 400), (300, 1008, 528),
                                   (513, 2048, 1024), (1000, 2064, 1040)])
def test_layer_garbage_workspace_repeated(M, N, K, path):
    """The workspace starts as random bytes and serves three calls with new
    activations; it is scrambled again between two of them."""
    w8.set_path(path)
    act = w8.ACT_GELU_TANH if M % 2 else w8.ACT_NONE
    inp = random_case(M * 7 + N, M, N, K, bias=True, n_outliers=K // 64, zero_row=True)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias), act=act)
    ws = torch.randint(0, 256, (w8.linear_workspace_bytes(M, N, K),), dtype=torch.uint8,
                       device="cuda")
    for i in range(3):
        xi = random_case(900 + i, M, N, K, bias=False, n_outliers=K // 64, zero_row=True).x
        y = w8.linear(dev_bf16(xi), layer.packed, layer.w_scale, layer.bias, N, act=act,
                      workspace=ws)
        torch.cuda.synchronize()
        _compare(y, _expect(xi, inp, act), act, f"call {i}")
        if i == 0:
            ws.random_(0, 256)


@pytest.mark.parametrize("M", [8192, 8193])
def test_tall_layer_on_random_workspace(M):
    """64 and 65 blocks of 128 rows, on the automatic, pair and 1-SM paths."""
    N, K = 256, 128
    inp = random_case(M, M, N, K, bias=True, n_outliers=2)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias))
    ws = torch.randint(0, 256, (w8.linear_workspace_bytes(M, N, K),), dtype=torch.uint8,
                       device="cuda")
    for path in (w8.PATH_AUTO, w8.PATH_LARGE_PAIR, w8.PATH_LARGE_BN128):
        w8.set_path(path)
        y = w8.linear(dev_bf16(inp.x), layer.packed, layer.w_scale, layer.bias, N, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(host_u16(y), _expect(inp.x, inp, w8.ACT_NONE)), f"path {path}"


@pytest.mark.parametrize("path", [w8.PATH_AUTO, w8.PATH_LARGE_PAIR, w8.PATH_LARGE_BN256])
@pytest.mark.parametrize("M,N,K", [(513, 1024, 1024), (4000, 512, 256)])
def test_layer_graph_replay_from_random_workspace(M, N, K, path):
    """Captured from a workspace of random bytes, then replayed four times
    with new inputs copied into the captured buffers, the workspace
    scrambled again before the third replay."""
    w8.set_path(path)
    inp = random_case(51 + M, M, N, K, bias=True, n_outliers=K // 64)
    packed = w8.pack_weight(dev(inp.w))
    w_s, b = dev(inp.w_scale), dev_bf16(inp.bias)
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.randint(0, 256, (w8.linear_workspace_bytes(M, N, K),), dtype=torch.uint8,
                       device="cuda")
    call = lambda: w8.linear(x, packed, w_s, b, N, out=y, workspace=ws)  # noqa: E731
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        x.copy_(dev_bf16(inp.x))
        call()  # warm the launch path before capture
        stream.synchronize()
        ws.random_(0, 256)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call()
    torch.cuda.synchronize()
    for i in range(4):
        xi = random_case(300 + i, M, N, K, bias=False, n_outliers=K // 64).x
        x.copy_(dev_bf16(xi))
        if i == 2:
            ws.random_(0, 256)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert w8.poll_status() == 0
        assert np.array_equal(host_u16(y), _expect(xi, inp, w8.ACT_NONE)), f"replay {i}"
    del g


def test_layers_back_to_back_share_a_workspace():
    """Two layers of different shapes alternate on one workspace without a
    synchronisation between them (stream order alone separates them)."""
    a = random_case(61, 700, 1024, 512, bias=True, n_outliers=8)
    b = random_case(62, 700, 512, 1024, bias=True, n_outliers=8)
    la = w8.W8A8Linear(dev(a.w), dev(a.w_scale), dev_bf16(a.bias))
    lb = w8.W8A8Linear(dev(b.w), dev(b.w_scale), dev_bf16(b.bias))
    ws = torch.randint(0, 256, (max(w8.linear_workspace_bytes(700, 1024, 512),
                                    w8.linear_workspace_bytes(700, 512, 1024)),),
                       dtype=torch.uint8, device="cuda")
    xa = dev_bf16(a.x)
    ya = [w8.linear(xa, la.packed, la.w_scale, la.bias, 1024, workspace=ws) for _ in range(2)]
    yb = w8.linear(ya[1], lb.packed, lb.w_scale, lb.bias, 512, workspace=ws)
    ya2 = w8.linear(xa, la.packed, la.w_scale, la.bias, 1024, workspace=ws)
    torch.cuda.synchronize()
    ya_ref = _expect(a.x, a, w8.ACT_NONE)
    for y in ya + [ya2]:
        assert np.array_equal(host_u16(y), ya_ref)
    assert np.array_equal(host_u16(yb), oracle.linear(ya_ref, b.w, b.w_scale, b.bias)[0])


def test_layers_from_two_host_threads():
    """Two host threads run layers of different shapes at the same time, each
    on its own stream and workspace (the library's per-context caches and
    launch settings are shared between them)."""
    import threading
    cases = [random_case(71, 600, 2048, 1024, bias=True, n_outliers=16),
             random_case(72, 40, 1024, 4096, bias=True, n_outliers=64),
             random_case(73, 8, 4096, 1024, bias=False, n_outliers=16)]
    results, errors = {}, []

    def worker(i, inp):
        try:
            torch.cuda.set_device(0)
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale),
                                      None if inp.bias is None else dev_bf16(inp.bias))
                x = dev_bf16(inp.x)
                ys = [layer(x) for _ in range(6)]
            s.synchronize()
            results[i] = [host_u16(y) for y in ys]
        except Exception as e:  # reported on the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i, c)) for i, c in enumerate(cases)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    for i, inp in enumerate(cases):
        y_ref = _expect(inp.x, inp, w8.ACT_NONE)
        assert len(results[i]) == 6
        for y in results[i]:
            assert np.array_equal(y, y_ref), f"thread {i}"


@pytest.mark.parametrize("path", [w8.PATH_AUTO, w8.PATH_LARGE_PAIR])
@pytest.mark.parametrize("M", [8192, 8000])
def test_row_tile_order_with_half_tile_round(path, M):
    """M > N: the pair kernel walks its tiles row tile by row tile; 8192 x
    2560 gives 320 tiles of 256 x 256 on the 74 SM pairs, the last 24 run as
    256 x 128 halves.  8000 rows: the last row tile holds 64 rows, so the odd
    CTA of each of its pairs lies wholly past M.  Every output against the
    oracle."""
    w8.set_path(path)
    N, K = 2560, 256
    inp = random_case(81 + M, M, N, K, bias=True, n_outliers=4)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias))
    y = layer(dev_bf16(inp.x))
    torch.cuda.synchronize()
    assert np.array_equal(host_u16(y), _expect(inp.x, inp, w8.ACT_NONE))
