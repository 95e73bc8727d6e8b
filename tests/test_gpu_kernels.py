"""GPU parity of every kernel against the CPU oracle, through the C ABI.

Bar: q, a_scale, the int32 accumulators and the packed bytes bit-exact; the
bf16 output within 1 bf16 ulp (the kernels follow the same fp32 operation
order as the oracle, so in practice it is bit-exact too, and the number of
differing elements is reported).  Shapes span several tiles plus ragged M / N
/ K tails, the zero-row case and decode sizes.
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_int8_dynamic_b200 as w8
from gpu_util import assert_bf16_close, dev, dev_bf16, host_u16, require_gpu
from w8a8_int8_dynamic_b200.workloads import f32_to_bf16_bits, random_case

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    w8.set_path(w8.PATH_AUTO)
    yield
    w8.set_path(w8.PATH_AUTO)
    assert w8.poll_status() == 0, "a kernel reported a device-side timeout"


# ---------------------------------------------------------------- quantisation
# Every kernel instance: 1-4 chunks a lane, 8 (rows x warps beyond two waves
# of resident warps: 1500 x 12288), 16 (rows of more than 16 warps at 8), and
# the two-pass kernel (rows beyond 65536).
QUANT_SHAPES = [(1, 16), (3, 48), (64, 256), (127, 4096), (129, 3072), (512, 4096),
                (7, 12288), (16, 5120), (5, 40000), (2, 131072), (33, 32784), (1500, 12288)]


@pytest.mark.parametrize("M,K", QUANT_SHAPES)
def test_quant_matches_oracle(M, K):
    rng = np.random.default_rng(M * 7 + K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.permutation(K)[:max(1, K // 100)]] *= 10.0
    if M > 2:
        x[1] = 0.0                 # zero row
        x[2] *= 1e-38              # subnormal-scale row (IEEE-quotient path)
    xb = f32_to_bf16_bits(x)
    q_ref, s_ref = oracle.quant_act(xb)
    q, s = w8.quant_act(dev_bf16(xb))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("K,reps", [(256, 1), (12288, 28), (40000, 1)])
def test_quant_near_ties_and_ties(K, reps):
    """Values whose quotient is exactly a half-integer, or a few fp32 ulps
    from one: the kernel's reciprocal fast path must round them exactly as
    the oracle's plain division does.  Rows of K elements (the pattern
    repeated), `reps` copies of the row set: short rows, the 8-chunk instance
    (54 x 28 rows of 12288) and the 16-chunk one."""
    rows = []
    for e in range(-20, 20, 3):
        s = 2.0 ** e
        amax = 127.0 * s
        k = np.arange(-126, 127, dtype=np.float64)
        ties = (k + 0.5) * s
        row = np.concatenate([[amax], ties]).astype(np.float32)
        rows.append(row[:256])
    rng = np.random.default_rng(11)
    for _ in range(40):
        amax = np.float32(rng.uniform(0.1, 500.0))
        s = np.float32(amax / np.float32(127.0))
        k = rng.integers(-126, 126, 255).astype(np.float32) + np.float32(0.5)
        near = (k * s).astype(np.float32)
        near = near + rng.integers(-3, 4, 255).astype(np.float32) * np.spacing(near)
        rows.append(np.concatenate([[amax], near]).astype(np.float32)[:256])
    x = np.tile(np.stack([np.resize(r, K) for r in rows]), (reps, 1))
    xb = f32_to_bf16_bits(x)
    q_ref, s_ref = oracle.quant_act(xb)
    q, s = w8.quant_act(dev_bf16(xb))
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quant_row_stride_and_no_overrun():
    M, K, ldx = 37, 272, 400
    rng = np.random.default_rng(5)
    big = f32_to_bf16_bits(rng.standard_normal((M, ldx)).astype(np.float32))
    big[:, K:] = f32_to_bf16_bits(np.array([3e4], np.float32))[0]
    xd = dev_bf16(big)[:, :K]
    guard = 64
    qbuf = torch.full((M * K + guard,), 0x5A, dtype=torch.int8, device="cuda")
    sbuf = torch.full((M + guard,), 7.0, dtype=torch.float32, device="cuda")
    w8.quant_act(xd, q=qbuf[:M * K].view(M, K), a_scale=sbuf[:M])
    q_ref, s_ref = oracle.quant_act(np.ascontiguousarray(big[:, :K]))
    assert np.array_equal(qbuf[:M * K].view(M, K).cpu().numpy(), q_ref)
    assert np.array_equal(sbuf[:M].cpu().numpy(), s_ref)
    assert (qbuf[M * K:].cpu().numpy() == 0x5A).all()
    assert (sbuf[M:].cpu().numpy() == 7.0).all()


# ---------------------------------------------------------------- weight repack
@pytest.mark.parametrize("N,K", [(8, 16), (128, 128), (304, 208), (256, 4096), (1000, 528), (12288, 256)])
def test_pack_matches_oracle_and_round_trips(N, K):
    rng = np.random.default_rng(N + K)
    w = rng.integers(-128, 128, (N, K), dtype=np.int8)
    wd = dev(w)
    packed = w8.pack_weight(wd)
    ref = oracle.pack_weight(w)
    assert packed.numel() == ref.size
    assert np.array_equal(packed.cpu().numpy().view(np.int8), ref)
    back = w8.unpack_weight(packed, N, K)
    assert torch.equal(back, wd)


def test_pack_overwrites_stale_buffer():
    N, K = 200, 144
    w = np.random.default_rng(0).integers(-127, 128, (N, K), dtype=np.int8)
    nbytes = w8.packed_weight_bytes(N, K)
    buf = torch.full((nbytes + 32,), 0x77, dtype=torch.uint8, device="cuda")
    from w8a8_int8_dynamic_b200.binding import _check, _ptr, _stream, lib
    _check(lib().w8a8_pack_weight(_ptr(dev(w)), N, K, _ptr(buf), nbytes, _stream()), "pack")
    assert np.array_equal(buf[:nbytes].cpu().numpy().view(np.int8), oracle.pack_weight(w))
    assert (buf[nbytes:].cpu().numpy() == 0x77).all()


# ---------------------------------------------------------------- GEMM
GEMM_SHAPES = [(1, 8, 16), (64, 128, 256), (127, 264, 272), (129, 392, 400), (256, 512, 1024),
               (300, 1000, 528), (513, 264, 4096), (1000, 2056, 144)]


@pytest.mark.parametrize("path", [w8.PATH_LARGE_BN128, w8.PATH_LARGE_BN256])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_i32_exact(M, N, K, path):
    w8.set_path(path)
    rng = np.random.default_rng(M * 31 + N * 7 + K)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    w = rng.integers(-128, 128, (N, K), dtype=np.int8)
    acc = w8.scaled_mm_i32(dev(q), w8.pack_weight(dev(w)), N)
    ref = oracle.gemm_i32(q, w)
    assert np.array_equal(acc.cpu().numpy(), ref)


def test_gemm_i32_extreme_values():
    M, N, K = 130, 136, 131072 // 8
    q = np.full((M, K), 127, np.int8)
    q[1::2] = -127
    w = np.full((N, K), -128, np.int8)
    acc = w8.scaled_mm_i32(dev(q), w8.pack_weight(dev(w)), N)
    assert np.array_equal(acc.cpu().numpy(), oracle.gemm_i32(q, w))


@pytest.mark.parametrize("bias", [False, True])
@pytest.mark.parametrize("path", [w8.PATH_LARGE_BN128, w8.PATH_LARGE_BN256, w8.PATH_LARGE_PAIR,
                                  w8.PATH_LARGE_PAIR128])
@pytest.mark.parametrize("M,N,K", [(64, 128, 256), (129, 392, 400), (300, 1000, 528), (512, 1024, 4096),
                                   (257, 264, 272), (700, 520, 144), (1000, 2056, 1040)])
def test_scaled_mm_matches_oracle(M, N, K, path, bias):
    w8.set_path(path)
    inp = random_case(M + N + K, M, N, K, bias=bias, n_outliers=K // 64, zero_row=True)
    q_ref, s_ref = oracle.quant_act(inp.x)
    acc_ref = oracle.gemm_i32(q_ref, inp.w)
    y_ref = oracle.epilogue(acc_ref, s_ref, inp.w_scale, inp.bias)
    b = None if inp.bias is None else dev_bf16(inp.bias)
    y = w8.scaled_mm(dev(q_ref), dev(s_ref), w8.pack_weight(dev(inp.w)), dev(inp.w_scale), b, N)
    y_h = host_u16(y)
    assert_bf16_close(y_h, y_ref)
    assert np.array_equal(y_h, y_ref), "expected bit-exact bf16"


@pytest.mark.parametrize("M,N,K", [(1, 27648, 5120), (4, 2056, 1040), (16, 4096, 12288)])
def test_decode_with_garbage_workspace_repeated(M, N, K):
    """The small-M kernel counts the CTAs that share a weight slab on
    call-tagged workspace words.  Here the workspace starts as random bytes
    (stale tags, counts in every state) and serves four calls with new
    activations; each call must match the oracle bit for bit."""
    w8.set_path(w8.PATH_SMALL)
    inp = random_case(M * 7 + N + K, M, N, K, bias=True, n_outliers=K // 64)
    packed = w8.pack_weight(dev(inp.w))
    need = w8.scaled_mm_workspace_bytes(M, N, K)
    assert need > 0
    ws = torch.randint(0, 256, (need,), dtype=torch.uint8, device="cuda")
    for i in range(4):
        xi = random_case(500 + i, M, N, K, bias=False, n_outliers=K // 64).x
        q_ref, s_ref = oracle.quant_act(xi)
        y_ref = oracle.epilogue(oracle.gemm_i32(q_ref, inp.w), s_ref, inp.w_scale, inp.bias)
        y = w8.scaled_mm(dev(q_ref), dev(s_ref), packed, dev(inp.w_scale), dev_bf16(inp.bias), N,
                         workspace=ws)
        assert np.array_equal(host_u16(y), y_ref), f"call {i}"
        # and a fresh scramble of the words between calls
        if i == 1:
            ws.random_(0, 256)


@pytest.mark.parametrize("path", [w8.PATH_LARGE_BN128, w8.PATH_LARGE_PAIR, w8.PATH_LARGE_PAIR128])
def test_scaled_mm_does_not_write_outside_y(path):
    w8.set_path(path)
    M, N, K = 130, 264, 272
    _guarded_scaled_mm(M, N, K)


def _guarded_scaled_mm(M, N, K):
    inp = random_case(9, M, N, K, bias=True)
    q_ref, s_ref = oracle.quant_act(inp.x)
    guard = 4096
    ybuf = torch.full((M * N + guard,), -1, dtype=torch.int16, device="cuda")
    y = ybuf[:M * N].view(torch.bfloat16).view(M, N)
    w8.scaled_mm(dev(q_ref), dev(s_ref), w8.pack_weight(dev(inp.w)), dev(inp.w_scale),
                 dev_bf16(inp.bias), N, out=y)
    y_ref = oracle.epilogue(oracle.gemm_i32(q_ref, inp.w), s_ref, inp.w_scale, inp.bias)
    assert np.array_equal(host_u16(y), y_ref)
    assert (ybuf[M * N:].cpu().numpy() == -1).all()


@pytest.mark.parametrize("M,N,K", [(300, 20480, 528), (600, 8200, 400)])
def test_pair_tail_split_matches_oracle(M, N, K):
    """Shapes whose 256 x 256 pair tiles fill the SM pairs once and leave a
    short last round (160 tiles: 12 left over; 99 tiles: 25 left over, the
    last one ragged in N and M): those tiles run as two 256 x 128 halves.
    Bit-exact against the oracle, automatic and forced pair path, nothing
    written past y."""
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    tiles = ((M + 255) // 256) * ((N + 255) // 256)
    if not (tiles > pairs and 0 < tiles % pairs <= pairs // 2):
        pytest.skip(f"{tiles} tiles on {pairs} SM pairs leave no short last round")
    for path in (w8.PATH_AUTO, w8.PATH_LARGE_PAIR):
        w8.set_path(path)
        assert "256x256" in w8.gemm_kernel_name(M, N, K)
        _guarded_scaled_mm(M, N, K)


# ---------------------------------------------------------------- decode path
@pytest.mark.parametrize("M", [1, 2, 4, 9, 16])
@pytest.mark.parametrize("N,K", [(8, 16), (264, 400), (4096, 4096), (2048, 12288)])
def test_decode_path_matches_oracle(M, N, K):
    inp = random_case(M * 3 + N + K, M, N, K, bias=(N % 16 == 0), n_outliers=K // 128)
    q_ref, s_ref = oracle.quant_act(inp.x)
    y_ref = oracle.epilogue(oracle.gemm_i32(q_ref, inp.w), s_ref, inp.w_scale, inp.bias)
    packed = w8.pack_weight(dev(inp.w))
    ws = torch.empty((w8.scaled_mm_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    b = None if inp.bias is None else dev_bf16(inp.bias)
    w8.set_path(w8.PATH_SMALL)
    for _ in range(2):  # second call reuses the workspace (counters left clean)
        y = w8.scaled_mm(dev(q_ref), dev(s_ref), packed, dev(inp.w_scale), b, N, workspace=ws)
        assert np.array_equal(host_u16(y), y_ref)
    w8.set_path(w8.PATH_LARGE)
    y2 = w8.scaled_mm(dev(q_ref), dev(s_ref), packed, dev(inp.w_scale), b, N)
    assert np.array_equal(host_u16(y2), y_ref)


# ---------------------------------------------------------------- fused layer
@pytest.mark.parametrize("path", [w8.PATH_AUTO, w8.PATH_LARGE_PAIR, w8.PATH_LARGE_PAIR128])
@pytest.mark.parametrize("M,N,K", [(1, 264, 400), (16, 1024, 1024), (17, 1024, 1024),
                                   (64, 128, 256), (300, 1000, 528), (512, 4096, 4096)])
def test_linear_matches_oracle(M, N, K, path):
    w8.set_path(path)
    inp = random_case(M * 5 + N + K, M, N, K, bias=True, n_outliers=K // 100, zero_row=True)
    y_ref, q_ref, s_ref, _ = oracle.linear(inp.x, inp.w, inp.w_scale, inp.bias)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale), dev_bf16(inp.bias))
    y = layer(dev_bf16(inp.x))
    assert np.array_equal(host_u16(y), y_ref)
    y = layer(dev_bf16(inp.x))  # workspace reuse
    assert np.array_equal(host_u16(y), y_ref)


def test_linear_nd_input_keeps_rank():
    M0, M1, N, K = 3, 50, 264, 272
    inp = random_case(4, M0 * M1, N, K, bias=False)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale))
    x3 = dev_bf16(inp.x).view(M0, M1, K)
    y3 = layer(x3)
    assert tuple(y3.shape) == (M0, M1, N)
    y_ref, *_ = oracle.linear(inp.x, inp.w, inp.w_scale, None)
    assert np.array_equal(host_u16(y3.reshape(-1, N)), y_ref)


def test_fused_qkv_split_equals_separate_layers():
    M, H, K = 200, 512, 640
    rng = np.random.default_rng(8)
    x = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    blocks = [rng.integers(-127, 128, (H, K), dtype=np.int8) for _ in range(3)]
    scales = [rng.uniform(lo, 4 * lo, H).astype(np.float32) for lo in (5e-4, 1e-3, 2e-3)]
    fused = w8.W8A8Linear.from_blocks([dev(b) for b in blocks], [dev(s) for s in scales])
    yq, yk, yv = fused.split(fused(dev_bf16(x)))
    for i, part in enumerate((yq, yk, yv)):
        sep = w8.W8A8Linear(dev(blocks[i]), dev(scales[i]))(dev_bf16(x))
        assert torch.equal(part.contiguous(), sep)


# ---------------------------------------------------------------- GELU harness
def test_gelu_within_one_ulp():
    rng = np.random.default_rng(2)
    x = f32_to_bf16_bits((rng.standard_normal(100003) * 3).astype(np.float32))
    y = w8.gelu_tanh(dev_bf16(x))
    assert_bf16_close(host_u16(y), oracle.gelu_tanh(x), max_ulp=1, what="gelu")


# ---------------------------------------------------------------- CUDA graph replay
@pytest.mark.parametrize("case", ["layer", "decode_layer", "tail_split"])
def test_cuda_graph_replay_with_new_inputs(case):
    """Kernels that count CTAs on call-tagged workspace words (the small-M
    kernel's slab reduction) see the same tag on every replay of a captured
    CUDA graph.  They must leave those words cleared: capture one call, then
    replay it three times with new inputs copied into the captured buffers,
    each replay checked against the oracle bit for bit (the large-M layer,
    quantisation + GEMM, alongside)."""
    M, N, K = {"layer": (512, 1024, 1024), "decode_layer": (4, 2056, 1040),
               "tail_split": (600, 8200, 400)}[case]
    inp = random_case(7, M, N, K, bias=True, n_outliers=K // 64)
    packed = w8.pack_weight(dev(inp.w))
    ws_s, b = dev(inp.w_scale), dev_bf16(inp.bias)
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    a = torch.empty((M,), dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((w8.linear_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    call = lambda: w8.linear(x, packed, ws_s, b, N, out=y, workspace=ws)  # noqa: E731
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        call()  # warm the launch path before capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call()
    torch.cuda.synchronize()
    for i in range(3):
        xi = random_case(100 + i, M, N, K, bias=False, n_outliers=K // 64).x
        y_ref, q_ref, s_ref, _ = oracle.linear(xi, inp.w, inp.w_scale, inp.bias)
        x.copy_(dev_bf16(xi))
        q.copy_(dev(q_ref))
        a.copy_(dev(s_ref))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert w8.poll_status() == 0
        assert np.array_equal(host_u16(y), y_ref), f"replay {i}"
    del g


# ---------------------------------------------------------------- int8 MMA rate
def test_int8_mma_rate_selftest():
    """The memory-free tcgen05.mma.kind::i8 loop: a rate between the bf16
    burst figure and twice the dense int8 spec (4.5 POPS), and no device-side
    timeout."""
    tops = w8.selftest_int8_mma_rate(4000)
    assert 1500.0 < tops < 9000.0, tops
    assert w8.poll_status() == 0


# ---------------------------------------------------------------- bounded waits
def test_timeout_is_reported_and_context_survives():
    w8.selftest_wait_timeout(2_000_000)  # 2 ms
    assert w8.poll_status() == 5         # W8A8_ERR_TIMEOUT
    assert w8.poll_status() == 0         # cleared
    inp = random_case(1, 64, 128, 256, bias=False)
    y_ref, *_ = oracle.linear(inp.x, inp.w, inp.w_scale, None)
    y = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale))(dev_bf16(inp.x))
    assert np.array_equal(host_u16(y), y_ref)


def test_launch_counter_counts_kernels():
    before = w8.launch_count()
    inp = random_case(1, 64, 128, 256, bias=False)
    layer = w8.W8A8Linear(dev(inp.w), dev(inp.w_scale))
    mid = w8.launch_count()
    layer(dev_bf16(inp.x))
    torch.cuda.synchronize()
    assert mid - before == 1             # pack
    assert w8.launch_count() - mid == 2  # quant + GEMM
