"""GPU parity of the load-time weight paths and the static activation scale.

* online quantisation ("Online Quantization", Overview; "Issue 5 probe: int8
  quantized DiT serve paths on the RTX 3090", Round one): bf16 W -> per-channel
  scales + packed tile image in one kernel, bit-exact against the oracle's
  per-channel quantisation followed by the oracle's repack;
* compressed-tensors int32 storage ("Issue 5 probe ...", Artifact): packed
  bytes bit-exact against the oracle's unpack followed by its repack;
* static activation scale ("Online Quantization", Parameters): codes and
  scales bit-exact, including saturation, ties and unusable scales.
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_int8_dynamic_b200 as w8
from gpu_util import assert_bf16_close, dev, dev_bf16, host_u16, require_gpu
from w8a8_int8_dynamic_b200.workloads import f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    w8.set_path(w8.PATH_AUTO)
    yield
    w8.set_path(w8.PATH_AUTO)
    assert w8.poll_status() == 0, "a kernel reported a device-side timeout"


def _weights(seed, N, K):
    """Gaussian rows with per-channel magnitudes spanning many decades, plus
    the special rows: all zero, subnormal-scale, huge, and exact ties."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K)).astype(np.float32)
    w *= (10.0 ** rng.uniform(-4, 2, size=N)).astype(np.float32)[:, None]
    if N >= 8:
        w[1] = 0.0
        w[2] *= np.float32(1e-38)          # scale < 1e-30 -> IEEE quotient path
        w[3] *= np.float32(1e30)
        s = 2.0 ** -7                       # row 4: exact half-integer quotients
        k = np.resize(np.arange(-126, 127, dtype=np.float64), K)
        row = (k + 0.5) * s
        row[0] = 127.0 * s
        w[4] = row.astype(np.float32)
    return f32_to_bf16_bits(w)


WEIGHT_SHAPES = [(8, 16), (256, 128), (264, 144), (1000, 4096), (3072, 1040), (136, 12304)]


@pytest.mark.parametrize("N,K", WEIGHT_SHAPES)
def test_quant_pack_weight_matches_oracle(N, K):
    wb = _weights(N * 31 + K, N, K)
    q_ref, s_ref = oracle.quant_weight(wb)
    packed_ref = oracle.pack_weight(q_ref)
    packed, s = w8.quant_pack_weight(dev_bf16(wb))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    got = packed.cpu().numpy()
    assert got.shape == packed_ref.shape
    assert np.array_equal(got, packed_ref.view(np.uint8))
    # the unpack of the image is the oracle's codes
    assert np.array_equal(w8.unpack_weight(packed, N, K).cpu().numpy(), q_ref)


def test_quant_pack_weight_full_size_mlp_up():
    """The DiT MLP up-projection weight, 12288 x 3072, quantised at load."""
    N, K = 12288, 3072
    wb = _weights(7, N, K)
    q_ref, s_ref = oracle.quant_weight(wb)
    packed, s = w8.quant_pack_weight(dev_bf16(wb))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(w8.unpack_weight(packed, N, K).cpu().numpy(), q_ref)


def test_from_float_layer_matches_oracle_linear():
    """Load-time quantisation feeding the whole layer: y is the oracle's
    linear with the oracle's per-channel weight codes and scales."""
    rng = np.random.default_rng(5)
    M, N, K = 200, 776, 1296
    wb = f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    xb = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    bias = f32_to_bf16_bits((rng.standard_normal(N) * 0.02).astype(np.float32))
    q_w, s_w = oracle.quant_weight(wb)
    y_ref, *_ = oracle.linear(xb, q_w, s_w, bias)
    layer = w8.W8A8Linear.from_float(dev_bf16(wb), dev_bf16(bias))
    y = layer(dev_bf16(xb))
    torch.cuda.synchronize()
    assert_bf16_close(host_u16(y), y_ref, max_ulp=1)


# ---------------------------------------------------------------- int32 storage
@pytest.mark.parametrize("N,K", [(8, 16), (256, 128), (264, 144), (1000, 4096), (520, 12304)])
def test_pack_weight_int32_matches_oracle(N, K):
    rng = np.random.default_rng(N + 3 * K)
    words = rng.integers(-2 ** 31, 2 ** 31, size=(N, K // 4), dtype=np.int64).astype(np.int32)
    words[0, :4] = [0, -1, 0x7F7F7F7F, -0x7F7F7F80]   # bytes 0, 255, 127, 128 (w = -128, 127, -1, 0)
    w_ref = oracle.unpack_int32(words, K)
    packed = w8.pack_weight_int32(dev(words), K)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), oracle.pack_weight(w_ref).view(np.uint8))


# ---------------------------------------------------------------- static activation scale
STATIC_SCALES = [1e-3, 0.0123, 0.05, 1.0, 0.0, -1.0, float("nan"), 1e-35, 1e35, 2.0 ** -7]


@pytest.mark.parametrize("scale", STATIC_SCALES)
@pytest.mark.parametrize("M,K", [(1, 16), (37, 1040), (512, 4096)])
def test_quant_act_static_matches_oracle(M, K, scale):
    rng = np.random.default_rng(M + K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.permutation(K)[:max(1, K // 50)]] *= 40.0       # saturating outliers
    if M > 2:
        x[1] = 0.0
        x[2] = (np.resize(np.arange(-140, 141), K) + 0.5) * 2.0 ** -7   # ties at scale 2^-7
    xb = f32_to_bf16_bits(x)
    q_ref, s_ref = oracle.quant_act_static(xb, scale)
    sc = torch.tensor([scale], dtype=torch.float32, device="cuda")
    q, s = w8.quant_act_static(dev_bf16(xb), sc)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quant_act_static_strided_rows_and_gemm_chain():
    """Rows with a stride larger than K, then the scaled GEMM on the codes:
    the static scale flows through a_scale unchanged."""
    rng = np.random.default_rng(11)
    M, N, K, ldx = 300, 512, 2048, 2048 + 64
    xfull = f32_to_bf16_bits(rng.standard_normal((M, ldx)).astype(np.float32))
    xb = np.ascontiguousarray(xfull[:, :K])
    scale = 0.031
    w = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    w_scale = rng.uniform(5e-4, 5e-3, size=N).astype(np.float32)
    q_ref, s_ref = oracle.quant_act_static(xb, scale)
    acc = oracle.gemm_i32(q_ref, w)
    y_ref = oracle.epilogue(acc, s_ref, w_scale, None)
    xd = dev_bf16(xfull)[:, :K]
    q, s = w8.quant_act_static(xd, torch.tensor([scale], dtype=torch.float32, device="cuda"))
    y = w8.scaled_mm(q, s, w8.pack_weight(dev(w)), dev(w_scale), None, N)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert_bf16_close(host_u16(y), y_ref, max_ulp=1)


def test_new_entries_reject_bad_arguments():
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")    # K % 16 != 0
    sc = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(w8.W8A8Error):
        w8.quant_act_static(x, sc)
    with pytest.raises(w8.W8A8Error):
        w8.quant_pack_weight(torch.zeros((12, 32), dtype=torch.bfloat16, device="cuda"))  # N % 8
    with pytest.raises(w8.W8A8Error):
        w8.pack_weight_int32(torch.zeros((8, 6), dtype=torch.int32, device="cuda"), 24)  # K % 16
