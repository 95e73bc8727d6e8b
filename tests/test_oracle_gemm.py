"""Pins for the oracle's int8 x int8 -> int32 product.

Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
Round two (the int8 scaled matmul); "INT8 Quant for Dual-Max Recipe" (int8 x
int8 on the integer tensor cores, no weight dequantisation).  The product is
an exact integer sum, so it is pinned by brute force with Python integers,
closed forms and an int64 library matmul.
"""
import numpy as np
import pytest

import oracle


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 7), (8, 8, 8), (2, 7, 3)])
def test_brute_force_python_ints(shape):
    M, N, K = shape
    rng = np.random.default_rng(sum(shape))
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    w = rng.integers(-128, 128, (N, K), dtype=np.int8)  # -128 included on purpose
    acc = oracle.gemm_i32(q, w)
    for m in range(M):
        for n in range(N):
            exp = sum(int(q[m, k]) * int(w[n, k]) for k in range(K))
            assert int(acc[m, n]) == exp


def test_identity_weight_returns_codes():
    rng = np.random.default_rng(1)
    q = rng.integers(-127, 128, (9, 32), dtype=np.int8)
    w = np.eye(32, dtype=np.int8)
    assert (oracle.gemm_i32(q, w) == q.astype(np.int32)).all()


def test_all_ones_weight_gives_row_sums():
    rng = np.random.default_rng(2)
    q = rng.integers(-127, 128, (6, 200), dtype=np.int8)
    w = np.ones((3, 200), np.int8)
    acc = oracle.gemm_i32(q, w)
    assert (acc == q.astype(np.int64).sum(axis=1, keepdims=True)).all()


def test_transposed_operand_is_detected():
    # acc[m, n] must pair row m of q with row n of w (both K-contiguous);
    # a product with w laid out [K, N] would differ on a non-square case
    q = np.arange(6, dtype=np.int8).reshape(2, 3)
    w = np.array([[1, 0, 0], [0, 0, 1]], np.int8)
    assert oracle.gemm_i32(q, w).tolist() == [[0, 2], [3, 5]]


def test_matches_int64_matmul():
    rng = np.random.default_rng(3)
    q = rng.integers(-127, 128, (64, 1024), dtype=np.int8)
    w = rng.integers(-127, 128, (96, 1024), dtype=np.int8)
    ref = q.astype(np.int64) @ w.astype(np.int64).T
    assert (oracle.gemm_i32(q, w).astype(np.int64) == ref).all()


def test_extreme_sum_fits_int32():
    # 131072 * 127 * 128 = 2,130,706,432 < 2^31: the largest K the library accepts
    K = 131072
    q = np.full((1, K), 127, np.int8)
    w = np.full((1, K), -128, np.int8)
    assert int(oracle.gemm_i32(q, w)[0, 0]) == -127 * 128 * K


def test_overflow_is_reported():
    K = 140000
    q = np.full((1, K), -127, np.int8)
    w = np.full((1, K), -128, np.int8)
    with pytest.raises(OverflowError):
        oracle.gemm_i32(q, w)


def test_sampled_matches_full():
    rng = np.random.default_rng(5)
    q = rng.integers(-127, 128, (16, 256), dtype=np.int8)
    w = rng.integers(-127, 128, (40, 256), dtype=np.int8)
    a_s = rng.uniform(1e-3, 1e-1, 16).astype(np.float32)
    w_s = rng.uniform(1e-3, 1e-2, 40).astype(np.float32)
    bias = rng.integers(0x3c00, 0x4100, 40).astype(np.uint16)  # bf16 bits, 0.0078 .. 8
    acc = oracle.gemm_i32(q, w)
    rows = rng.integers(0, 16, 50)
    cols = rng.integers(0, 40, 50)
    for b in (None, bias):
        y = oracle.epilogue(acc, a_s, w_s, b)
        acc_s, y_s = oracle.sampled(q, a_s, w, w_s, b, rows, cols)
        assert (acc_s == acc[rows, cols]).all()
        assert (y_s == y[rows, cols]).all()
