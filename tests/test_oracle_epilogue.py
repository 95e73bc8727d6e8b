"""Pins for the oracle's dequantising epilogue and its bf16 rounding.

Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
Round two: int8 weights with fp32 per-channel scales, per-token activation
scales, bf16 output; the lesson recorded there (a missing x act_scale factor
makes the out/ref norm ratio equal E[act_scale]) shows the row scale
multiplies the integer product.  The operation order (acc*a_s)*w_s (+bias),
each step one fp32 rounding, then one rounding to bf16, is this library's
reading; it is pinned with exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from exact import epilogue_element, from_bf16_bits, from_f32, rn_bf16
from w8a8_int8_dynamic_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits


def test_bf16_rounding_worked_examples():
    f2b = oracle.f32_to_bf16
    assert f2b(1.0) == 0x3F80
    assert f2b(-2.0) == 0xC000
    assert f2b(1.0 + 2.0 ** -8) == 0x3F80          # tie, even neighbour below
    assert f2b(1.0 + 3 * 2.0 ** -8) == 0x3F82      # tie, even neighbour above
    assert f2b(1.0 + 2.0 ** -8 + 2.0 ** -20) == 0x3F81  # just above the tie
    assert f2b(float(np.float32(3.4e38))) == 0x7F80  # rounds up to +inf
    assert f2b(0.0) == 0x0000 and f2b(-0.0) == 0x8000
    assert f2b(2.0 ** -133) == 0x0001 or f2b(2.0 ** -133) == 0x0000  # subnormal region
    assert oracle.f64_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81  # single rounding


def test_double_to_bf16_is_one_rounding_next_to_a_tie():
    """Doubles a hair from a bf16 midpoint, closer than half an fp32 ulp: a
    first rounding to fp32 would land on the midpoint itself, so only a
    single correct rounding (nearest, ties even) gets these right."""
    f = oracle.f64_to_bf16
    eps = 2.0 ** -40
    for sign, bits in ((1.0, 0x0000), (-1.0, 0x8000)):
        assert f(sign * (1.0 + 2.0 ** -8 - eps)) == bits | 0x3F80   # below the tie: down
        assert f(sign * (1.0 + 2.0 ** -8)) == bits | 0x3F80         # the tie: even (down)
        assert f(sign * (1.0 + 2.0 ** -8 + eps)) == bits | 0x3F81   # above the tie: up
        assert f(sign * (1.0 + 3 * 2.0 ** -8 - eps)) == bits | 0x3F81  # below the next tie
        assert f(sign * (1.0 + 3 * 2.0 ** -8)) == bits | 0x3F82     # that tie: even (up)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(20000) * rng.choice([1e-3, 1.0, 1e3], 20000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(t)) for t in v], np.uint16)
    assert (got == ref).all()


def test_exact_rational_emulation():
    rng = np.random.default_rng(1)
    M, N = 12, 20
    acc = rng.integers(-2 ** 30, 2 ** 30, (M, N), dtype=np.int64).astype(np.int32)
    acc[0, :5] = [0, 1, -1, 2 ** 24 + 1, -(2 ** 24 + 3)]  # exact and inexact int->float
    a_s = rng.uniform(1e-4, 1e-1, M).astype(np.float32)
    w_s = rng.uniform(5e-4, 5e-3, N).astype(np.float32)
    bias = f32_to_bf16_bits((rng.standard_normal(N) * 0.02).astype(np.float32))
    for b in (None, bias):
        y = oracle.epilogue(acc, a_s, w_s, b)
        for m in range(M):
            for n in range(N):
                bb = None if b is None else from_bf16_bits(int(b[n]))
                e = epilogue_element(int(acc[m, n]), from_f32(a_s[m]), from_f32(w_s[n]), bb)
                if e is None:  # exact zero: +0 or -0 both acceptable for equality
                    assert int(y[m, n]) & 0x7FFF == 0
                else:
                    assert int(y[m, n]) == e, (m, n)


def test_order_discriminating_cases():
    """Cases where acc*(a_s*w_s) or (acc*w_s)*a_s lands on a different bf16
    than (acc*a_s)*w_s; the oracle must follow the stated order."""
    rng = np.random.default_rng(2)
    n = 4_000_000
    acc = rng.integers(-2 ** 28, 2 ** 28, n).astype(np.int32)
    a_s = rng.uniform(1e-3, 1e-1, n).astype(np.float32)
    w_s = rng.uniform(1e-3, 1e-2, n).astype(np.float32)
    accf = acc.astype(np.float32)
    t_ref = (accf * a_s) * w_s
    t_alt = accf * (a_s * w_s)
    b_ref = f32_to_bf16_bits(t_ref)
    b_alt = f32_to_bf16_bits(t_alt)
    idx = np.nonzero(b_ref != b_alt)[0][:30]
    assert idx.size >= 3
    for i in idx:
        y = oracle.epilogue(acc[i:i + 1, None], a_s[i:i + 1], w_s[i:i + 1])
        e = epilogue_element(int(acc[i]), from_f32(a_s[i]), from_f32(w_s[i]), None)
        assert int(y[0, 0]) == e


def test_within_half_ulp_of_exact_value():
    rng = np.random.default_rng(3)
    M, N = 64, 64
    acc = rng.integers(-2 ** 27, 2 ** 27, (M, N)).astype(np.int32)
    a_s = rng.uniform(1e-3, 1e-1, M).astype(np.float32)
    w_s = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    y = bf16_bits_to_f32(oracle.epilogue(acc, a_s, w_s)).astype(np.float64)
    exact = acc.astype(np.float64) * a_s[:, None].astype(np.float64) * w_s[None, :].astype(np.float64)
    ulp = np.abs(exact) * 2.0 ** -7
    # half a bf16 ulp plus three fp32 roundings
    assert (np.abs(y - exact) <= 0.5 * ulp + 4 * 2.0 ** -24 * np.abs(exact) + 1e-45).all()


def test_row_scale_norm_ratio_diagnostic():
    """Dropping the row scale makes out/ref equal E[a_scale] (the diagnostic
    of the page's 97%-error scare): with the scale applied the ratio is ~1."""
    rng = np.random.default_rng(4)
    M, N, K = 128, 96, 256
    x = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = rng.integers(-127, 128, (N, K), dtype=np.int8)
    w_s = rng.uniform(5e-4, 5e-3, N).astype(np.float32)
    y, q, a_s, acc = oracle.linear(x, w, w_s)
    yf = bf16_bits_to_f32(y).astype(np.float64)
    wdq = w.astype(np.float64) * w_s[:, None]
    ref_good = (q.astype(np.float64) * a_s[:, None]) @ wdq.T
    ref_missing = q.astype(np.float64) @ wdq.T
    r_good = np.linalg.norm(yf) / np.linalg.norm(ref_good)
    r_missing = np.linalg.norm(yf) / np.linalg.norm(ref_missing)
    assert abs(r_good - 1) < 1e-3
    assert abs(r_missing / a_s.mean() - 1) < 0.05


def test_bias_is_added_in_fp32():
    acc = np.array([[1000]], np.int32)
    a_s = np.array([0.5], np.float32)
    w_s = np.array([0.25], np.float32)
    bias = f32_to_bf16_bits(np.array([1.0], np.float32))
    y = oracle.epilogue(acc, a_s, w_s, bias)
    assert bf16_bits_to_f32(y)[0, 0] == 126.0  # 1000*0.5*0.25 + 1 = 126


def test_layer_reads_rows_at_their_stride():
    """The whole layer on rows spaced ldx > K apart equals the layer on the
    same rows packed densely: the columns past K never enter it."""
    import ctypes
    rng = np.random.default_rng(12)
    M, N, K, ldx = 9, 24, 64, 80
    big = f32_to_bf16_bits(rng.standard_normal((M, ldx)).astype(np.float32) * 2)
    big[:, K:] = f32_to_bf16_bits(np.full((M, ldx - K), 3e4, np.float32))
    w = rng.integers(-127, 128, (N, K), dtype=np.int8)
    w_s = rng.uniform(5e-4, 5e-3, N).astype(np.float32)
    bias = f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    y_ref, q_ref, s_ref, acc_ref = oracle.linear(np.ascontiguousarray(big[:, :K]), w, w_s, bias)
    y = np.empty((M, N), np.uint16)
    q = np.empty((M, K), np.int8)
    a_s = np.empty((M,), np.float32)
    acc = np.empty((M, N), np.int32)
    p_ = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = oracle.lib().w8a8o_linear(p_(big), ldx, p_(w), p_(w_s), p_(bias), M, N, K,
                                   p_(y), p_(q), p_(a_s), p_(acc))
    assert rc == 0
    assert (q == q_ref).all() and (a_s.view(np.uint32) == s_ref.view(np.uint32)).all()
    assert (acc == acc_ref).all() and (y == y_ref).all()
