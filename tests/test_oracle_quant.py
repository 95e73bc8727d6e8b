"""Pins for the oracle's dynamic per-token activation quantisation.

Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
Round two (int8 weights; int8 activations with one symmetric scale per
token, computed at run time);
"Online Quantization", Parameters (activation_scheme "dynamic").

The oracle is checked against the mathematics, not against a retyped copy of
itself: exact rational arithmetic with explicit IEEE rounding, hand-worked
examples, closed forms and invariants.
"""
import ctypes
from fractions import Fraction

import numpy as np
import pytest

import oracle
from exact import from_bf16_bits, quant_element, rn32
from w8a8_int8_dynamic_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits


def bf(vals):
    return f32_to_bf16_bits(np.asarray(vals, np.float32))


def test_worked_half_even_example():
    # amax = 127 gives scale exactly 1, so x/s = x and the ties are exact:
    # 2.5 -> 2, 3.5 -> 4, -2.5 -> -2, 0.5 -> 0, 1.5 -> 2 (round half to even)
    x = bf([[127.0, 2.5, 3.5, -2.5, 0.5, 1.5, -0.5, 126.5]])
    q, s = oracle.quant_act(x)
    assert s[0] == np.float32(1.0)
    assert q.tolist() == [[127, 2, 4, -2, 0, 2, 0, 126]]


def test_worked_scale_two_example():
    # amax = 254 -> s = 2 exactly; x = 5 -> 2.5 -> 2; x = 7 -> 3.5 -> 4; x = -1 -> -0.5 -> 0
    x = bf([[254.0, 5.0, 7.0, -1.0, -3.0]])
    q, s = oracle.quant_act(x)
    assert s[0] == np.float32(2.0)
    assert q.tolist() == [[127, 2, 4, 0, -2]]


def test_zero_row_gives_zero_scale_and_codes():
    x = np.zeros((3, 32), np.uint16)
    x[1, 5] = bf([1.0])[0]
    q, s = oracle.quant_act(x)
    assert s[0] == 0.0 and s[2] == 0.0
    assert not q[0].any() and not q[2].any()
    assert q[1, 5] == 127 and s[1] == np.float32(1.0) / np.float32(127.0)


def test_negative_zero_row_is_a_zero_row():
    x = np.full((1, 16), 0x8000, np.uint16)  # -0.0 everywhere
    q, s = oracle.quant_act(x)
    assert s[0] == 0.0 and not q.any()


@pytest.mark.parametrize("c", [1.0, -3.25, 1e-30, 6.5e4, -2.0 ** -130])
def test_all_equal_row(c):
    # every element equals c: q = sign(c) * 127 and s = RN32(|c| / 127)
    x = bf(np.full((1, 48), c, np.float32))
    cb = from_bf16_bits(int(x[0, 0]))
    q, s = oracle.quant_act(x)
    assert Fraction(float(s[0])) == rn32(abs(cb) / 127)
    assert (q == (127 if cb > 0 else -127)).all()


def _exact_rows(x_bits):
    """Quantise rows with exact rational arithmetic (independent of C)."""
    M, K = x_bits.shape
    qs = np.zeros((M, K), np.int64)
    ss = []
    for m in range(M):
        vals = [from_bf16_bits(int(h)) for h in x_bits[m]]
        amax = max(abs(v) for v in vals)
        s = None
        for k, v in enumerate(vals):
            s, qk = quant_element(v, amax)
            qs[m, k] = qk
        if amax == 0:
            s = Fraction(0)
        ss.append(s)
    return qs, ss


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_exact_rational_arithmetic(seed):
    rng = np.random.default_rng(100 + seed)
    M, K = 6, 96
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.permutation(K)[:3]] *= 20.0
    x[1] *= 1e-3
    x[2] *= 3e4
    x[3, :] = 0.0
    x[3, 7] = -2.0 ** -133  # subnormal-only row: the scale is subnormal too
    xb = bf(x)
    q, s = oracle.quant_act(xb)
    qe, se = _exact_rows(xb)
    assert (q.astype(np.int64) == qe).all()
    for m in range(M):
        assert Fraction(float(s[m])) == se[m]


def test_division_not_reciprocal_multiply():
    """Find bf16 (amax, x) pairs where multiplying by RN32(1/s) rounds to a
    different integer than the IEEE quotient; the oracle must follow the
    quotient (exactly as rational arithmetic gives it)."""
    rng = np.random.default_rng(7)
    found = 0
    for _ in range(4000):
        amax = float(bf16_bits_to_f32(bf([rng.uniform(0.5, 400.0)]))[0])
        s = np.float32(np.float32(amax) / np.float32(127.0))
        inv = np.float32(np.float32(1.0) / s)
        xs = bf16_bits_to_f32(bf(rng.uniform(-amax, amax, 64).astype(np.float32)))
        v_div = (xs / s).astype(np.float32)
        v_rcp = (xs * inv).astype(np.float32)
        diff = np.nonzero(np.rint(v_div) != np.rint(v_rcp))[0]
        if diff.size == 0:
            continue
        row = np.concatenate([[np.float32(amax)], xs[diff]]).astype(np.float32)
        xb = bf(row[None, :])
        q, _ = oracle.quant_act(xb)
        qe, _ = _exact_rows(xb)
        assert (q.astype(np.int64) == qe).all()
        # and the oracle indeed differs from the reciprocal route there
        assert (q[0, 1:] != np.rint(v_rcp[diff]).astype(np.int64)).all()
        found += diff.size
        if found >= 20:
            break
    assert found >= 5, "search found too few discriminating cases"


@pytest.mark.parametrize("seed", [0, 1])
def test_invariants_random(seed):
    rng = np.random.default_rng(seed)
    M, K = 64, 512
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.permutation(K)[:8]] *= 10.0
    xb = bf(x)
    q, s = oracle.quant_act(xb)
    xf = bf16_bits_to_f32(xb).astype(np.float64)
    assert q.min() >= -127 and q.max() <= 127
    amax = np.abs(xf).max(axis=1)
    # scale is amax/127 rounded once to fp32
    assert (s == (amax.astype(np.float32) / np.float32(127.0))).all()
    # the amax element(s) map to +-127
    for m in range(M):
        idx = np.nonzero(np.abs(xf[m]) == amax[m])[0]
        assert (np.abs(q[m, idx]) == 127).all()
        assert (np.sign(q[m, idx]) == np.sign(xf[m, idx])).all()
    # |x - q s| <= s (1/2 + 128 * 2^-24)
    err = np.abs(xf - q.astype(np.float64) * s[:, None].astype(np.float64))
    bound = s[:, None].astype(np.float64) * (0.5 + 128 * 2.0 ** -24)
    assert (err <= bound).all()


@pytest.mark.parametrize("K", [1, 7, 256])
def test_row_maximum_at_every_position(K):
    """Row m of a K x K input has its largest magnitude in column m (the
    first, a middle and the last column among them): wherever it sits, the
    scale is that magnitude / 127 and its code is +-127."""
    rng = np.random.default_rng(K)
    x = rng.uniform(-1.0, 1.0, (K, K)).astype(np.float32)
    big = np.where(rng.random(K) < 0.5, -4.0, 4.0).astype(np.float32)
    x[np.arange(K), np.arange(K)] = big
    q, s = oracle.quant_act(bf(x))
    assert (s == np.float32(4.0) / np.float32(127.0)).all()
    assert (q[np.arange(K), np.arange(K)] == np.where(big < 0, -127, 127)).all()


def test_sign_symmetry():
    rng = np.random.default_rng(3)
    xb = bf(rng.standard_normal((8, 128)).astype(np.float32))
    q1, s1 = oracle.quant_act(xb)
    q2, s2 = oracle.quant_act(xb ^ np.uint16(0x8000))
    assert (s1 == s2).all() and (q1 == -q2).all()


def test_row_stride():
    """ldx > K: the padding columns must not influence the row."""
    rng = np.random.default_rng(4)
    M, K, ldx = 5, 64, 80
    big = bf(rng.standard_normal((M, ldx)).astype(np.float32) * 3)
    big[:, K:] = bf([1e4])[0]  # huge values in the padding
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    rc = oracle.lib().w8a8o_quant_act(big.ctypes.data_as(ctypes.c_void_p), M, K, ldx,
                                      q.ctypes.data_as(ctypes.c_void_p),
                                      s.ctypes.data_as(ctypes.c_void_p))
    assert rc == 0
    q2, s2 = oracle.quant_act(np.ascontiguousarray(big[:, :K]))
    assert (q == q2).all() and (s == s2).all()
