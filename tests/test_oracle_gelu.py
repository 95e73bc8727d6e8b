"""Pins for the oracle's GELU (tanh form), used only between the up and
down projections of the DiT MLP workload (the pages do not define it).

Pinned by closed forms of the tanh form, its odd-part identity, and its known
distance from the exact erf GELU (a library routine)."""
from decimal import Decimal, getcontext

import numpy as np
from scipy.special import erf

import oracle
from w8a8_int8_dynamic_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _g(vals):
    x = f32_to_bf16_bits(np.asarray(vals, np.float32))
    return bf16_bits_to_f32(oracle.gelu_tanh(x)).astype(np.float64), bf16_bits_to_f32(x).astype(np.float64)


def test_closed_forms():
    y, x = _g([0.0, 20.0, -20.0, 100.0])
    assert y[0] == 0.0
    assert y[1] == 20.0 and y[3] == 100.0     # tanh saturates: gelu(x) = x
    assert y[2] == 0.0 or abs(y[2]) < 1e-30   # gelu(-20) underflows towards 0


def test_odd_part_identity():
    # gelu(x) - gelu(-x) = x for the tanh form; bf16 rounding of each side
    rng = np.random.default_rng(0)
    v = rng.standard_normal(4000).astype(np.float32) * 3
    yp, x = _g(v)
    ym, _ = _g(-v)
    tol = 2.0 ** -8 * (np.abs(yp) + np.abs(ym)) + 1e-30
    assert (np.abs((yp - ym) - x) <= tol).all()


def test_close_to_erf_gelu():
    rng = np.random.default_rng(1)
    v = rng.uniform(-6, 6, 20000).astype(np.float32)
    y, x = _g(v)
    exact = 0.5 * x * (1 + erf(x / np.sqrt(2)))
    # tanh-approximation error (< 5e-4 in absolute terms) + half a bf16 ulp
    assert (np.abs(y - exact) <= 5e-4 + 2.0 ** -8 * np.abs(exact)).all()


def test_positive_part_monotone():
    v = np.linspace(0, 8, 2001, dtype=np.float32)
    y, _ = _g(v)
    assert (np.diff(y) >= 0).all()


def _gelu_decimal(x: float) -> Decimal:
    """GELU_tanh at 60 significant digits: 0.5 x (1 + tanh(u)) with tanh
    written through exp, evaluated in decimal arithmetic."""
    getcontext().prec = 60
    d = Decimal(x)
    pi = Decimal("3.14159265358979323846264338327950288419716939937510582097494")
    u = (Decimal(2) / pi).sqrt() * (d + Decimal("0.044715") * d * d * d)
    t = ((2 * u).exp() - 1) / ((2 * u).exp() + 1)  # tanh(u)
    return Decimal("0.5") * d * (1 + t)


def test_matches_high_precision_including_negative_tail():
    """Against a 60-digit evaluation of the tanh form, including the tail
    x in [-12, -3] where 1 + tanh(u) cancels in binary floating point."""
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.uniform(-12, -3, 600), rng.uniform(-3, 3, 300),
                        rng.uniform(3, 12, 100)]).astype(np.float32)
    y, x = _g(v)
    for xi, yi in zip(x, y):
        ref = _gelu_decimal(float(xi))
        if ref == 0:
            assert yi == 0
            continue
        # one correct rounding to bf16: half an ulp of 8 significant bits, or
        # half the smallest bf16 subnormal (2^-133) below the normal range
        tol = max(abs(ref) * Decimal(2) ** -8, Decimal(2) ** -134)
        assert abs(Decimal(float(yi)) - ref) <= tol, (xi, yi, ref)
