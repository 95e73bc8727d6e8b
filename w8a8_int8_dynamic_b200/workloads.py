"""Seeded synthetic inputs for the W8A8 int8-dynamic linear workloads.

This module only draws random inputs.  It holds none of the method's
arithmetic (no quantisation, no matmul, no scaling), so that both the CUDA
path and the CPU oracle can be fed the same bytes without sharing any of the
computation.  bf16 tensors are returned as uint16 bit patterns.

Recipe (numpy PCG64, ``np.random.default_rng(seed)``, draws in this order):
  1. x  : fp32 N(0, 1) of shape [M, K];
  2. outlier channels: the first ``n_outliers`` entries of a random
     permutation of range(K); those columns of x are multiplied by
     ``outlier_factor`` in fp32; then x is rounded to bf16 (nearest even);
     if ``zero_row`` the last row is set to +0;
  3. w  : int8 uniform on [-127, 127], shape [N, K] (K contiguous);
  4. w_scale: fp32 uniform on [lo, hi) for each block of output channels;
  5. bias (if any): fp32 N(0, 0.02) per output channel, rounded to bf16.

The shapes and distributions are those of the five workloads the method is
measured on: a small verification shape, a square 4096 projection, the fused
Q/K/V projection, the DiT MLP up/down pair at image-token scale and the
decode-shaped weight-streaming sweep.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np
import torch


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), rounding to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact)."""
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    n_outliers: int = 0
    outlier_factor: float = 1.0
    # (lo, hi, width) blocks of output channels; widths sum to N
    w_scale_blocks: Tuple[Tuple[float, float, int], ...] = ()
    bias: bool = False
    zero_row: bool = False
    seed: int = 0
    note: str = ""

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K


def _blocks(lo, hi, n):
    return ((lo, hi, n),)


WORKLOADS = {
    # small verification shape: 2 of 256 channels x20
    "small_64x128x256": Workload("small_64x128x256", 64, 128, 256, 2, 20.0,
                                 _blocks(1e-3, 1e-2, 128), False, False),
    # square projection, 1% outlier channels x10, bias, last row all zero
    "square_512x4096x4096": Workload("square_512x4096x4096", 512, 4096, 4096, 41, 10.0,
                                     _blocks(5e-4, 5e-3, 4096), True, True),
    # fused Q/K/V: three 4096-wide blocks with their own scale ranges, no bias
    "fused_qkv_512x12288x4096": Workload(
        "fused_qkv_512x12288x4096", 512, 12288, 4096, 41, 10.0,
        ((5e-4, 2e-3, 4096), (1e-3, 4e-3, 4096), (2e-3, 8e-3, 4096)), False, False),
    # DiT MLP up-projection at image-token scale
    "dit_mlp_up_4096x12288x3072": Workload("dit_mlp_up_4096x12288x3072", 4096, 12288, 3072, 0, 1.0,
                                           _blocks(5e-4, 5e-3, 12288), True, False),
    # DiT MLP row-parallel (wide-in) down-projection; in the chain its input is
    # GELU(tanh) of the up-projection output, standalone it is N(0, 1)
    "dit_mlp_down_4096x3072x12288": Workload("dit_mlp_down_4096x3072x12288", 4096, 3072, 12288, 0, 1.0,
                                             _blocks(5e-4, 5e-3, 3072), True, False, seed=1),
    # decode-shaped weight streaming, 0.5% outlier channels x30
    "decode_m1_27648x5120": Workload("decode_m1_27648x5120", 1, 27648, 5120, 26, 30.0,
                                     _blocks(5e-4, 5e-3, 27648), False, False),
    "decode_m4_27648x5120": Workload("decode_m4_27648x5120", 4, 27648, 5120, 26, 30.0,
                                     _blocks(5e-4, 5e-3, 27648), False, False),
    "decode_m16_27648x5120": Workload("decode_m16_27648x5120", 16, 27648, 5120, 26, 30.0,
                                      _blocks(5e-4, 5e-3, 27648), False, False),
}


@dataclass
class Inputs:
    x: np.ndarray          # uint16 bf16 bits [M, K]
    w: np.ndarray          # int8 [N, K]
    w_scale: np.ndarray    # fp32 [N]
    bias: Optional[np.ndarray]  # uint16 bf16 bits [N] or None
    outlier_channels: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


def make_activations(rng: np.random.Generator, M: int, K: int, n_outliers: int,
                     factor: float, zero_row: bool) -> Tuple[np.ndarray, np.ndarray]:
    x = rng.standard_normal((M, K), dtype=np.float32)
    ch = rng.permutation(K)[:n_outliers].astype(np.int64)
    if n_outliers:
        x[:, ch] *= np.float32(factor)
    xb = f32_to_bf16_bits(x)
    if zero_row and M > 0:
        xb[M - 1, :] = 0
    return xb, ch


def make_inputs(wl: Workload, M: Optional[int] = None) -> Inputs:
    """Draw the inputs of a workload.  ``M`` overrides the row count (the
    weights and scales do not depend on M)."""
    M = wl.M if M is None else M
    rng = np.random.default_rng(wl.seed)
    x, ch = make_activations(rng, M, wl.K, wl.n_outliers, wl.outlier_factor, wl.zero_row)
    w = rng.integers(-127, 128, size=(wl.N, wl.K), dtype=np.int8)
    parts = [rng.uniform(lo, hi, size=width).astype(np.float32)
             for (lo, hi, width) in wl.w_scale_blocks]
    w_scale = np.concatenate(parts) if parts else np.ones(wl.N, np.float32)
    assert w_scale.shape == (wl.N,)
    bias = None
    if wl.bias:
        bias = f32_to_bf16_bits((rng.standard_normal(wl.N) * 0.02).astype(np.float32))
    return Inputs(x, w, w_scale, bias, ch)


def random_case(seed: int, M: int, N: int, K: int, bias: bool = True,
                n_outliers: int = 0, factor: float = 10.0, zero_row: bool = False,
                scale_lo: float = 5e-4, scale_hi: float = 5e-3) -> Inputs:
    """An ad-hoc case for tests that sweep shapes (tails, odd M, ...)."""
    wl = Workload(f"case_{M}x{N}x{K}", M, N, K, n_outliers, factor,
                  _blocks(scale_lo, scale_hi, N), bias, zero_row, seed)
    return make_inputs(wl)


def list_workloads() -> List[str]:
    return list(WORKLOADS)
