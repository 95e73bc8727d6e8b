"""Pins for the oracle's load-time weight repack.

Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
Round two (kernel-path verification): the layer's weights are transposed
and repacked once as they are loaded, then applied, and the loaded weights
(the fused Q/K/V ones too) are checked bit for bit.  The packed layout itself is this library's
own (the UMMA K-major 128-byte-swizzled shared-memory tile image); it is
pinned by hand-derived offsets, a bijection check, the padding rule, and the
128-byte swizzle identity it must equal.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pack_offsets.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            n, k, off = (int(t) for t in line.split())
            rows.append((n, k, off))
    return rows


def test_hand_derived_offsets():
    N, K = 300, 200
    assert oracle.packed_bytes(N, K) == 131072
    rng = np.random.default_rng(0)
    w = rng.integers(-127, 128, (N, K), dtype=np.int8)
    p = oracle.pack_weight(w)
    for n, k, off in _golden():
        assert p[off] == w[n, k], (n, k, off)


@pytest.mark.parametrize("shape", [(128, 128), (300, 200), (256, 16), (1, 48), (520, 384)])
def test_bijection_and_zero_padding(shape):
    N, K = shape
    # unique tag per element: use an int32 index image packed as 4 byte planes
    idx = np.arange(N * K, dtype=np.int64).reshape(N, K)
    seen = np.zeros(oracle.packed_bytes(N, K), np.int64)
    for plane in range(3):
        w = ((idx >> (8 * plane)) & 0xFF).astype(np.uint8).view(np.int8)
        seen |= (oracle.pack_weight(w).view(np.uint8).astype(np.int64) << (8 * plane))
    w1 = np.ones((N, K), np.int8)
    mask = oracle.pack_weight(w1) == 1
    assert mask.sum() == N * K
    assert sorted(seen[mask].tolist()) == list(range(N * K))
    assert (oracle.pack_weight(w1)[~mask] == 0).all()


def test_equals_128B_swizzle_of_row_major_tiles():
    """Inside a tile, the image is the row-major 128x128 tile with the
    16-byte chunk index XOR-ed with (row mod 8) -- i.e. byte offset o maps to
    o XOR (((o >> 7) & 7) << 4), the 128-byte swizzle pattern."""
    rng = np.random.default_rng(1)
    w = rng.integers(-127, 128, (256, 128), dtype=np.int8)
    p = oracle.pack_weight(w)
    tile = w[:128, :128].reshape(-1)
    o = np.arange(128 * 128)
    sw = o ^ (((o >> 7) & 7) << 4)
    assert (p[:16384][sw] == tile).all()


def test_fused_qkv_blocks_pack_like_one_weight():
    """Stacking Q, K, V along N and packing once equals packing each block
    into its own 4096-row slice (tile rows never straddle the blocks)."""
    rng = np.random.default_rng(2)
    K = 256
    blocks = [rng.integers(-127, 128, (512, K), dtype=np.int8) for _ in range(3)]
    fused = oracle.pack_weight(np.concatenate(blocks, axis=0))
    per = [oracle.pack_weight(b) for b in blocks]
    step = oracle.packed_bytes(512, K)
    for i in range(3):
        assert (fused[i * step:(i + 1) * step] == per[i]).all()
