"""The layer entry point that takes no workspace (w8a8_linear_noalloc).

It exists for callers that cannot allocate device memory when they run a
layer -- for example a plugin whose host framework owns all device memory and
forbids cudaMalloc inside its execution callbacks.  The library instead keeps
one fixed scratch array per GPU.  These tests call it through the C ABI and
check that two calls in a row give exactly what the workspace-taking entry
point (w8a8_linear) gives, on a large-M shape and on a small-M shape (whose
split-K counters in the shared array must be cleared on every call), and that
a problem too large for the array is refused without a launch.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import w8a8_int8_dynamic_b200 as w8
from w8a8_int8_dynamic_b200.binding import _ptr, _stream, lib
from w8a8_int8_dynamic_b200.workloads import random_case

pytestmark = pytest.mark.gpu


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _noalloc(x, packed, w_scale, bias, N):
    M, K = x.shape
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rc = lib().w8a8_linear_noalloc(_ptr(x), x.stride(0), _ptr(packed), _ptr(w_scale), _ptr(bias),
                                   _ptr(y), M, N, K, _stream())
    assert rc == 0, rc
    return y


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    w8.set_path(w8.PATH_AUTO)
    yield
    assert w8.poll_status() == 0


@pytest.mark.parametrize("M,N,K", [(512, 4096, 4096), (300, 1000, 528), (4, 27648, 5120), (16, 2048, 12288)])
def test_matches_workspace_entry_point_twice(M, N, K):
    inp = random_case(M + N + K, M, N, K, bias=True, n_outliers=K // 100, zero_row=M > 1)
    x = _dev_bf16(inp.x)
    packed = w8.pack_weight(torch.from_numpy(inp.w).cuda())
    ws = torch.from_numpy(inp.w_scale).cuda()
    b = _dev_bf16(inp.bias)
    ref = w8.linear(x, packed, ws, b, N)
    for _ in range(2):  # the second call sees the first call's leftovers in the array
        y = _noalloc(x, packed, ws, b, N)
        torch.cuda.synchronize()
        d = (y.view(torch.int16) != ref.view(torch.int16)).sum().item()
        assert d == 0, f"{d} outputs differ from w8a8_linear"


def test_refuses_problems_larger_than_the_array():
    cap = lib().w8a8_linear_noalloc_max_bytes()
    assert cap == 8 << 20
    M, N, K = 4096, 256, 4096  # 16 MiB of activation codes
    need = w8.linear_workspace_bytes(M, N, K)
    assert need > cap
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    before = w8.launch_count()
    rc = lib().w8a8_linear_noalloc(fake, K, fake, fake, None, fake, M, N, K, None)
    assert rc == 6  # W8A8_ERR_BUFFER_TOO_SMALL
    assert w8.launch_count() == before
