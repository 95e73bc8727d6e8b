"""Helpers for the GPU parity tests: host <-> device moves and comparisons.
No arithmetic of the method lives here."""
import numpy as np
import pytest
import torch


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")


def dev_bf16(a_u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_ulp_diff(a_u16: np.ndarray, b_u16: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps (units of the ordered integer encoding);
    +0 and -0 are the same value."""
    def ordered(h):
        h = h.astype(np.int32)
        mag = h & 0x7FFF
        return np.where(h & 0x8000, -mag, mag)
    return np.abs(ordered(a_u16) - ordered(b_u16))


def assert_bf16_close(got_u16, exp_u16, max_ulp=1, what="y"):
    d = bf16_ulp_diff(got_u16, exp_u16)
    worst = int(d.max()) if d.size else 0
    n_bad = int((d > max_ulp).sum())
    assert n_bad == 0, f"{what}: {n_bad} elements differ by more than {max_ulp} bf16 ulp (worst {worst})"
    return int((d != 0).sum())
