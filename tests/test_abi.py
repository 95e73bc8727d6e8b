"""The C ABI library loads (no GPU needed), exports every entry point that
include/w8a8.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w8a8.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(w8a8_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from w8a8_int8_dynamic_b200 import build
    build.build()
    from w8a8_int8_dynamic_b200 import binding
    return binding.lib()


def test_header_declares_the_entry_points():
    d = _declared()
    for name in ["w8a8_quant_act", "w8a8_pack_weight", "w8a8_scaled_mm", "w8a8_linear",
                 "w8a8_poll_status", "w8a8_status_string"]:
        assert name in d


def test_library_exports_every_declared_symbol(L):
    from w8a8_int8_dynamic_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    extra = [n for n in exported if not n.startswith("w8a8_")]
    assert not extra, f"non-ABI symbols exported: {extra[:10]}"
    for n in _declared():
        assert hasattr(L, n)


def test_status_strings(L):
    assert L.w8a8_status_string(0) == b"W8A8_OK"
    assert L.w8a8_status_string(5) == b"W8A8_ERR_TIMEOUT"
    assert L.w8a8_status_string(99) == b"W8A8_ERR_UNKNOWN"
    assert L.w8a8_abi_version() >> 16 == 1


def test_packed_weight_bytes(L):
    from w8a8_int8_dynamic_b200 import binding
    assert binding.packed_weight_bytes(4096, 4096) == 4096 * 4096
    assert binding.packed_weight_bytes(304, 208) == 512 * 256
    assert binding.packed_weight_bytes(27648, 5120) == 27648 * 5120
    out = ctypes.c_size_t()
    assert L.w8a8_packed_weight_bytes(100, 20, ctypes.byref(out)) == 3  # K % 16
    assert L.w8a8_packed_weight_bytes(100, 16, ctypes.byref(out)) == 3  # N % 8
    assert L.w8a8_packed_weight_bytes(0, 16, ctypes.byref(out)) == 1
    assert L.w8a8_packed_weight_bytes(8, 131072 + 16, ctypes.byref(out)) == 3
    assert L.w8a8_packed_weight_bytes(8, 16, None) == 1


FAKE = ctypes.c_void_p(1 << 20)        # never dereferenced: checks fail first
FAKE_MIS = ctypes.c_void_p((1 << 20) + 4)


def test_quant_rejects_bad_arguments(L):
    f = L.w8a8_quant_act
    assert f(None, 4, 16, 16, FAKE, FAKE, None) == 1
    assert f(FAKE, 0, 16, 16, FAKE, FAKE, None) == 1
    assert f(FAKE, 4, 16, 8, FAKE, FAKE, None) == 1      # ldx < K
    assert f(FAKE, 4, 24, 24, FAKE, FAKE, None) == 3     # K % 16
    assert f(FAKE, 4, 16, 20, FAKE, FAKE, None) == 2     # ldx % 8
    assert f(FAKE_MIS, 4, 16, 16, FAKE, FAKE, None) == 2


def test_gemm_rejects_bad_arguments(L):
    f = L.w8a8_scaled_mm
    assert f(None, FAKE, FAKE, FAKE, None, FAKE, 4, 8, 16, None, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 12, 16, None, 0, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 8, 40, None, 0, None) == 3
    assert f(FAKE, FAKE, FAKE_MIS, FAKE, None, FAKE, 4, 8, 16, None, 0, None) == 2
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE_MIS, FAKE, 4, 8, 16, None, 0, None) == 2
    g = L.w8a8_linear
    assert g(FAKE, 16, FAKE, FAKE, None, FAKE, 4, 8, 16, None, 0, None) == 1       # no workspace
    assert g(FAKE, 16, FAKE, FAKE, None, FAKE, 4, 8, 16, FAKE, 1, None) == 6       # too small
    assert g(FAKE, 8, FAKE, FAKE, None, FAKE, 4, 8, 16, FAKE, 1 << 30, None) == 1  # ldx < K
    assert L.w8a8_set_path(9) == 1
    assert L.w8a8_set_path(8) == 1
    assert L.w8a8_set_path(6) == 1
    assert L.w8a8_set_path(7) == 0
    assert L.w8a8_set_path(0) == 0


def test_workspace_sizes(L):
    """Host-side sizing (no GPU: the SM count falls back to the B200's 148).
    The large-M kernels need no GEMM workspace, under every path setting; the
    layer's workspace is then the codes and scales, each rounded up to 256
    bytes.  Small M needs the split-K partials of the weight-streaming
    kernel."""
    from w8a8_int8_dynamic_b200 import binding
    assert binding.scaled_mm_workspace_bytes(512, 4096, 4096) == 0
    assert binding.linear_workspace_bytes(512, 4096, 4096) == 512 * 4096 + 2048
    assert binding.scaled_mm_workspace_bytes(4096, 12288, 3072) == 0
    assert binding.linear_workspace_bytes(4096, 12288, 3072) == 4096 * 3072 + 4096 * 4
    assert binding.scaled_mm_workspace_bytes(16, 27648, 5120) > 0
    for path in (1, 3, 4, 5, 7):
        assert L.w8a8_set_path(path) == 0
        try:
            assert binding.scaled_mm_workspace_bytes(512, 4096, 4096) == 0
            assert binding.linear_workspace_bytes(512, 4096, 4096) == 512 * 4096 + 2048
        finally:
            assert L.w8a8_set_path(0) == 0


def test_act_quant_rejects_bad_arguments_and_sizes_its_workspace(L):
    """w8a8_linear_act_quant: host-side checks before any launch, and the
    workspace: w8a8_linear's, then the row maxima (4 bytes a row), one 8-byte
    completion word per 128-row block, and one exit word, each rounded up to
    256 bytes."""
    from w8a8_int8_dynamic_b200 import binding
    f = L.w8a8_linear_act_quant
    big = 1 << 30
    ok = (FAKE, 16, FAKE, FAKE, None, FAKE, 4, 16, 16, 0, FAKE, FAKE, FAKE, big, None)
    # every argument valid but the one under test (nothing may launch)
    def call(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)
    assert call(a10=None) == 1                 # no q_next
    assert call(a11=None) == 1                 # no a_scale_next
    assert call(a12=None) == 1                 # no workspace
    assert call(a9=7) == 1                     # unknown activation
    assert call(a10=FAKE_MIS) == 2             # q_next misaligned
    assert call(a11=FAKE_MIS) == 2             # a_scale_next misaligned
    assert call(a13=1) == 6                    # workspace too small
    assert call(a7=(1 << 28) + 16) == 3        # N beyond the fused limit
    assert call(a7=24) == 3                    # N % 16 (the next layer's K)
    assert call(a8=40) == 3                    # K % 16
    for M, N, K in [(4096, 12288, 3072), (1000, 2064, 1040), (16, 4096, 4096)]:
        lin = binding.linear_workspace_bytes(M, N, K)
        rnd = lambda v: (v + 255) // 256 * 256  # noqa: E731
        extra = rnd(4 * M) + rnd(8 * ((M + 127) // 128)) + 256
        assert binding.linear_act_quant_workspace_bytes(M, N, K) == lin + extra


def test_mma_rate_selftest_rejects_bad_arguments(L):
    f = L.w8a8_selftest_int8_mma_rate
    tops = ctypes.c_double(0.0)
    assert f(0, None, ctypes.byref(tops)) == 1
    assert f(200001, None, ctypes.byref(tops)) == 1   # beyond the bounded wait's reach
    assert f(100, None, None) == 1
