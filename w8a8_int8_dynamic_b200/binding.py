"""Thin ctypes binding of libw8a8.so.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch is used for device memory and the current stream.  There is
no fallback: if the shared library is missing or a call fails, this raises.

N-D activations [..., K] are flattened to [M, K] around the call and the
output is viewed back as [..., N] (the "Diffusion Quantization Reference",
GGUF rules: flatten N-D activations around the matmul and restore the shape;
its "Common Failures" table lists the output-rank collapse this avoids).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libw8a8.so")

OK = 0
STATUS_NAMES = {
    0: "W8A8_OK", 1: "W8A8_ERR_INVALID_ARG", 2: "W8A8_ERR_ALIGNMENT",
    3: "W8A8_ERR_UNSUPPORTED_SHAPE", 4: "W8A8_ERR_CUDA", 5: "W8A8_ERR_TIMEOUT",
    6: "W8A8_ERR_BUFFER_TOO_SMALL",
}

PATH_AUTO, PATH_LARGE, PATH_SMALL, PATH_LARGE_BN128, PATH_LARGE_BN256, PATH_LARGE_PAIR = 0, 1, 2, 3, 4, 5
PATH_LARGE_PAIR128 = 7
# activations fused into the GEMM epilogue (w8a8_act)
ACT_NONE, ACT_GELU_TANH = 0, 1


class W8A8Error(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "w8a8_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "w8a8_abi_version": ([], ctypes.c_int),
    "w8a8_quant_act": ([_P, _I64, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "w8a8_quant_act_static": ([_P, _I64, _I64, _I64, _P, _P, _P, _P], ctypes.c_int),
    "w8a8_packed_weight_bytes": ([_I64, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "w8a8_pack_weight": ([_P, _I64, _I64, _P, _SZ, _P], ctypes.c_int),
    "w8a8_unpack_weight": ([_P, _I64, _I64, _P, _P], ctypes.c_int),
    "w8a8_quant_pack_weight": ([_P, _I64, _I64, _P, _SZ, _P, _P], ctypes.c_int),
    "w8a8_pack_weight_int32": ([_P, _I64, _I64, _P, _SZ, _P], ctypes.c_int),
    "w8a8_scaled_mm_workspace_bytes": ([_I64, _I64, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "w8a8_scaled_mm": ([_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P], ctypes.c_int),
    "w8a8_scaled_mm_act": ([_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _SZ, _P],
                           ctypes.c_int),
    "w8a8_scaled_mm_i32": ([_P, _P, _P, _I64, _I64, _I64, _P], ctypes.c_int),
    "w8a8_linear_workspace_bytes": ([_I64, _I64, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "w8a8_linear": ([_P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P], ctypes.c_int),
    "w8a8_linear_act": ([_P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _SZ, _P],
                        ctypes.c_int),
    "w8a8_linear_act_quant_workspace_bytes": ([_I64, _I64, _I64, ctypes.POINTER(_SZ)],
                                              ctypes.c_int),
    "w8a8_linear_act_quant": ([_P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _P, _P,
                               _SZ, _P], ctypes.c_int),
    "w8a8_linear_noalloc_max_bytes": ([], _SZ),
    "w8a8_linear_noalloc": ([_P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, _P], ctypes.c_int),
    "w8a8_set_path": ([ctypes.c_int], ctypes.c_int),
    "w8a8_gemm_kernel_name": ([_I64, _I64, _I64], ctypes.c_char_p),
    "w8a8_gelu_tanh": ([_P, _P, _I64, _P], ctypes.c_int),
    "w8a8_poll_status": ([_P], ctypes.c_int),
    "w8a8_selftest_wait_timeout": ([_I64, _P], ctypes.c_int),
    "w8a8_selftest_int8_mma_rate": ([_I64, _P, ctypes.POINTER(ctypes.c_double)], ctypes.c_int),
    "w8a8_launch_count": ([], ctypes.c_int64),
}


def lib() -> ctypes.CDLL:
    """Load libw8a8.so (built in-tree by ``w8a8_int8_dynamic_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libw8a8.so not found at {LIB_PATH}; build it with "
                "`python -m w8a8_int8_dynamic_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != OK:
        raise W8A8Error(what, rc)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


# ---- sizes -------------------------------------------------------------------
def packed_weight_bytes(N: int, K: int) -> int:
    out = _SZ()
    _check(lib().w8a8_packed_weight_bytes(N, K, ctypes.byref(out)), "w8a8_packed_weight_bytes")
    return out.value


def linear_workspace_bytes(M: int, N: int, K: int) -> int:
    out = _SZ()
    _check(lib().w8a8_linear_workspace_bytes(M, N, K, ctypes.byref(out)),
           "w8a8_linear_workspace_bytes")
    return out.value


def linear_act_quant_workspace_bytes(M: int, N: int, K: int) -> int:
    out = _SZ()
    _check(lib().w8a8_linear_act_quant_workspace_bytes(M, N, K, ctypes.byref(out)),
           "w8a8_linear_act_quant_workspace_bytes")
    return out.value


def scaled_mm_workspace_bytes(M: int, N: int, K: int) -> int:
    out = _SZ()
    _check(lib().w8a8_scaled_mm_workspace_bytes(M, N, K, ctypes.byref(out)),
           "w8a8_scaled_mm_workspace_bytes")
    return out.value


# ---- ops ---------------------------------------------------------------------
def quant_act(x: torch.Tensor, q: Optional[torch.Tensor] = None,
              a_scale: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """x bf16 [M, K] (row stride may exceed K) -> (q int8 [M, K], a_scale fp32 [M])."""
    _need_cuda(x, "x", torch.bfloat16)
    M, K = x.shape
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if a_scale is None:
        a_scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().w8a8_quant_act(_ptr(x), M, K, x.stride(0), _ptr(q), _ptr(a_scale), _stream(stream)),
           "w8a8_quant_act")
    return q, a_scale


def quant_act_static(x: torch.Tensor, scale: torch.Tensor, q: Optional[torch.Tensor] = None,
                     a_scale: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """x bf16 [M, K] with one calibrated fp32 scale (a 1-element CUDA tensor)
    -> (q int8 [M, K], a_scale fp32 [M] filled with the scale used)."""
    _need_cuda(x, "x", torch.bfloat16)
    _need_cuda(scale, "scale", torch.float32)
    if scale.numel() != 1:
        raise ValueError("scale must hold exactly one value")
    M, K = x.shape
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if a_scale is None:
        a_scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().w8a8_quant_act_static(_ptr(x), M, K, x.stride(0), _ptr(scale), _ptr(q),
                                       _ptr(a_scale), _stream(stream)), "w8a8_quant_act_static")
    return q, a_scale


def quant_pack_weight(w: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 [N, K] -> (packed int8 tile image, fp32 per-channel w_scale [N]):
    quantisation at load time, in one pass."""
    _need_cuda(w, "w", torch.bfloat16)
    w = w.contiguous()
    N, K = w.shape
    nbytes = packed_weight_bytes(N, K)
    packed = torch.empty((nbytes,), dtype=torch.uint8, device=w.device)
    w_scale = torch.empty((N,), dtype=torch.float32, device=w.device)
    _check(lib().w8a8_quant_pack_weight(_ptr(w), N, K, _ptr(packed), nbytes, _ptr(w_scale),
                                        _stream(stream)), "w8a8_quant_pack_weight")
    return packed, w_scale


def pack_weight_int32(w_i32: torch.Tensor, K: int, stream=None) -> torch.Tensor:
    """int32 [N, K/4] biased-uint8 storage (four elements per word) -> packed
    tile image."""
    _need_cuda(w_i32, "w_i32", torch.int32)
    w_i32 = w_i32.contiguous()
    N = w_i32.shape[0]
    if w_i32.shape[1] * 4 != K:
        raise ValueError("w_i32 must be [N, K/4]")
    nbytes = packed_weight_bytes(N, K)
    packed = torch.empty((nbytes,), dtype=torch.uint8, device=w_i32.device)
    _check(lib().w8a8_pack_weight_int32(_ptr(w_i32), N, K, _ptr(packed), nbytes, _stream(stream)),
           "w8a8_pack_weight_int32")
    return packed


def pack_weight(w: torch.Tensor, stream=None) -> torch.Tensor:
    """int8 [N, K] (K contiguous) -> packed tile image (uint8, flat)."""
    _need_cuda(w, "w", torch.int8)
    w = w.contiguous()
    N, K = w.shape
    nbytes = packed_weight_bytes(N, K)
    packed = torch.empty((nbytes,), dtype=torch.uint8, device=w.device)
    _check(lib().w8a8_pack_weight(_ptr(w), N, K, _ptr(packed), nbytes, _stream(stream)),
           "w8a8_pack_weight")
    return packed


def unpack_weight(packed: torch.Tensor, N: int, K: int, stream=None) -> torch.Tensor:
    _need_cuda(packed, "packed")
    w = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    _check(lib().w8a8_unpack_weight(_ptr(packed), N, K, _ptr(w), _stream(stream)),
           "w8a8_unpack_weight")
    return w


def scaled_mm(q: torch.Tensor, a_scale: torch.Tensor, packed_w: torch.Tensor,
              w_scale: torch.Tensor, bias: Optional[torch.Tensor], N: int,
              out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
              stream=None, act: int = ACT_NONE) -> torch.Tensor:
    """q int8 [M, K] x packed W -> y bf16 [M, N] (``act``: epilogue activation)."""
    _need_cuda(q, "q", torch.int8)
    M, K = q.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        need = scaled_mm_workspace_bytes(M, N, K)
        if need:
            workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().w8a8_scaled_mm_act(_ptr(q), _ptr(a_scale), _ptr(packed_w), _ptr(w_scale),
                                    _ptr(bias), _ptr(out), M, N, K, act, _ptr(workspace), ws_bytes,
                                    _stream(stream)),
           "w8a8_scaled_mm_act")
    return out


def scaled_mm_i32(q: torch.Tensor, packed_w: torch.Tensor, N: int,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need_cuda(q, "q", torch.int8)
    M, K = q.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32, device=q.device)
    _check(lib().w8a8_scaled_mm_i32(_ptr(q), _ptr(packed_w), _ptr(out), M, N, K, _stream(stream)),
           "w8a8_scaled_mm_i32")
    return out


def linear(x: torch.Tensor, packed_w: torch.Tensor, w_scale: torch.Tensor,
           bias: Optional[torch.Tensor], N: int, out: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, stream=None,
           act: int = ACT_NONE) -> torch.Tensor:
    """The whole layer: y[..., N] = W8A8(x[..., K]) (``act``: epilogue activation)."""
    _need_cuda(x, "x", torch.bfloat16)
    lead = x.shape[:-1]
    K = x.shape[-1]
    x2 = x.reshape(-1, K)
    if x2.stride(1) != 1:
        x2 = x2.contiguous()
    M = x2.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty((linear_workspace_bytes(M, N, K),), dtype=torch.uint8,
                                device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().w8a8_linear_act(_ptr(x2), x2.stride(0), _ptr(packed_w), _ptr(w_scale), _ptr(bias),
                                 _ptr(out), M, N, K, act, _ptr(workspace), ws_bytes,
                                 _stream(stream)),
           "w8a8_linear_act")
    return out.view(*lead, N)


def linear_act_quant(x: torch.Tensor, packed_w: torch.Tensor, w_scale: torch.Tensor,
                     bias: Optional[torch.Tensor], N: int, out: Optional[torch.Tensor] = None,
                     q_next: Optional[torch.Tensor] = None,
                     a_scale_next: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None,
                     act: int = ACT_NONE) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """A layer whose output feeds another W8A8 layer: y = act(W8A8(x)) and
    the next layer's codes and scales of y, (y, q_next, a_scale_next), equal
    to ``linear`` followed by ``quant_act`` of its output."""
    _need_cuda(x, "x", torch.bfloat16)
    K = x.shape[-1]
    x2 = x.reshape(-1, K)
    if x2.stride(1) != 1:
        x2 = x2.contiguous()
    M = x2.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if q_next is None:
        q_next = torch.empty((M, N), dtype=torch.int8, device=x.device)
    if a_scale_next is None:
        a_scale_next = torch.empty((M,), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty((linear_act_quant_workspace_bytes(M, N, K),), dtype=torch.uint8,
                                device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().w8a8_linear_act_quant(_ptr(x2), x2.stride(0), _ptr(packed_w), _ptr(w_scale),
                                       _ptr(bias), _ptr(out), M, N, K, act, _ptr(q_next),
                                       _ptr(a_scale_next), _ptr(workspace), ws_bytes,
                                       _stream(stream)),
           "w8a8_linear_act_quant")
    return out, q_next, a_scale_next


def linear_noalloc(x: torch.Tensor, packed_w: torch.Tensor, w_scale: torch.Tensor,
                   bias: Optional[torch.Tensor], N: int, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """The whole layer with no workspace argument, for callers that cannot
    allocate device memory when they run a layer: the library keeps one
    scratch array per GPU (``linear_noalloc_max_bytes()`` bytes) for the codes,
    scales and small-M partials.  Calls that overlap on the GPU share it and
    race; order them on one stream."""
    _need_cuda(x, "x", torch.bfloat16)
    lead = x.shape[:-1]
    K = x.shape[-1]
    x2 = x.reshape(-1, K)
    if x2.stride(1) != 1:
        x2 = x2.contiguous()
    M = x2.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().w8a8_linear_noalloc(_ptr(x2), x2.stride(0), _ptr(packed_w), _ptr(w_scale), _ptr(bias),
                                     _ptr(out), M, N, K, _stream(stream)),
           "w8a8_linear_noalloc")
    return out.view(*lead, N)


def linear_noalloc_max_bytes() -> int:
    return int(lib().w8a8_linear_noalloc_max_bytes())


def gelu_tanh(x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need_cuda(x, "x", torch.bfloat16)
    x = x.contiguous()
    if out is None:
        out = torch.empty_like(x)
    _check(lib().w8a8_gelu_tanh(_ptr(x), _ptr(out), x.numel(), _stream(stream)), "w8a8_gelu_tanh")
    return out


def gemm_kernel_name(M: int, N: int, K: int) -> str:
    return lib().w8a8_gemm_kernel_name(M, N, K).decode()


def set_path(path: int):
    _check(lib().w8a8_set_path(path), "w8a8_set_path")


def poll_status(stream=None) -> int:
    return int(lib().w8a8_poll_status(_stream(stream)))


def selftest_int8_mma_rate(iters: int = 20000, stream=None) -> float:
    """int8 TOPS of a memory-free tcgen05.mma loop on every SM (synchronises)."""
    out = ctypes.c_double(0.0)
    _check(lib().w8a8_selftest_int8_mma_rate(iters, _stream(stream), ctypes.byref(out)),
           "w8a8_selftest_int8_mma_rate")
    return out.value


def selftest_wait_timeout(timeout_ns: int, stream=None):
    _check(lib().w8a8_selftest_wait_timeout(timeout_ns, _stream(stream)), "w8a8_selftest_wait_timeout")


def launch_count() -> int:
    return int(lib().w8a8_launch_count())


class W8A8Linear:
    """A pre-quantised linear layer: int8 weights [N, K] repacked once at
    load time, then applied on every call, fp32 per-output-channel
    scales, optional bf16 bias.  For fused Q/K/V, build it from the three
    blocks with :meth:`from_blocks` and split the output with :meth:`split`.
    """

    def __init__(self, w: torch.Tensor, w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                 splits: Optional[Tuple[int, ...]] = None, act: int = ACT_NONE):
        _need_cuda(w, "w", torch.int8)
        self.act = act
        self.N, self.K = w.shape
        self.packed = pack_weight(w)
        self.w_scale = w_scale.to(device=w.device, dtype=torch.float32).contiguous()
        self.bias = None if bias is None else bias.to(device=w.device, dtype=torch.bfloat16).contiguous()
        self.splits = tuple(splits) if splits else (self.N,)
        self._ws = None

    @classmethod
    def from_float(cls, w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                   act: int = ACT_NONE):
        """Online quantisation: a bf16 [N, K] weight quantised per output
        channel and packed on the device at load time."""
        self = cls.__new__(cls)
        self.act = act
        _need_cuda(w, "w", torch.bfloat16)
        self.N, self.K = w.shape
        self.packed, self.w_scale = quant_pack_weight(w)
        self.bias = None if bias is None else bias.to(device=w.device, dtype=torch.bfloat16).contiguous()
        self.splits = (self.N,)
        self._ws = None
        return self

    @classmethod
    def from_blocks(cls, blocks, scales, biases=None):
        w = torch.cat(list(blocks), dim=0)
        s = torch.cat(list(scales), dim=0)
        b = None if biases is None else torch.cat(list(biases), dim=0)
        return cls(w, s, b, splits=tuple(int(t.shape[0]) for t in blocks))

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        M = x.numel() // x.shape[-1]
        need = linear_workspace_bytes(M, self.N, self.K)
        if self._ws is None or self._ws.numel() < need or self._ws.device != x.device:
            self._ws = torch.empty((need,), dtype=torch.uint8, device=x.device)
        return linear(x, self.packed, self.w_scale, self.bias, self.N, workspace=self._ws,
                      act=self.act)

    def split(self, y: torch.Tensor):
        return torch.split(y, list(self.splits), dim=-1)
