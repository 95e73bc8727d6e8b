"""CPU oracle for the W8A8 int8-dynamic linear path -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline / reference
leg may import this package.  The product library never does, and this package
never imports the product library.

The arithmetic lives in ``w8a8_oracle.c`` (plain C); this module only moves
numpy arrays in and out through ctypes.  bf16 arrays are carried as uint16.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        # The mutation test points W8A8_ORACLE_LIB at a deliberately altered
        # build of this oracle, to check that the pins catch the alteration.
        path = os.environ.get("W8A8_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.w8a8o_quant_act.argtypes = [P, I64, I64, I64, P, P]
        L.w8a8o_gemm_i32.argtypes = [P, P, I64, I64, I64, P]
        L.w8a8o_epilogue.argtypes = [P, P, P, P, I64, I64, P]
        L.w8a8o_linear.argtypes = [P, I64, P, P, P, I64, I64, I64, P, P, P, P]
        L.w8a8o_sampled.argtypes = [P, P, P, P, P, I64, P, P, I64, P, P]
        L.w8a8o_pack_weight.argtypes = [P, I64, I64, P]
        L.w8a8o_packed_bytes.argtypes = [I64, I64]
        L.w8a8o_packed_bytes.restype = I64
        L.w8a8o_gelu_tanh.argtypes = [P, I64, P]
        L.w8a8o_f32_to_bf16.argtypes = [ctypes.c_float]
        L.w8a8o_f32_to_bf16.restype = ctypes.c_uint16
        L.w8a8o_f64_to_bf16.argtypes = [ctypes.c_double]
        L.w8a8o_f64_to_bf16.restype = ctypes.c_uint16
        L.w8a8o_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.w8a8o_bf16_to_f32.restype = ctypes.c_float
        L.w8a8o_num_threads.restype = ctypes.c_int
        L.w8a8o_set_num_threads.argtypes = [ctypes.c_int]
        L.w8a8o_set_num_threads.restype = None
        L.w8a8o_quant_weight.argtypes = [P, I64, I64, P, P]
        L.w8a8o_quant_act_static.argtypes = [P, I64, I64, I64, ctypes.c_float, P, P]
        L.w8a8o_unpack_int32.argtypes = [P, I64, I64, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc == 2:
        raise OverflowError(f"{what}: an int32 accumulator overflowed")
    if rc != 0:
        raise ValueError(f"{what}: invalid arguments (rc={rc})")


def num_threads() -> int:
    return lib().w8a8o_num_threads()


def set_num_threads(n: int) -> None:
    """Threads used by later calls (OpenMP); for timing the oracle alone."""
    lib().w8a8o_set_num_threads(int(n))


def quant_act(x_bf16: np.ndarray):
    """x: uint16 (bf16 bits) [M, K] -> (q int8 [M, K], a_scale fp32 [M])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty((M,), np.float32)
    _check(lib().w8a8o_quant_act(_p(x), M, K, K, _p(q), _p(s)), "quant_act")
    return q, s


def gemm_i32(q: np.ndarray, w: np.ndarray) -> np.ndarray:
    """q int8 [M, K], w int8 [N, K] -> acc int32 [M, N] (exact)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    w = np.ascontiguousarray(w, dtype=np.int8)
    M, K = q.shape
    N = w.shape[0]
    assert w.shape[1] == K
    acc = np.empty((M, N), np.int32)
    _check(lib().w8a8o_gemm_i32(_p(q), _p(w), M, N, K, _p(acc)), "gemm_i32")
    return acc


def epilogue(acc, a_scale, w_scale, bias=None) -> np.ndarray:
    """acc int32 [M, N] -> y bf16 bits (uint16) [M, N]."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    a_scale = np.ascontiguousarray(a_scale, dtype=np.float32)
    w_scale = np.ascontiguousarray(w_scale, dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    M, N = acc.shape
    y = np.empty((M, N), np.uint16)
    _check(lib().w8a8o_epilogue(_p(acc), _p(a_scale), _p(w_scale), _p(b), M, N, _p(y)),
           "epilogue")
    return y


def linear(x_bf16, w, w_scale, bias=None):
    """The whole layer.  Returns (y, q, a_scale, acc)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.int8)
    w_scale = np.ascontiguousarray(w_scale, dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    M, K = x.shape
    N = w.shape[0]
    y = np.empty((M, N), np.uint16)
    q = np.empty((M, K), np.int8)
    s = np.empty((M,), np.float32)
    acc = np.empty((M, N), np.int32)
    _check(lib().w8a8o_linear(_p(x), K, _p(w), _p(w_scale), _p(b), M, N, K,
                              _p(y), _p(q), _p(s), _p(acc)), "linear")
    return y, q, s, acc


def sampled(q, a_scale, w, w_scale, bias, rows, cols):
    """acc and y at the output positions (rows[i], cols[i])."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    w = np.ascontiguousarray(w, dtype=np.int8)
    a_scale = np.ascontiguousarray(a_scale, dtype=np.float32)
    w_scale = np.ascontiguousarray(w_scale, dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    K = q.shape[1]
    acc = np.empty(rows.shape, np.int32)
    y = np.empty(rows.shape, np.uint16)
    _check(lib().w8a8o_sampled(_p(q), _p(a_scale), _p(w), _p(w_scale), _p(b), K,
                               _p(rows), _p(cols), rows.size, _p(acc), _p(y)),
           "sampled")
    return acc, y


def packed_bytes(N: int, K: int) -> int:
    return int(lib().w8a8o_packed_bytes(N, K))


def pack_weight(w: np.ndarray) -> np.ndarray:
    """int8 [N, K] -> packed tile image (uint8 bytes, flat)."""
    w = np.ascontiguousarray(w, dtype=np.int8)
    N, K = w.shape
    out = np.empty((packed_bytes(N, K),), np.int8)
    _check(lib().w8a8o_pack_weight(_p(w), N, K, _p(out)), "pack_weight")
    return out


def gelu_tanh(x_bf16: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    y = np.empty_like(x)
    _check(lib().w8a8o_gelu_tanh(_p(x), x.size, _p(y)), "gelu_tanh")
    return y


def f32_to_bf16(v: float) -> int:
    return int(lib().w8a8o_f32_to_bf16(v))


def f64_to_bf16(v: float) -> int:
    return int(lib().w8a8o_f64_to_bf16(v))


def bf16_to_f32(h: int) -> float:
    return float(lib().w8a8o_bf16_to_f32(h))


def quant_weight(w_bf16: np.ndarray):
    """bf16 bits [N, K] -> (int8 [N, K], fp32 per-output-channel scale [N])."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N,), np.float32)
    _check(lib().w8a8o_quant_weight(_p(w), N, K, _p(q), _p(s)), "quant_weight")
    return q, s


def quant_act_static(x_bf16: np.ndarray, scale: float):
    """Per-tensor calibrated scale -> (q int8 [M, K], a_scale fp32 [M])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty((M,), np.float32)
    _check(lib().w8a8o_quant_act_static(_p(x), M, K, K, float(np.float32(scale)), _p(q), _p(s)),
           "quant_act_static")
    return q, s


def unpack_int32(packed: np.ndarray, K: int) -> np.ndarray:
    """compressed-tensors int32 words [N, K/4] -> int8 [N, K]."""
    p = np.ascontiguousarray(packed, dtype=np.int32)
    N = p.shape[0]
    w = np.empty((N, K), np.int8)
    _check(lib().w8a8o_unpack_int32(_p(p), N, K, _p(w)), "unpack_int32")
    return w
