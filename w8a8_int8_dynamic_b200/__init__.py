"""B200-native W8A8 int8-dynamic linear layers.

Dynamic per-token symmetric int8 activation quantisation, a load-time weight
repack into tensor-core tile images, and int8 x int8 -> int32 GEMMs on the
sm_100a tensor cores (tcgen05, TMEM accumulators) with a dequantising bf16
epilogue -- exposed as the C ABI of libw8a8.so (include/w8a8.h) and bound here
with ctypes.  The library is loaded on first use; there is no CPU fallback.
"""
from .binding import (  # noqa: F401
    ACT_GELU_TANH, ACT_NONE, PATH_AUTO, PATH_LARGE, PATH_LARGE_BN128, PATH_LARGE_BN256, PATH_LARGE_PAIR, PATH_LARGE_PAIR128,
    PATH_SMALL, W8A8Error, W8A8Linear,
    gelu_tanh, gemm_kernel_name, launch_count, lib, linear, linear_act_quant,
    linear_act_quant_workspace_bytes, linear_workspace_bytes, pack_weight, pack_weight_int32, packed_weight_bytes,
    poll_status, quant_act, quant_act_static, quant_pack_weight, scaled_mm, scaled_mm_i32, scaled_mm_workspace_bytes, selftest_int8_mma_rate, selftest_wait_timeout,
    set_path, unpack_weight)
