"""W8A8 int8-dynamic linear layer for NVIDIA B200 (sm_100a).

The layer: per-token symmetric int8 quantization of bf16 activations, an
int8 x int8 -> int32 GEMM against per-output-channel int8 weights on the
tcgen05 tensor cores (or a streaming GEMV for M <= 16), and a fused fp32
dequantization/bias epilogue producing bf16.  The kernels live in
``libw8a8.so`` (C ABI: ``include/w8a8.h``); this package is its binding.
"""
from .binding import (  # noqa: F401
    LIB_PATH, VARIANT_AUTO, VARIANT_GEMM_BN64, VARIANT_GEMM_BN128, VARIANT_GEMM_BN256,
    VARIANT_GEMM_PAIR, VARIANT_GEMV, VARIANT_GEMV_TC,
    W8A8Error, last_device_error, lib, linear, linear_fused, linear_fused_host, quant_act,
    quantize_weights, select, selftest_bounded_wait, status_string, unpack_int32_weights, version,
    w8a16_linear, workspace_size,
)
