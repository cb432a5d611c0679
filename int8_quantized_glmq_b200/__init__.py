"""B200-native weight-only INT4/INT8 quantization and W4A16/W8A16 GEMM for GLM-130B shapes.

The compute lives in ``libglmq.so`` (CUDA C++ for sm_100a, C ABI in
``include/glmq.h``); this package is its Python binding.
"""
from ._binding import (  # noqa: F401
    DECODE_MAX_M,
    EPILOGUE_GEGLU,
    EPILOGUE_NONE,
    MAX_K,
    GlmqError,
    abi_version,
    gemm,
    gemm_fused,
    gemm_zp,
    gemm_decode,
    gemm_decode_prefetch,
    gemm_prefill,
    kernel_launches,
    last_device_error,
    lib,
    packed_bytes,
    quantize,
    quantize_zp,
    raw_gemm,
    raw_quantize,
    set_wait_limit_ns,
    status_string,
)
