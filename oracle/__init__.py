"""CPU oracle (test infrastructure only; see :mod:`oracle.glmq_oracle`)."""
from .glmq_oracle import (  # noqa: F401
    divisor,
    row_absmax,
    row_scale,
    quantize_rows,
    pack_int4,
    pack,
    quantize_linear,
    unpack,
    dequantize,
    linear_forward,
    linear_forward_rows,
    relative_max_error,
)
from .glmq_epilogue import (  # noqa: F401,E402
    linear_pre,
    linear_bias_forward,
    gelu,
    geglu_forward,
    geglu_row_order,
    quantize_linear_geglu,
)
from .glmq_zeropoint import (  # noqa: F401,E402
    zp_range,
    zp_scale,
    zp_zero,
    zp_codes,
    pack_u4,
    unpack_u4,
    quantize_linear_zp,
    dequantize_zp,
    linear_forward_zp,
)
