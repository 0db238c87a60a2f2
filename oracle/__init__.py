"""Float64 CPU oracle (test infrastructure only; never used by the product path).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline /
reference arm may import this package.  It shares no code with the CUDA path.
"""
from .paro_oracle import (AWQ_ORDER, QSCALE_MAX, QSCALE_MIN, SYM_QMAX, SYM_QMIN,  # noqa: F401
                          SYM_ZERO_CODE, awq_pack, awq_unpack, dequant, inverse_rotate,
                          normalize_group_size, quantize_sym4, quantize_weight, rotate,
                          transform_weight, w4_linear, w4_linear_columns, w4_linear_from_codes,
                          moe_linear_from_codes)
