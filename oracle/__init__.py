"""Float64 CPU oracle (test infrastructure only; never used by the product path).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline /
reference arm may import this package.  It shares no code with the CUDA path.
"""
from .paro_oracle import (AWQ_ORDER, awq_pack, awq_unpack, dequant, inverse_rotate,  # noqa: F401
                          normalize_group_size, rotate, w4_linear, w4_linear_columns,
                          w4_linear_from_codes)
