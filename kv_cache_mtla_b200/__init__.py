"""B200-native (sm_100a) MTLA attention hot path.

``mtla`` is the Python binding of libmtla.so (C ABI in include/mtla.h);
``inputs`` draws the seeded synthetic workloads.
"""
from . import inputs  # noqa: F401
from .mtla import (  # noqa: F401
    BF16, FP32, GATE_COMPUTED, GATE_SUPPLIED, GATE_UNIT, Buffers, Config, MtlaError,
    decode_step, get_device_status, kernel_launches, load, make_config, prefill, status_string,
    workspace_size,
)
