"""B200-native per-group low-bit weight quantization and quantized linear layers.

The computation lives in ``libwq.so`` (C ABI, include/wq.h); this package holds the thin
ctypes binding (``wq_*`` functions, same names as the C calls), the build script and the
seeded synthetic-input generators (``synth``). Importing the package does not load the
library; the first ``wq_*`` call does, and raises if it is missing.
"""
from ._binding import (  # noqa: F401
    PATHS,
    SYMBOLS,
    PackJobs,
    WQError,
    lib,
    status_string,
    wq_dequantize,
    wq_device_status,
    wq_launch_count,
    wq_linear,
    wq_linear_workspace_bytes,
    wq_packed_bytes,
    wq_pd_search,
    wq_quant_error,
    wq_quant_error_many,
    wq_quantize_pack,
    wq_quantize_pack_many,
    wq_scales_count,
    wq_selftest_bounded_wait,
    wq_version,
)
