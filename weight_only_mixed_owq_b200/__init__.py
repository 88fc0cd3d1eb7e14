"""OWQ mixed-precision weight-only matmul for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library libowq_b200.so (include/owq.h); this package is its
ctypes binding.  Importing it fails loudly if the library has not been built.
"""
from .binding import (  # noqa: F401
    LIB, LIB_PATH, OWQ_OK, OwqError, OwqLayer, PROTOTYPES, STATUS_NAMES,
    owq_dequant, owq_device_status, owq_gemm, owq_gemv, owq_gemv_multi, owq_layer_bytes,
    owq_layer_free, owq_layer_info, owq_pack, owq_quantize, owq_status_string, owq_version,
    quantize, quantize_pack,
)
