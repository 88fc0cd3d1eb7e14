"""OWQ mixed-precision weight-only matmul for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library libowq_b200.so (include/owq.h); this package is its
ctypes binding.  The binding is loaded on first use of any name below, and that first use
raises ImportError if the library has not been built (there is no fallback).  The build
script, `weight_only_mixed_owq_b200.build`, imports without the library.
"""
import importlib

_EXPORTS = (
    "LIB", "LIB_PATH", "OWQ_OK", "OWQ_INJECT_NONE", "OWQ_INJECT_GEMV_TAG", "OWQ_INJECT_GEMM_ARRIVE", "OWQ_INJECT_BOUNDS",
    "OwqError", "OwqLayer", "PROTOTYPES", "STATUS_NAMES",
    "owq_debug_inject", "owq_dequant", "owq_device_status", "owq_gemm", "owq_gemm_plan", "owq_gemv", "owq_gemv_multi", "owq_input_grad", "owq_layer_bytes",
    "owq_layer_free", "owq_layer_info", "owq_pack", "owq_pack_storage", "owq_quantize", "owq_quantize_noalloc", "owq_quantize_optq",
    "owq_optq", "owq_search_params", "owq_storage_pack", "owq_storage_unpack", "owq_storage_words",
    "owq_status_string", "owq_version", "owq_weak_grad", "quantize", "quantize_optq", "quantize_pack",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        binding = importlib.import_module(".binding", __name__)
        return getattr(binding, name)
    raise AttributeError(name)
