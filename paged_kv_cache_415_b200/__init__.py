"""Paged-KV-cache decode attention for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libpa.so`` (declared in include/pa.h):
``pa_reshape_and_cache``, ``pa_copy_blocks`` and ``pa_paged_decode`` (plus
``pa_paged_decode_no_alloc``), all hand-written CUDA.  ``binding`` wraps them
for torch CUDA tensors (argument marshalling only); ``step`` strings the
calls into one decode step; ``build`` compiles the library.

The binding is loaded on first use of any of its names and raises if
libpa.so has not been built: there is no fallback.
"""
import importlib

_BINDING_NAMES = {
    "PA_STATUS_BAD_BLOCK", "PA_STATUS_BAD_CONTEXT", "PA_STATUS_BAD_SLOT",
    "PA_STATUS_COPY_CONFLICT", "PA_STATUS_TIMEOUT", "PA_NO_ALLOC_WORKSPACE_BYTES", "PAError",
    "pa_copy_blocks", "pa_paged_decode", "pa_paged_decode_no_alloc",
    "pa_paged_decode_shared_prefix", "pa_paged_decode_shared_prefix_workspace_size",
    "pa_paged_decode_append", "pa_reshape_and_cache_fp8", "pa_paged_decode_fp8",
    "pa_paged_decode_fp8_append", "pa_reshape_and_cache_int8", "pa_paged_decode_int8",
    "pa_paged_decode_int8_append", "pa_swap_blocks",
    "pa_paged_decode_partition_size", "pa_paged_decode_workspace_size", "pa_reshape_and_cache",
    "pa_status_string", "pa_version",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(importlib.import_module(".binding", __name__), name)
    if name == "DecodeStep":
        return importlib.import_module(".step", __name__).DecodeStep
    raise AttributeError(name)
