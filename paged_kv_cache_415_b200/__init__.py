"""Paged-KV-cache decode attention for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libpa.so`` (declared in include/pa.h):
``pa_reshape_and_cache``, ``pa_copy_blocks`` and ``pa_paged_decode``, all
hand-written CUDA.  ``binding`` wraps them for torch CUDA tensors (argument
marshalling only); ``step`` strings the three calls into one decode step.
Importing the package raises if libpa.so has not been built.
"""
from .binding import (  # noqa: F401
    PA_STATUS_BAD_BLOCK, PA_STATUS_BAD_CONTEXT, PA_STATUS_BAD_SLOT, PA_STATUS_COPY_CONFLICT,
    PA_STATUS_TIMEOUT, PAError, pa_copy_blocks, pa_paged_decode,
    pa_paged_decode_partition_size, pa_paged_decode_workspace_size, pa_reshape_and_cache,
    pa_status_string, pa_version)
from .step import DecodeStep  # noqa: F401
