"""Thin ctypes binding of libpa.so: argument marshalling only.

Every function has the name of the C entry point it calls and takes torch
CUDA tensors (for device memory) plus the few host scalars the C call needs.
All arithmetic runs in the library's CUDA kernels; nothing here computes a
result, and there is no fallback: if libpa.so is missing or cannot be
loaded, importing this module raises.

Errors: a non-PA_OK return raises ``PAError`` carrying the status name.
Asynchronous data errors land in the optional ``d_status`` device int32
tensor (bits PA_STATUS_*).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA = 0, 1, 2, 3
PA_DTYPE_F16, PA_DTYPE_BF16, PA_DTYPE_FP8_E4M3, PA_DTYPE_INT8, PA_DTYPE_F32 = 0, 1, 2, 3, 4
PA_STATUS_BAD_BLOCK = 1
PA_STATUS_BAD_SLOT = 2
PA_STATUS_BAD_CONTEXT = 4
PA_STATUS_COPY_CONFLICT = 8
PA_STATUS_TIMEOUT = 16

_DTYPES = {torch.float16: PA_DTYPE_F16, torch.bfloat16: PA_DTYPE_BF16,
           torch.uint8: PA_DTYPE_FP8_E4M3, torch.float8_e4m3fn: PA_DTYPE_FP8_E4M3,
           torch.int8: PA_DTYPE_INT8, torch.float32: PA_DTYPE_F32}

# Every entry point declared in include/pa.h.
EXPORTS = ("pa_reshape_and_cache", "pa_copy_blocks", "pa_paged_decode_partition_size",
           "pa_paged_decode_workspace_size", "pa_paged_decode", "pa_paged_decode_no_alloc",
           "pa_paged_decode_shared_prefix_workspace_size", "pa_paged_decode_shared_prefix",
           "pa_paged_decode_append", "pa_reshape_and_cache_fp8", "pa_paged_decode_fp8",
           "pa_paged_decode_fp8_append", "pa_reshape_and_cache_int8", "pa_paged_decode_int8",
           "pa_paged_decode_int8_append", "pa_reshape_and_cache_fp8_rowscale",
           "pa_reshape_and_cache_int8_rowscale", "pa_paged_decode_fp8_rowscale",
           "pa_paged_decode_int8_rowscale", "pa_paged_decode_fp8_rowscale_append",
           "pa_paged_decode_int8_rowscale_append", "pa_swap_blocks",
           "pa_status_string", "pa_version")
# The test entry points declared in include/pa_selftest.h.
SELFTEST_EXPORTS = ("pa_selftest_bounded_wait", "pa_selftest_decode_abort",
                    "pa_selftest_shared_prefix_abort")
# Size of the library-owned scratch of pa_paged_decode_no_alloc (the
# PA_NO_ALLOC_WORKSPACE_BYTES of include/pa.h; a CPU test compares the two).
PA_NO_ALLOC_WORKSPACE_BYTES = 32 << 20


class PAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {pa_status_string(code)}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python -m paged_kv_cache_415_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    p, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    lib.pa_reshape_and_cache.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i32, p, p]
    lib.pa_reshape_and_cache.restype = i32
    lib.pa_copy_blocks.argtypes = [p, p, p, i32, i32, i32, i32, i64, i32, p, p]
    lib.pa_copy_blocks.restype = i32
    lib.pa_paged_decode_partition_size.argtypes = [i32] * 7
    lib.pa_paged_decode_partition_size.restype = i32
    lib.pa_paged_decode_workspace_size.argtypes = [i32] * 7
    lib.pa_paged_decode_workspace_size.restype = sz
    lib.pa_paged_decode.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64, i32, f32,
                                    i32, p, sz, i32, p, p]
    lib.pa_paged_decode.restype = i32
    lib.pa_paged_decode_no_alloc.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64,
                                             i32, f32, i32, i32, p, p]
    lib.pa_paged_decode_no_alloc.restype = i32
    lib.pa_paged_decode_shared_prefix_workspace_size.argtypes = [i32] * 9
    lib.pa_paged_decode_shared_prefix_workspace_size.restype = sz
    lib.pa_paged_decode_shared_prefix.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32,
                                                  i32, i32, i64, i32, i32, f32, i32, p, sz, i32,
                                                  p, p]
    lib.pa_paged_decode_shared_prefix.restype = i32
    lib.pa_paged_decode_append.argtypes = [p, p, p, p, p, p, p, p, i32, i32, i32, i32, i32, i32,
                                           i64, i32, f32, i32, p, sz, i32, p, p]
    lib.pa_paged_decode_append.restype = i32
    lib.pa_reshape_and_cache_fp8.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i32, f32,
                                             f32, p, p]
    lib.pa_reshape_and_cache_fp8.restype = i32
    lib.pa_paged_decode_fp8.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64, i32,
                                        f32, f32, f32, i32, p, sz, i32, p, p]
    lib.pa_paged_decode_fp8.restype = i32
    lib.pa_paged_decode_fp8_append.argtypes = [p, p, p, p, p, p, p, p, i32, i32, i32, i32, i32,
                                               i32, i64, i32, f32, f32, f32, i32, p, sz, i32, p, p]
    lib.pa_paged_decode_fp8_append.restype = i32
    lib.pa_reshape_and_cache_int8.argtypes = lib.pa_reshape_and_cache_fp8.argtypes
    lib.pa_reshape_and_cache_int8.restype = i32
    lib.pa_paged_decode_int8.argtypes = lib.pa_paged_decode_fp8.argtypes
    lib.pa_paged_decode_int8.restype = i32
    lib.pa_paged_decode_int8_append.argtypes = lib.pa_paged_decode_fp8_append.argtypes
    lib.pa_paged_decode_int8_append.restype = i32
    for fmt in ("fp8", "int8"):
        w = getattr(lib, f"pa_reshape_and_cache_{fmt}_rowscale")
        w.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i64, i32, p, p]
        w.restype = i32
        dcd = getattr(lib, f"pa_paged_decode_{fmt}_rowscale")
        dcd.argtypes = [p, p, p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64, i32, f32, i32,
                        p, sz, i32, p, p]
        dcd.restype = i32
        app = getattr(lib, f"pa_paged_decode_{fmt}_rowscale_append")
        app.argtypes = [p, p, p, p, p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64, i32, f32,
                        i32, p, sz, i32, p, p]
        app.restype = i32
    lib.pa_swap_blocks.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i64, i32, p, p]
    lib.pa_swap_blocks.restype = i32
    lib.pa_selftest_bounded_wait.argtypes = [p, p, ctypes.c_uint32, i32, p]
    lib.pa_selftest_bounded_wait.restype = i32
    lib.pa_selftest_decode_abort.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64,
                                             i32, f32, i32, p, sz, i32, i32, ctypes.c_uint32, p,
                                             p]
    lib.pa_selftest_decode_abort.restype = i32
    lib.pa_selftest_shared_prefix_abort.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32,
                                                    i32, i32, i64, i32, i32, f32, i32, p, sz, i32,
                                                    ctypes.c_uint32, p, p]
    lib.pa_selftest_shared_prefix_abort.restype = i32
    lib.pa_status_string.argtypes = [i32]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = ctypes.c_char_p
    return lib


LIB = _load()


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        return 99          # rejected by the library as PA_ERR_UNSUPPORTED


def _check(fn: str, code: int) -> None:
    if code != PA_OK:
        raise PAError(fn, code)


def pa_status_string(code: int) -> str:
    return LIB.pa_status_string(int(code)).decode()


def pa_version() -> str:
    return LIB.pa_version().decode()


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, d_status=None,
                         stream=None) -> None:
    """key/value [T][Hkv][D]; k_cache/v_cache [num_blocks][B][Hkv][D];
    slot_mapping int64 [T]."""
    num_blocks, block_size, hkv, d = k_cache.shape
    _check("pa_reshape_and_cache", LIB.pa_reshape_and_cache(
        _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
        int(slot_mapping.shape[0]), hkv, d, block_size, num_blocks, _dtype(k_cache),
        _ptr(d_status), _stream(stream)))


def pa_copy_blocks(k_cache, v_cache, block_mapping, d_status=None, stream=None) -> None:
    """block_mapping int64 [P][2] of (src, dst) block ids, on the device."""
    num_blocks, block_size, hkv, d = k_cache.shape
    _check("pa_copy_blocks", LIB.pa_copy_blocks(
        _ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), int(block_mapping.shape[0]), hkv, d,
        block_size, num_blocks, _dtype(k_cache), _ptr(d_status), _stream(stream)))


def pa_paged_decode_partition_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                   max_context_len, partition_size=0) -> int:
    return int(LIB.pa_paged_decode_partition_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                  block_size, max_context_len, partition_size))


def pa_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                   max_context_len, partition_size=0) -> int:
    return int(LIB.pa_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                  block_size, max_context_len, partition_size))


def pa_paged_decode(out, query, k_cache, v_cache, block_tables, context_lens, max_context_len,
                    scale, partition_size=0, workspace=None, d_status=None, stream=None) -> None:
    """out/query [S][Hq][D]; k_cache/v_cache [num_blocks][B][Hkv][D];
    block_tables int32 [S][max_blocks_per_seq]; context_lens int32 [S];
    workspace: a uint8 device tensor of at least
    pa_paged_decode_workspace_size(...) bytes (or None when that is 0)."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_paged_decode", LIB.pa_paged_decode(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), num_seqs, hq, hkv, d, block_size, int(block_tables.shape[1]),
        num_blocks, int(max_context_len), float(scale), int(partition_size), _ptr(workspace),
        ws_bytes, _dtype(query), _ptr(d_status), _stream(stream)))


def pa_paged_decode_no_alloc(out, query, k_cache, v_cache, block_tables, context_lens,
                             max_context_len, scale, partition_size=0, d_status=None,
                             stream=None) -> None:
    """pa_paged_decode for callers that cannot allocate device memory: the
    split-context scratch is the library's own fixed array of
    PA_NO_ALLOC_WORKSPACE_BYTES per GPU.  Shapes needing more raise PAError
    (PA_ERR_INVALID_ARG) before any work is enqueued.  Calls share that
    array, so calls that overlap on the GPU must not be issued."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    _check("pa_paged_decode_no_alloc", LIB.pa_paged_decode_no_alloc(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), num_seqs, hq, hkv, d, block_size, int(block_tables.shape[1]),
        num_blocks, int(max_context_len), float(scale), int(partition_size), _dtype(query),
        _ptr(d_status), _stream(stream)))


def pa_paged_decode_shared_prefix_workspace_size(num_seqs, group_size, num_q_heads, num_kv_heads,
                                                 head_dim, block_size, max_context_len,
                                                 max_prefix_len, partition_size=0) -> int:
    return int(LIB.pa_paged_decode_shared_prefix_workspace_size(
        num_seqs, group_size, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
        max_prefix_len, partition_size))


def pa_paged_decode_shared_prefix(out, query, k_cache, v_cache, block_tables, context_lens,
                                  prefix_lens, group_size, max_context_len, max_prefix_len, scale,
                                  workspace, partition_size=0, d_status=None, stream=None) -> None:
    """pa_paged_decode for groups of group_size consecutive sequences that
    share their first prefix_lens[g] tokens (int32 device tensor, one entry
    per group, whole blocks).  workspace may be None when
    pa_paged_decode_shared_prefix_workspace_size(...) is 0."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_paged_decode_shared_prefix", LIB.pa_paged_decode_shared_prefix(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), _ptr(prefix_lens), num_seqs, int(group_size), hq, hkv, d, block_size,
        int(block_tables.shape[1]), num_blocks, int(max_context_len), int(max_prefix_len),
        float(scale), int(partition_size), _ptr(workspace), ws_bytes, _dtype(query),
        _ptr(d_status), _stream(stream)))


def pa_paged_decode_append(out, query, key, value, k_cache, v_cache, block_tables, context_lens,
                           max_context_len, scale, partition_size=0, workspace=None,
                           d_status=None, stream=None) -> None:
    """One decode step in one launch: key/value [S][Hkv][D] hold each
    sequence's new token (position context_lens[s] - 1, slot from its block
    table); it is written into k_cache/v_cache and attended to."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_paged_decode_append", LIB.pa_paged_decode_append(
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), _ptr(context_lens), num_seqs, hq, hkv, d, block_size,
        int(block_tables.shape[1]), num_blocks, int(max_context_len), float(scale),
        int(partition_size), _ptr(workspace), ws_bytes, _dtype(query), _ptr(d_status),
        _stream(stream)))


def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             d_status=None, stream=None) -> None:
    """Quantising cache write: key/value [T][Hkv][D] (fp16/bf16) into e4m3
    pools k_cache/v_cache [num_blocks][B][Hkv][D] (uint8 tensors)."""
    num_blocks, block_size, hkv, d = k_cache.shape
    _check("pa_reshape_and_cache_fp8", LIB.pa_reshape_and_cache_fp8(
        _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
        int(slot_mapping.shape[0]), hkv, d, block_size, num_blocks, _dtype(key), float(k_scale),
        float(v_scale), _ptr(d_status), _stream(stream)))


def pa_paged_decode_fp8(out, query, k_cache, v_cache, block_tables, context_lens, max_context_len,
                        scale, k_scale, v_scale, partition_size=0, workspace=None, d_status=None,
                        stream=None) -> None:
    """pa_paged_decode over e4m3 pools (uint8 tensors) with per-pool scales."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_paged_decode_fp8", LIB.pa_paged_decode_fp8(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), num_seqs, hq, hkv, d, block_size, int(block_tables.shape[1]),
        num_blocks, int(max_context_len), float(scale), float(k_scale), float(v_scale),
        int(partition_size), _ptr(workspace), ws_bytes, _dtype(query), _ptr(d_status),
        _stream(stream)))


def pa_paged_decode_fp8_append(out, query, key, value, k_cache, v_cache, block_tables,
                               context_lens, max_context_len, scale, k_scale, v_scale,
                               partition_size=0, workspace=None, d_status=None,
                               stream=None) -> None:
    """pa_paged_decode_fp8 with each sequence's new token (key/value
    [S][Hkv][D], fp16/bf16) quantised into its slot inside the launch."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_paged_decode_fp8_append", LIB.pa_paged_decode_fp8_append(
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), _ptr(context_lens), num_seqs, hq, hkv, d, block_size,
        int(block_tables.shape[1]), num_blocks, int(max_context_len), float(scale),
        float(k_scale), float(v_scale), int(partition_size), _ptr(workspace), ws_bytes,
        _dtype(query), _ptr(d_status), _stream(stream)))

def pa_reshape_and_cache_int8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                              d_status=None, stream=None) -> None:
    """Quantising cache write: key/value [T][Hkv][D] (fp16/bf16) into int8
    pools k_cache/v_cache [num_blocks][B][Hkv][D] (int8 tensors)."""
    num_blocks, block_size, hkv, d = k_cache.shape
    _check("pa_reshape_and_cache_int8", LIB.pa_reshape_and_cache_int8(
        _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
        int(slot_mapping.shape[0]), hkv, d, block_size, num_blocks, _dtype(key), float(k_scale),
        float(v_scale), _ptr(d_status), _stream(stream)))


def pa_paged_decode_int8(out, query, k_cache, v_cache, block_tables, context_lens,
                         max_context_len, scale, k_scale, v_scale, partition_size=0,
                         workspace=None, d_status=None, stream=None) -> None:
    """pa_paged_decode over int8 pools (int8 tensors) with per-pool scales."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_paged_decode_int8", LIB.pa_paged_decode_int8(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), num_seqs, hq, hkv, d, block_size, int(block_tables.shape[1]),
        num_blocks, int(max_context_len), float(scale), float(k_scale), float(v_scale),
        int(partition_size), _ptr(workspace), ws_bytes, _dtype(query), _ptr(d_status),
        _stream(stream)))


def pa_paged_decode_int8_append(out, query, key, value, k_cache, v_cache, block_tables,
                                context_lens, max_context_len, scale, k_scale, v_scale,
                                partition_size=0, workspace=None, d_status=None,
                                stream=None) -> None:
    """pa_paged_decode_int8 with each sequence's new token (key/value
    [S][Hkv][D], fp16/bf16) quantised into its slot inside the launch."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_paged_decode_int8_append", LIB.pa_paged_decode_int8_append(
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), _ptr(context_lens), num_seqs, hq, hkv, d, block_size,
        int(block_tables.shape[1]), num_blocks, int(max_context_len), float(scale),
        float(k_scale), float(v_scale), int(partition_size), _ptr(workspace), ws_bytes,
        _dtype(query), _ptr(d_status), _stream(stream)))


# ---------------------------------------------------------------------------
# Row-scaled one-byte pools: codes [num_blocks][B][Hkv][D] (uint8 e4m3 or
# int8) and fp32 scales [num_blocks][Hkv][B], one per (token, kv head) row
# ---------------------------------------------------------------------------

def _rowscale_write(fmt, key, value, k_cache, v_cache, k_scales, v_scales, slot_mapping,
                    d_status=None, stream=None) -> None:
    num_blocks, block_size, hkv, d = k_cache.shape
    fn = f"pa_reshape_and_cache_{fmt}_rowscale"
    _check(fn, getattr(LIB, fn)(
        _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(k_scales), _ptr(v_scales),
        _ptr(slot_mapping), int(slot_mapping.shape[0]), hkv, d, block_size, num_blocks,
        _dtype(key), _ptr(d_status), _stream(stream)))


def pa_reshape_and_cache_fp8_rowscale(key, value, k_cache, v_cache, k_scales, v_scales,
                                      slot_mapping, d_status=None, stream=None) -> None:
    """Quantising write into e4m3 pools with one scale per row:
    s = max |x| / 448 stored in k_scales / v_scales [num_blocks][Hkv][B]."""
    _rowscale_write("fp8", key, value, k_cache, v_cache, k_scales, v_scales, slot_mapping,
                    d_status, stream)


def pa_reshape_and_cache_int8_rowscale(key, value, k_cache, v_cache, k_scales, v_scales,
                                       slot_mapping, d_status=None, stream=None) -> None:
    """As pa_reshape_and_cache_fp8_rowscale into int8 pools (s = max |x| / 127)."""
    _rowscale_write("int8", key, value, k_cache, v_cache, k_scales, v_scales, slot_mapping,
                    d_status, stream)


def _rowscale_decode(fmt, out, query, k_cache, v_cache, k_scales, v_scales, block_tables,
                     context_lens, max_context_len, scale, partition_size, workspace, d_status,
                     stream) -> None:
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = f"pa_paged_decode_{fmt}_rowscale"
    _check(fn, getattr(LIB, fn)(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(k_scales), _ptr(v_scales),
        _ptr(block_tables), _ptr(context_lens), num_seqs, hq, hkv, d, block_size,
        int(block_tables.shape[1]), num_blocks, int(max_context_len), float(scale),
        int(partition_size), _ptr(workspace), ws_bytes, _dtype(query), _ptr(d_status),
        _stream(stream)))


def pa_paged_decode_fp8_rowscale(out, query, k_cache, v_cache, k_scales, v_scales, block_tables,
                                 context_lens, max_context_len, scale, partition_size=0,
                                 workspace=None, d_status=None, stream=None) -> None:
    """pa_paged_decode over e4m3 pools with one scale per row."""
    _rowscale_decode("fp8", out, query, k_cache, v_cache, k_scales, v_scales, block_tables,
                     context_lens, max_context_len, scale, partition_size, workspace, d_status,
                     stream)


def pa_paged_decode_int8_rowscale(out, query, k_cache, v_cache, k_scales, v_scales, block_tables,
                                  context_lens, max_context_len, scale, partition_size=0,
                                  workspace=None, d_status=None, stream=None) -> None:
    """pa_paged_decode over int8 pools with one scale per row."""
    _rowscale_decode("int8", out, query, k_cache, v_cache, k_scales, v_scales, block_tables,
                     context_lens, max_context_len, scale, partition_size, workspace, d_status,
                     stream)


def _rowscale_append(fmt, out, query, key, value, k_cache, v_cache, k_scales, v_scales,
                     block_tables, context_lens, max_context_len, scale, partition_size,
                     workspace, d_status, stream) -> None:
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = f"pa_paged_decode_{fmt}_rowscale_append"
    _check(fn, getattr(LIB, fn)(
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
        _ptr(k_scales), _ptr(v_scales), _ptr(block_tables), _ptr(context_lens), num_seqs, hq,
        hkv, d, block_size, int(block_tables.shape[1]), num_blocks, int(max_context_len),
        float(scale), int(partition_size), _ptr(workspace), ws_bytes, _dtype(query),
        _ptr(d_status), _stream(stream)))


def pa_paged_decode_fp8_rowscale_append(out, query, key, value, k_cache, v_cache, k_scales,
                                        v_scales, block_tables, context_lens, max_context_len,
                                        scale, partition_size=0, workspace=None, d_status=None,
                                        stream=None) -> None:
    """pa_paged_decode_fp8_rowscale with each sequence's new token quantised
    (codes and row scales) into its slot inside the launch."""
    _rowscale_append("fp8", out, query, key, value, k_cache, v_cache, k_scales, v_scales,
                     block_tables, context_lens, max_context_len, scale, partition_size,
                     workspace, d_status, stream)


def pa_paged_decode_int8_rowscale_append(out, query, key, value, k_cache, v_cache, k_scales,
                                         v_scales, block_tables, context_lens, max_context_len,
                                         scale, partition_size=0, workspace=None, d_status=None,
                                         stream=None) -> None:
    """pa_paged_decode_int8_rowscale with the fused row-scaled cache write."""
    _rowscale_append("int8", out, query, key, value, k_cache, v_cache, k_scales, v_scales,
                     block_tables, context_lens, max_context_len, scale, partition_size,
                     workspace, d_status, stream)


def pa_copy_block_scales(k_scales, v_scales, block_mapping, d_status=None, stream=None) -> None:
    """pa_copy_blocks over the row-scale pools [num_blocks][Hkv][B] (fp32):
    the scales of each (src, dst) block move with its codes."""
    num_blocks, hkv, block_size = k_scales.shape
    _check("pa_copy_blocks", LIB.pa_copy_blocks(
        _ptr(k_scales), _ptr(v_scales), _ptr(block_mapping), int(block_mapping.shape[0]), hkv,
        1, block_size, num_blocks, PA_DTYPE_F32, _ptr(d_status), _stream(stream)))


def _addr(t) -> int:
    """Device-usable address of a CUDA tensor or a pinned host tensor (on a
    system with unified addressing the pinned host pointer is the device
    pointer)."""
    if t is None:
        return None
    if not t.is_cuda and not t.is_pinned():
        raise ValueError("host pools must be pinned memory")
    return t.data_ptr()


def pa_swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, d_status=None, stream=None) -> None:
    """Whole-block copies src -> dst between two pools (one of them usually
    a pinned host tensor): block_mapping int64 [P][2] of (src, dst) ids.
    Pools are [num_blocks][B][Hkv][D], or fp32 row-scale pools
    [num_blocks][Hkv][B] (moved as PA_DTYPE_F32 with head_dim 1)."""
    if src_k.dim() == 3:
        src_nb, hkv, block_size = src_k.shape
        d = 1
    else:
        src_nb, block_size, hkv, d = src_k.shape
    dst_nb = dst_k.shape[0]
    _check("pa_swap_blocks", LIB.pa_swap_blocks(
        _addr(src_k), _addr(src_v), _addr(dst_k), _addr(dst_v), _addr(block_mapping),
        int(block_mapping.shape[0]), hkv, d, block_size, src_nb, dst_nb, _dtype(src_k),
        _ptr(d_status), _stream(stream)))


# ---------------------------------------------------------------------------
# Test entry points of the bounded waits (include/pa_selftest.h)
# ---------------------------------------------------------------------------

def pa_selftest_bounded_wait(d_status, wait_limit_us, num_ctas=1, d_wait_ns=None,
                             stream=None) -> None:
    """num_ctas CTAs wait on an mbarrier nothing arrives on, bounded by
    wait_limit_us; each warp that gives up sets PA_STATUS_TIMEOUT in
    d_status.  d_wait_ns (int64 [num_ctas], optional) gets each CTA's wait."""
    _check("pa_selftest_bounded_wait", LIB.pa_selftest_bounded_wait(
        _ptr(d_status), _ptr(d_wait_ns), int(wait_limit_us), int(num_ctas), _stream(stream)))


def pa_selftest_decode_abort(out, query, k_cache, v_cache, block_tables, context_lens,
                             max_context_len, scale, wait_limit_us, partition_size=0,
                             workspace=None, d_status=None, stream=None) -> None:
    """pa_paged_decode (16-bit pools) or the e4m3 / int8 decode (uint8 / int8
    pools, scales 1) with every warp's first wait sent to an mbarrier that
    nothing completes: the abort path of a timed-out copy runs in every CTA."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_selftest_decode_abort", LIB.pa_selftest_decode_abort(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), num_seqs, hq, hkv, d, block_size, int(block_tables.shape[1]),
        num_blocks, int(max_context_len), float(scale), int(partition_size), _ptr(workspace),
        ws_bytes, _dtype(query), _dtype(k_cache), int(wait_limit_us), _ptr(d_status),
        _stream(stream)))


def pa_selftest_shared_prefix_abort(out, query, k_cache, v_cache, block_tables, context_lens,
                                    prefix_lens, group_size, max_context_len, max_prefix_len,
                                    scale, workspace, wait_limit_us, partition_size=0,
                                    d_status=None, stream=None) -> None:
    """pa_paged_decode_shared_prefix with every warp's first wait sent to an
    mbarrier that nothing completes."""
    num_seqs, hq, d = query.shape
    num_blocks, block_size, hkv, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_selftest_shared_prefix_abort", LIB.pa_selftest_shared_prefix_abort(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), _ptr(prefix_lens), num_seqs, int(group_size), hq, hkv, d, block_size,
        int(block_tables.shape[1]), num_blocks, int(max_context_len), int(max_prefix_len),
        float(scale), int(partition_size), _ptr(workspace), ws_bytes, _dtype(query),
        int(wait_limit_us), _ptr(d_status), _stream(stream)))
