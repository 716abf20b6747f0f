"""fp64 CPU oracle for the paged-KV-cache decode path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``paged_kv_cache_415_b200``) never imports it and shares no code with it.

``pa_oracle.c`` holds the definitions (reshape_and_cache, copy_blocks,
swap_blocks, paged decode in fp64; the e4m3 and int8 pools' encode, write and
decode, with one scale per pool or one per (token, kv head) row); this module compiles it with gcc (``-O2``, OpenMP, no
fast-math) into ``liboracle.so`` beside it and wraps it with ctypes.
``brute.py`` holds pure-Python/numpy restatements used to pin it.

Arrays are numpy: fp16/bf16 tensors are passed as their raw ``uint16`` bit
patterns together with a dtype name ("f16" or "bf16").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_DTYPES = {"f16": 0, "bf16": 1}
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle source into a shared library (gcc -O2 -fopenmp)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-Wall", "-Wextra", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """ctypes handle of the oracle library (the default build, or ``path``:
    the tests load deliberately broken variants to check that the pins
    catch them)."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(build() if path is None else path)
    p = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    lib.oracle_decode_bits.argtypes = [p, p, i64, i32]
    lib.oracle_decode_bits.restype = None
    lib.oracle_reshape_and_cache.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64]
    lib.oracle_reshape_and_cache.restype = i32
    lib.oracle_copy_blocks.argtypes = [p, p, p, i32, i32, i32, i32, i64]
    lib.oracle_copy_blocks.restype = i32
    lib.oracle_swap_blocks.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i64, i32]
    lib.oracle_swap_blocks.restype = i32
    lib.oracle_paged_decode.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64,
                                        f64, i32, i32, i32]
    lib.oracle_paged_decode.restype = i32
    lib.oracle_paged_decode_rows.argtypes = [p, p, i32, p, p, p, p, p, i32, i32, i32, i32,
                                             i32, i64, f64, i32, i32]
    lib.oracle_paged_decode_rows.restype = i32
    lib.oracle_decode_e4m3.argtypes = [p, p, i64]
    lib.oracle_decode_e4m3.restype = None
    lib.oracle_encode_e4m3.argtypes = [p, p, i64]
    lib.oracle_encode_e4m3.restype = None
    lib.oracle_reshape_and_cache_fp8.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i32,
                                                 ctypes.c_float, ctypes.c_float]
    lib.oracle_reshape_and_cache_fp8.restype = i32
    lib.oracle_paged_decode_fp8.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64,
                                            f64, i32, f64, f64, i32]
    lib.oracle_paged_decode_fp8.restype = i32
    lib.oracle_decode_int8.argtypes = [p, p, i64]
    lib.oracle_decode_int8.restype = None
    lib.oracle_encode_int8.argtypes = [p, p, i64]
    lib.oracle_encode_int8.restype = None
    lib.oracle_reshape_and_cache_int8.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i32,
                                                  ctypes.c_float, ctypes.c_float]
    lib.oracle_reshape_and_cache_int8.restype = i32
    lib.oracle_paged_decode_int8.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32,
                                             i64, f64, i32, f64, f64, i32]
    lib.oracle_paged_decode_int8.restype = i32
    for fmt in ("fp8", "int8"):
        w = getattr(lib, f"oracle_reshape_and_cache_{fmt}_rowscale")
        w.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i64, i32]
        w.restype = i32
        dcd = getattr(lib, f"oracle_paged_decode_{fmt}_rowscale")
        dcd.argtypes = [p, p, p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i64, f64, i32, i32]
        dcd.restype = i32
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = i32
    if path is None:
        _lib = lib
    return lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _u16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16, f"expected 16-bit patterns, got {a.dtype}"
    return a


def max_threads(lib=None) -> int:
    return int((lib or load()).oracle_max_threads())


def decode_bits(bits: np.ndarray, dtype: str, lib=None) -> np.ndarray:
    """Exact fp16/bf16 bit pattern -> float64."""
    bits = _u16(bits)
    out = np.empty(bits.shape, dtype=np.float64)
    (lib or load()).oracle_decode_bits(_ptr(bits), _ptr(out), bits.size, _DTYPES[dtype])
    return out


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, block_size, lib=None) -> int:
    """In place on k_cache / v_cache ([num_blocks][block_size][Hkv][D] uint16).

    key/value: [T][Hkv][D]; slot_mapping int64 [T].  Returns status bits."""
    key, value = _u16(key), _u16(value)
    assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    num_blocks, bs, hkv, d = k_cache.shape
    assert bs == block_size
    return int((lib or load()).oracle_reshape_and_cache(
        _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
        key.shape[0], hkv, d, block_size, num_blocks))


def copy_blocks(k_cache, v_cache, block_mapping, lib=None) -> int:
    """In place: for each (src, dst) row of block_mapping, copy block src to dst.

    Pools of 16-bit elements, or of one-byte codes (uint8 / int8, head_dim
    even), which move as the same bytes seen in pairs."""
    block_mapping = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    assert k_cache.dtype == v_cache.dtype and k_cache.shape == v_cache.shape
    assert k_cache.flags["C_CONTIGUOUS"] and v_cache.flags["C_CONTIGUOUS"]
    if k_cache.dtype.itemsize == 1:
        assert k_cache.shape[-1] % 2 == 0, "one-byte pools copy as byte pairs"
        k_cache, v_cache = k_cache.view(np.uint16), v_cache.view(np.uint16)
    elif k_cache.dtype == np.float32:
        # row-scale pools [num_blocks][Hkv][B]: a block is Hkv * B scales, copied as 16-bit pairs
        nb = k_cache.shape[0]
        k_cache = k_cache.view(np.uint16).reshape(nb, 1, 1, -1)
        v_cache = v_cache.view(np.uint16).reshape(nb, 1, 1, -1)
    assert k_cache.dtype.itemsize == 2, f"16-bit or one-byte pools, got {k_cache.dtype}"
    num_blocks, bs, hkv, d = k_cache.shape
    return int((lib or load()).oracle_copy_blocks(
        _ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), block_mapping.shape[0],
        hkv, d, bs, num_blocks))


def swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, lib=None) -> int:
    """In place on dst: for each (src, dst) row of block_mapping, block src of
    the source pools becomes block dst of the destination pools (raw bytes;
    pools of any one element type, [num_blocks][B][Hkv][D])."""
    block_mapping = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    assert src_k.dtype == dst_k.dtype and src_k.shape[1:] == dst_k.shape[1:]
    if src_k.ndim == 3:                  # row-scale pools [num_blocks][Hkv][B]: bytes of a block
        src_k, src_v, dst_k, dst_v = (a.reshape(a.shape[0], 1, 1, -1)
                                      for a in (src_k, src_v, dst_k, dst_v))
    for a in (src_k, src_v, dst_k, dst_v):
        assert a.flags["C_CONTIGUOUS"]
    src_nb, bs, hkv, d = src_k.shape
    return int((lib or load()).oracle_swap_blocks(
        _ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v), _ptr(block_mapping),
        block_mapping.shape[0], hkv, d, bs, src_nb, dst_k.shape[0], src_k.dtype.itemsize))


def paged_decode(query, k_cache, v_cache, block_tables, context_lens, scale, dtype,
                 blocked=False, num_threads=0, lib=None):
    """fp64 paged decode attention.  Returns (out [S][Hq][D] float64, status)."""
    query = _u16(query)
    k_cache, v_cache = _u16(k_cache), _u16(v_cache)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    s, hq, d = query.shape
    num_blocks, bs, hkv, d2 = k_cache.shape
    assert d2 == d
    out = np.empty((s, hq, d), dtype=np.float64)
    st = (lib or load()).oracle_paged_decode(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), s, hq, hkv, d, bs, block_tables.shape[1], num_blocks,
        float(scale), _DTYPES[dtype], 1 if blocked else 0, num_threads)
    return out, int(st)


def paged_decode_rows(rows, query, k_cache, v_cache, block_tables, context_lens, scale, dtype,
                      num_threads=0, lib=None):
    """fp64 paged decode for selected (sequence, query head) rows only.

    rows: int [n][2].  Returns (out [n][D] float64, status)."""
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 2)
    query = _u16(query)
    k_cache, v_cache = _u16(k_cache), _u16(v_cache)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    s, hq, d = query.shape
    num_blocks, bs, hkv, _ = k_cache.shape
    out = np.empty((rows.shape[0], d), dtype=np.float64)
    st = (lib or load()).oracle_paged_decode_rows(
        _ptr(out), _ptr(rows), rows.shape[0], _ptr(query), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), _ptr(context_lens), hq, hkv, d, bs, block_tables.shape[1],
        num_blocks, float(scale), _DTYPES[dtype], num_threads)
    return out, int(st)


# ---- FP8 (e4m3) caches: uint8 codes, per-tensor scales ------------------------

def decode_e4m3(codes: np.ndarray, lib=None) -> np.ndarray:
    """e4m3 code -> float64 (exact; 0x7F / 0xFF -> NaN)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    (lib or load()).oracle_decode_e4m3(_ptr(codes), _ptr(out), codes.size)
    return out


def encode_e4m3(x: np.ndarray, lib=None) -> np.ndarray:
    """float32 -> e4m3 code, round to nearest even, saturating at +-448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    (lib or load()).oracle_encode_e4m3(_ptr(x), _ptr(out), x.size)
    return out


def _code_bytes(a: np.ndarray) -> np.ndarray:
    """An 8-bit pool (uint8 or int8) as contiguous raw bytes."""
    a = np.ascontiguousarray(a)
    assert a.dtype in (np.uint8, np.int8), f"expected 8-bit codes, got {a.dtype}"
    return a.view(np.uint8)


def _reshape_and_cache_q8(fn, key, value, k_cache, v_cache, slot_mapping, block_size, dtype,
                          k_scale, v_scale):
    key, value = _u16(key), _u16(value)
    assert k_cache.dtype in (np.uint8, np.int8) and v_cache.dtype == k_cache.dtype
    assert k_cache.flags["C_CONTIGUOUS"] and v_cache.flags["C_CONTIGUOUS"]
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    num_blocks, bs, hkv, d = k_cache.shape
    return int(fn(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                  key.shape[0], hkv, d, block_size, num_blocks, _DTYPES[dtype], float(k_scale),
                  float(v_scale)))


def _paged_decode_q8(fn, query, k_cache, v_cache, block_tables, context_lens, scale, dtype,
                     k_scale, v_scale, num_threads):
    query = _u16(query)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    s, hq, d = query.shape
    num_blocks, bs, hkv, _ = k_cache.shape
    out = np.empty((s, hq, d), dtype=np.float64)
    st = fn(_ptr(out), _ptr(query), _ptr(_code_bytes(k_cache)), _ptr(_code_bytes(v_cache)),
            _ptr(block_tables), _ptr(context_lens), s, hq, hkv, d, bs, block_tables.shape[1],
            num_blocks, float(scale), _DTYPES[dtype], float(k_scale), float(v_scale), num_threads)
    return out, int(st)


def reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, block_size, dtype,
                          k_scale, v_scale, lib=None) -> int:
    """Quantising cache write into uint8 e4m3 pools [num_blocks][B][Hkv][D]."""
    return _reshape_and_cache_q8((lib or load()).oracle_reshape_and_cache_fp8, key, value,
                                 k_cache, v_cache, slot_mapping, block_size, dtype, k_scale,
                                 v_scale)


def paged_decode_fp8(query, k_cache, v_cache, block_tables, context_lens, scale, dtype, k_scale,
                     v_scale, num_threads=0, lib=None):
    """fp64 paged decode over e4m3 pools (dequantised with the scales)."""
    return _paged_decode_q8((lib or load()).oracle_paged_decode_fp8, query, k_cache, v_cache,
                            block_tables, context_lens, scale, dtype, k_scale, v_scale,
                            num_threads)


# ---- INT8 caches: two's-complement codes, per-tensor scales -------------------

def decode_int8(codes: np.ndarray, lib=None) -> np.ndarray:
    """int8 code (given as raw bytes, uint8 or int8) -> float64."""
    codes = _code_bytes(codes)
    out = np.empty(codes.shape, dtype=np.float64)
    (lib or load()).oracle_decode_int8(_ptr(codes), _ptr(out), codes.size)
    return out


def encode_int8(x: np.ndarray, lib=None) -> np.ndarray:
    """float32 -> int8 code (returned as int8): nearest, ties to even,
    saturating at -128 / 127, NaN -> 0."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    (lib or load()).oracle_encode_int8(_ptr(x), _ptr(out), x.size)
    return out.view(np.int8)


def reshape_and_cache_int8(key, value, k_cache, v_cache, slot_mapping, block_size, dtype,
                           k_scale, v_scale, lib=None) -> int:
    """Quantising cache write into int8 pools [num_blocks][B][Hkv][D]."""
    return _reshape_and_cache_q8((lib or load()).oracle_reshape_and_cache_int8, key, value,
                                 k_cache, v_cache, slot_mapping, block_size, dtype, k_scale,
                                 v_scale)


def paged_decode_int8(query, k_cache, v_cache, block_tables, context_lens, scale, dtype, k_scale,
                      v_scale, num_threads=0, lib=None):
    """fp64 paged decode over int8 pools (code x scale)."""
    return _paged_decode_q8((lib or load()).oracle_paged_decode_int8, query, k_cache, v_cache,
                            block_tables, context_lens, scale, dtype, k_scale, v_scale,
                            num_threads)


# ---- Row-scaled one-byte caches: one fp32 scale per (token, kv head) row ------

def _scale_pool(a: np.ndarray, num_blocks: int, num_kv_heads: int, block_size: int) -> np.ndarray:
    assert a.dtype == np.float32 and a.flags["C_CONTIGUOUS"], "scale pools are float32, contiguous"
    assert a.shape == (num_blocks, num_kv_heads, block_size), a.shape
    return a


def _reshape_and_cache_rowscale(fmt, key, value, k_cache, v_cache, k_scales, v_scales,
                                slot_mapping, block_size, dtype, lib):
    key, value = _u16(key), _u16(value)
    assert k_cache.dtype in (np.uint8, np.int8) and v_cache.dtype == k_cache.dtype
    assert k_cache.flags["C_CONTIGUOUS"] and v_cache.flags["C_CONTIGUOUS"]
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    num_blocks, bs, hkv, d = k_cache.shape
    assert bs == block_size
    _scale_pool(k_scales, num_blocks, hkv, bs)
    _scale_pool(v_scales, num_blocks, hkv, bs)
    fn = getattr(lib or load(), f"oracle_reshape_and_cache_{fmt}_rowscale")
    return int(fn(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(k_scales),
                  _ptr(v_scales), _ptr(slot_mapping), key.shape[0], hkv, d, block_size,
                  num_blocks, _DTYPES[dtype]))


def _paged_decode_rowscale(fmt, query, k_cache, v_cache, k_scales, v_scales, block_tables,
                           context_lens, scale, dtype, num_threads, lib):
    query = _u16(query)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    s, hq, d = query.shape
    num_blocks, bs, hkv, _ = k_cache.shape
    _scale_pool(k_scales, num_blocks, hkv, bs)
    _scale_pool(v_scales, num_blocks, hkv, bs)
    out = np.empty((s, hq, d), dtype=np.float64)
    fn = getattr(lib or load(), f"oracle_paged_decode_{fmt}_rowscale")
    st = fn(_ptr(out), _ptr(query), _ptr(_code_bytes(k_cache)), _ptr(_code_bytes(v_cache)),
            _ptr(k_scales), _ptr(v_scales), _ptr(block_tables), _ptr(context_lens), s, hq, hkv,
            d, bs, block_tables.shape[1], num_blocks, float(scale), _DTYPES[dtype], num_threads)
    return out, int(st)


def reshape_and_cache_fp8_rowscale(key, value, k_cache, v_cache, k_scales, v_scales,
                                   slot_mapping, block_size, dtype, lib=None) -> int:
    """Quantising cache write into uint8 e4m3 pools [num_blocks][B][Hkv][D]
    with one fp32 scale per row in k_scales / v_scales [num_blocks][Hkv][B]:
    s = fp32(max |x| / 448), code = e4m3(fp32(x * fp32(1 / s)))."""
    return _reshape_and_cache_rowscale("fp8", key, value, k_cache, v_cache, k_scales, v_scales,
                                       slot_mapping, block_size, dtype, lib)


def reshape_and_cache_int8_rowscale(key, value, k_cache, v_cache, k_scales, v_scales,
                                    slot_mapping, block_size, dtype, lib=None) -> int:
    """As reshape_and_cache_fp8_rowscale for int8 pools: s = fp32(max |x| / 127)."""
    return _reshape_and_cache_rowscale("int8", key, value, k_cache, v_cache, k_scales, v_scales,
                                       slot_mapping, block_size, dtype, lib)


def paged_decode_fp8_rowscale(query, k_cache, v_cache, k_scales, v_scales, block_tables,
                              context_lens, scale, dtype, num_threads=0, lib=None):
    """fp64 paged decode over e4m3 pools, each row dequantised with its own scale."""
    return _paged_decode_rowscale("fp8", query, k_cache, v_cache, k_scales, v_scales,
                                  block_tables, context_lens, scale, dtype, num_threads, lib)


def paged_decode_int8_rowscale(query, k_cache, v_cache, k_scales, v_scales, block_tables,
                               context_lens, scale, dtype, num_threads=0, lib=None):
    """fp64 paged decode over int8 pools, each row dequantised with its own scale."""
    return _paged_decode_rowscale("int8", query, k_cache, v_cache, k_scales, v_scales,
                                  block_tables, context_lens, scale, dtype, num_threads, lib)
