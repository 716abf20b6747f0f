"""ctypes binding of the native host block manager (include/pa_block_manager.h).

Argument marshalling only; the block tables, reference counts, free queue,
copy-on-write decisions, prefix cache and host-pool swap bookkeeping live in
C++ inside libpa.so.
"""
from __future__ import annotations

import ctypes

import numpy as np

from .binding import LIB

PA_BM_OK, PA_BM_NO_SPACE, PA_BM_BAD_ARG, PA_BM_CAPACITY = 0, 1, 2, 3

_p, _i32, _i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
LIB.pa_bm_create.argtypes = [_i32, _i32, _i32]
LIB.pa_bm_create.restype = _p
LIB.pa_bm_destroy.argtypes = [_p]
LIB.pa_bm_destroy.restype = None
LIB.pa_bm_num_free_blocks.argtypes = [_p]
LIB.pa_bm_num_free_blocks.restype = _i32
LIB.pa_bm_ref_count.argtypes = [_p, _i32]
LIB.pa_bm_ref_count.restype = _i32
LIB.pa_bm_num_cached_blocks.argtypes = [_p]
LIB.pa_bm_num_cached_blocks.restype = _i32
LIB.pa_bm_add_sequence.argtypes = [_p, _i64, _p, _i32, _i64, _p, _p]
LIB.pa_bm_add_sequence.restype = _i32
LIB.pa_bm_add_sequence_priority.argtypes = [_p, _i64, _p, _i32, _i64, _i32, _p, _p]
LIB.pa_bm_add_sequence_priority.restype = _i32
LIB.pa_bm_fork.argtypes = [_p, _i64, _i64]
LIB.pa_bm_fork.restype = _i32
LIB.pa_bm_append_slots.argtypes = [_p, _i64, _p, _i32, _p, _p, _i32, _p]
LIB.pa_bm_append_slots.restype = _i32
LIB.pa_bm_free_sequence.argtypes = [_p, _i64]
LIB.pa_bm_free_sequence.restype = _i32
LIB.pa_bm_block_table.argtypes = [_p, _i64, _p, _i32, _p]
LIB.pa_bm_block_table.restype = _i32
LIB.pa_bm_context_len.argtypes = [_p, _i64]
LIB.pa_bm_context_len.restype = _i32
LIB.pa_bm_check.argtypes = [_p]
LIB.pa_bm_check.restype = _i32
LIB.pa_bm_set_watermark.argtypes = [_p, _i32]
LIB.pa_bm_set_watermark.restype = _i32
LIB.pa_bm_attach_host_pool.argtypes = [_p, _i32]
LIB.pa_bm_attach_host_pool.restype = _i32
LIB.pa_bm_num_free_host_blocks.argtypes = [_p]
LIB.pa_bm_num_free_host_blocks.restype = _i32
LIB.pa_bm_is_swapped.argtypes = [_p, _i64]
LIB.pa_bm_is_swapped.restype = _i32
LIB.pa_bm_swap_out.argtypes = [_p, _p, _i32, _p, _i32, _p]
LIB.pa_bm_swap_out.restype = _i32
LIB.pa_bm_swap_in.argtypes = [_p, _p, _i32, _p, _i32, _p]
LIB.pa_bm_swap_in.restype = _i32


class BlockManagerStats(ctypes.Structure):
    """pa_bm_stats_t (include/pa_block_manager.h)."""
    _fields_ = [(n, ctypes.c_int32) for n in ("num_blocks", "block_size", "used_blocks",
                                             "free_blocks", "cached_blocks", "num_seqs",
                                             "swapped_seqs", "free_host_blocks")] + \
               [(n, ctypes.c_int64) for n in ("stored_tokens", "prefix_queries", "prefix_hits")]

    @property
    def utilisation(self) -> float:
        cap = self.used_blocks * self.block_size
        return self.stored_tokens / cap if cap else 1.0

    @property
    def hit_rate(self) -> float:
        return self.prefix_hits / self.prefix_queries if self.prefix_queries else 0.0


LIB.pa_bm_stats.argtypes = [_p, _p]
LIB.pa_bm_stats.restype = _i32


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


class NativeBlockManager:
    """Same operations as the Python allocator model, in C++."""

    def __init__(self, num_blocks: int, block_size: int, prefix_caching: bool = False):
        self.h = LIB.pa_bm_create(num_blocks, block_size, 1 if prefix_caching else 0)
        if not self.h:
            raise ValueError("pa_bm_create failed")
        self.num_blocks, self.block_size = num_blocks, block_size

    def __del__(self):
        h = getattr(self, "h", None)
        if h:
            LIB.pa_bm_destroy(h)
            self.h = None

    def num_free(self) -> int:
        return int(LIB.pa_bm_num_free_blocks(self.h))

    def ref(self, block: int) -> int:
        return int(LIB.pa_bm_ref_count(self.h, block))

    def num_cached(self) -> int:
        return int(LIB.pa_bm_num_cached_blocks(self.h))

    def add_sequence(self, seq: int, num_tokens: int, tokens=None, extra_key: int = 0,
                     high_priority: bool = False):
        """Returns (slots, cached_tokens), or None when the pool is too small.
        high_priority: the request may use the watermark reserve."""
        toks = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(num_tokens, dtype=np.int64)
        cached = ctypes.c_int32(0)
        rc = LIB.pa_bm_add_sequence_priority(self.h, seq, _ptr(toks), num_tokens, extra_key,
                                             1 if high_priority else 0, _ptr(slots),
                                             ctypes.byref(cached))
        if rc == PA_BM_NO_SPACE:
            return None
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_add_sequence: {rc}")
        return slots.tolist(), int(cached.value)

    def fork(self, src: int, dst: int) -> None:
        rc = LIB.pa_bm_fork(self.h, src, dst)
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_fork: {rc}")

    def append_slots(self, seq: int, n: int, tokens=None):
        """Returns (slots, cow_pairs), or None when the pool is too small."""
        toks = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(max(n, 1), dtype=np.int64)
        cow = np.empty((1, 2), dtype=np.int64)
        ncow = ctypes.c_int32(0)
        rc = LIB.pa_bm_append_slots(self.h, seq, _ptr(toks), n, _ptr(slots), _ptr(cow), 1,
                                    ctypes.byref(ncow))
        if rc == PA_BM_NO_SPACE:
            return None
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_append_slots: {rc}")
        return slots[:n].tolist(), [tuple(int(x) for x in cow[i]) for i in range(ncow.value)]

    def free_sequence(self, seq: int) -> None:
        rc = LIB.pa_bm_free_sequence(self.h, seq)
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_free_sequence: {rc}")

    def block_table(self, seq: int) -> list[int]:
        n = ctypes.c_int32(0)
        LIB.pa_bm_block_table(self.h, seq, None, 0, ctypes.byref(n))
        out = np.empty(max(n.value, 1), dtype=np.int32)
        rc = LIB.pa_bm_block_table(self.h, seq, _ptr(out), out.shape[0], ctypes.byref(n))
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_block_table: {rc}")
        return out[:n.value].tolist()

    def context_len(self, seq: int) -> int:
        return int(LIB.pa_bm_context_len(self.h, seq))

    def check(self) -> int:
        return int(LIB.pa_bm_check(self.h))

    def stats(self) -> BlockManagerStats:
        st = BlockManagerStats()
        rc = LIB.pa_bm_stats(self.h, ctypes.byref(st))
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_stats: {rc}")
        return st

    def set_watermark(self, reserved_blocks: int) -> None:
        """Free blocks that admissions (add_sequence, swap_in) must leave."""
        rc = LIB.pa_bm_set_watermark(self.h, reserved_blocks)
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_set_watermark: {rc}")

    # ---- swapping to a host pool ----------------------------------------------

    def attach_host_pool(self, num_host_blocks: int) -> None:
        rc = LIB.pa_bm_attach_host_pool(self.h, num_host_blocks)
        if rc != PA_BM_OK:
            raise ValueError(f"pa_bm_attach_host_pool: {rc}")

    def num_free_host(self) -> int:
        return int(LIB.pa_bm_num_free_host_blocks(self.h))

    def is_swapped(self, seq: int) -> int:
        return int(LIB.pa_bm_is_swapped(self.h, seq))

    def _swap(self, fn, name, seqs):
        ids = np.ascontiguousarray(list(seqs), dtype=np.int64)
        cap = max(1, sum(max(0, -(-self.context_len(int(s)) // self.block_size)) for s in ids))
        pairs = np.empty((cap, 2), dtype=np.int64)
        n = ctypes.c_int32(0)
        rc = fn(self.h, _ptr(ids), ids.shape[0], _ptr(pairs), cap, ctypes.byref(n))
        if rc == PA_BM_NO_SPACE:
            return None
        if rc != PA_BM_OK:
            raise ValueError(f"{name}: {rc}")
        return [tuple(int(x) for x in pairs[i]) for i in range(n.value)]

    def swap_out(self, seqs):
        """The group's (device block, host block) copies for pa_swap_blocks,
        or None when the host pool is too small."""
        return self._swap(LIB.pa_bm_swap_out, "pa_bm_swap_out", seqs)

    def swap_in(self, seqs):
        """The group's (host block, device block) copies for pa_swap_blocks,
        or None when the device pool is too small."""
        return self._swap(LIB.pa_bm_swap_in, "pa_bm_swap_in", seqs)
