"""Algorithmic byte counts of the decode step and the pages' memory figures.

Algorithmic bytes are the bytes the step must move at least once, whatever
the kernel does: every context token's K and V row of its kv head, the
query, the output, the block-table entries in use and the context lengths,
plus the appended tokens' K/V (read once, written once) and, when there are
copy-on-write pairs, each copied block read and written once.

Pages cited (title, then section):
  [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
  [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
  [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
"""
from __future__ import annotations

import numpy as np

ELEM_BYTES = {"f16": 2, "bf16": 2}


def block_elements(block_size: int, num_heads: int, head_dim: int) -> int:
    """Elements in one physical block holding K and V of one layer
    ([Practice §3.1 物理块分配器设计]: tokens x heads x head_dim x 2)."""
    return block_size * num_heads * head_dim * 2


def kv_bytes_per_token(num_layers: int, num_heads: int, head_dim: int, elem_bytes: int) -> int:
    """K and V bytes one token occupies across all layers
    ([Manager, 第一部分 内存成本的量化分析])."""
    return 2 * num_layers * num_heads * head_dim * elem_bytes


def contiguous_utilisation(used_tokens: int, reserved_tokens: int) -> float:
    """Fraction of a max-length contiguous reservation actually used
    ([Practice §1]; [Manager, 第二部分 朴素方案的内存碎片噩梦])."""
    return used_tokens / reserved_tokens


def paged_waste_slots(context_len: int, block_size: int) -> int:
    """Unused slots of a sequence under paging: only the last block's tail
    ([Manager, 第二部分 碎片问题的解决]: at most block_size - 1)."""
    return (-context_len) % block_size


def decode_bytes(ctx: np.ndarray, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 block_size: int, elem_bytes: int, kv_elem_bytes: int | None = None,
                 row_scale_bytes: int = 0) -> dict:
    """Algorithmic bytes of the attention part of one decode step
    (kv_elem_bytes: bytes of a cached K/V element when it differs from the
    query's, e.g. 1 for e4m3 pools; row_scale_bytes: bytes of the scale each
    (token, kv head) row carries in row-scaled pools, 4)."""
    ctx = np.asarray(ctx, dtype=np.int64)
    s = ctx.shape[0]
    row = num_kv_heads * (head_dim * (elem_bytes if kv_elem_bytes is None else kv_elem_bytes)
                          + row_scale_bytes)
    kv = int(ctx.sum()) * row * 2
    q = s * num_q_heads * head_dim * elem_bytes
    out = q
    nb = -(-ctx // block_size)
    table = int(nb.sum()) * 4
    lens = 4 * s
    return {"kv": kv, "query": q, "out": out, "block_table": table, "context_lens": lens,
            "total": kv + q + out + table + lens}


def kv_elem_bytes(wl) -> int:
    """Bytes of one cached K/V element: 1 for e4m3 and int8 pools, else the
    element type's."""
    return 1 if wl.extra.get("kv_dtype") in ("fp8", "int8") else ELEM_BYTES[wl.dtype]


def row_scale_bytes(wl) -> int:
    """Bytes of the scale every (token, kv head) row carries: 4 for
    row-scaled one-byte pools, else 0."""
    return 4 if wl.extra.get("rowscale") else 0


def step_bytes(wl) -> dict:
    """Algorithmic bytes of a whole decode step of a workload (attention,
    appended tokens, copy-on-write copies)."""
    e = ELEM_BYTES[wl.dtype]
    ekv = kv_elem_bytes(wl)
    rs = row_scale_bytes(wl)
    att = decode_bytes(wl.context_lens, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                       wl.block_size, e, ekv, rs)
    row_in = wl.num_kv_heads * wl.head_dim * e
    row = wl.num_kv_heads * (wl.head_dim * ekv + rs)
    t = wl.num_new_tokens
    append = 2 * t * row_in + 2 * t * row + 8 * t   # K,V read + written, slot ids
    blk = wl.block_size * row
    p = int(wl.block_mapping.shape[0])
    copies = 2 * (2 * p * blk) + 16 * p          # K,V blocks read + written, pairs
    return {"attention": att["total"], "kv": att["kv"], "append": append, "copy": copies,
            "total": att["total"] + append + copies}


def unique_kv_bytes(wl) -> int:
    """K/V bytes of the distinct physical blocks the step reads (shared
    blocks counted once), for workloads with block sharing."""
    row = wl.num_kv_heads * (wl.head_dim * kv_elem_bytes(wl) + row_scale_bytes(wl))
    seen = {}
    for s in range(wl.num_seqs):
        c = int(wl.context_lens[s])
        for j in range(-(-c // wl.block_size)):
            blk = int(wl.block_tables[s, j])
            n = min(wl.block_size, c - j * wl.block_size)
            seen[blk] = max(seen.get(blk, 0), n)
    return sum(seen.values()) * row * 2
