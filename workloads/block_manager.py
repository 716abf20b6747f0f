"""Host-side block allocator model: free pool, per-sequence block tables,
reference counts and copy-on-write decisions.

It produces the inputs the kernels consume (block tables, slot mappings and
the (src, dst) pairs of copy-on-write copies); it never touches K/V data.

Pages cited (title, then section):
  [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
  [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
  [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"

Behaviour followed:
  * fixed-size physical blocks taken on demand from one free pool; a block
    table per sequence maps logical block j to a physical id
    ([VM-paging, 虚拟内存分页机制到KV Cache的映射]; [Practice §3.2, §3.3]);
  * on-demand allocation: if the last logical block has room the token goes
    there, otherwise a new physical block is taken, the table is extended and
    then the token's K/V is written ([Practice §3.3 按需分配策略], steps 1-4);
  * sharing: sequences that share a prefix point at the same physical blocks
    and each share raises the block's reference count
    ([VM-paging, 写时复制与块共享机制]; [Practice §4.1]);
  * copy-on-write: a sequence that must modify a block whose count is 1
    modifies it in place; with a count above 1 it copies the block to a new
    physical block, writes there, remaps its table and drops one reference
    on the original ([VM-paging, 写时复制与块共享机制]; [Practice §4.1] steps 1-4);
  * reclamation: freeing a sequence drops one reference on each of its
    blocks; a block whose count reaches 0 returns to the free pool
    ([VM-paging, 写时复制与块共享机制], last paragraph);
  * exhaustion: a request that needs more blocks than are free fails with
    ``None`` and leaves the state unchanged ([Manager, 第四部分
    KVCacheManager 与 allocate_slots()]);
  * internal waste is at most block_size - 1 slots per sequence
    ([Manager, 第二部分 碎片问题的解决]).
"""
from __future__ import annotations

from collections import deque

import numpy as np


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        """free_order: the order in which physical ids leave the free pool
        (a seeded permutation gives randomly scattered blocks)."""
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = range(num_blocks) if free_order is None else [int(b) for b in free_order]
        self.free = deque(order)
        assert len(self.free) == num_blocks and len(set(self.free)) == num_blocks
        self.ref = np.zeros(num_blocks, dtype=np.int64)
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    # -- queries ---------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def internal_waste(self, seq: int) -> int:
        return len(self.tables[seq]) * self.block_size - self.lens[seq]

    def slot(self, seq: int, pos: int) -> int:
        table = self.tables[seq]
        return table[pos // self.block_size] * self.block_size + pos % self.block_size

    def blocks_needed(self, seq: int, n: int) -> int:
        """New physical blocks that appending n tokens to seq would take."""
        if n <= 0:
            return 0
        length = self.lens.get(seq, 0)
        b = self.block_size
        need = -(-(length + n) // b) - (-(-length // b))
        if length % b != 0 and self.ref[self.tables[seq][-1]] > 1:
            need += 1                      # copy-on-write of the shared last block
        return need

    def block_table_array(self, seqs, max_blocks: int | None = None) -> np.ndarray:
        seqs = list(seqs)
        width = max(len(self.tables[s]) for s in seqs) if max_blocks is None else max_blocks
        arr = np.full((len(seqs), max(width, 1)), -1, dtype=np.int32)
        for i, s in enumerate(seqs):
            t = self.tables[s]
            arr[i, :len(t)] = t
        return arr

    # -- mutations -------------------------------------------------------
    def _take(self) -> int:
        b = self.free.popleft()
        assert self.ref[b] == 0
        self.ref[b] = 1
        return b

    def add_sequence(self, seq: int, num_tokens: int):
        """Register a new sequence and give slots to its first num_tokens
        tokens.  Returns the slot list, or None if the pool is too small."""
        assert seq not in self.tables
        self.tables[seq] = []
        self.lens[seq] = 0
        res = self.append_slots(seq, num_tokens)
        if res is None:
            del self.tables[seq], self.lens[seq]
            return None
        return res[0]

    def fork(self, src: int, dst: int) -> None:
        """dst shares every block of src (reference counts rise by one)."""
        assert dst not in self.tables
        self.tables[dst] = list(self.tables[src])
        self.lens[dst] = self.lens[src]
        for b in self.tables[dst]:
            self.ref[b] += 1

    def append_slots(self, seq: int, n: int):
        """Slots for the next n tokens of seq.  Returns (slots, cow_pairs),
        cow_pairs being the (src, dst) block copies that must run before the
        tokens are written; or None (state unchanged) when the free pool is
        too small."""
        if self.blocks_needed(seq, n) > len(self.free):
            return None
        b = self.block_size
        table = self.tables[seq]
        slots, cow = [], []
        for _ in range(n):
            pos = self.lens[seq]
            if pos % b == 0:
                table.append(self._take())
            else:
                last = table[-1]
                if self.ref[last] > 1:
                    new = self._take()
                    cow.append((last, new))
                    self.ref[last] -= 1
                    table[-1] = new
            slots.append(table[pos // b] * b + pos % b)
            self.lens[seq] = pos + 1
        return slots, cow

    def free_sequence(self, seq: int) -> None:
        for blk in reversed(self.tables.pop(seq)):         # last block first
            self.ref[blk] -= 1
            assert self.ref[blk] >= 0
            if self.ref[blk] == 0:
                self.free.append(blk)
        del self.lens[seq]

    # -- invariants ------------------------------------------------------
    def check_invariants(self) -> None:
        counts = np.zeros(self.num_blocks, dtype=np.int64)
        for t in self.tables.values():
            for blk in t:
                counts[blk] += 1
        assert np.array_equal(counts, self.ref), "reference counts != table references"
        free = set(self.free)
        assert len(free) == len(self.free), "a block is twice in the free pool"
        for blk in range(self.num_blocks):
            assert (blk in free) == (self.ref[blk] == 0), f"block {blk} free/ref mismatch"
        for s in self.tables:
            w = self.internal_waste(s)
            assert 0 <= w <= self.block_size - 1, f"seq {s} wastes {w} slots"
