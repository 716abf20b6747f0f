"""Host allocator model: the invariants the pages fix (CPU only).

Pages cited (title, then section):
  [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
  [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
  [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
"""
import numpy as np
import pytest

from workloads import generators as gen
from workloads.block_manager import BlockManager


def _random_run(seed, num_blocks=200, block_size=16, steps=400):
    rng = np.random.Generator(np.random.PCG64(seed))
    mgr = BlockManager(num_blocks, block_size, free_order=rng.permutation(num_blocks))
    live, next_id = [], 0
    for _ in range(steps):
        op = rng.integers(0, 4)
        if op == 0 or not live:
            if mgr.add_sequence(next_id, int(rng.integers(0, 70))) is not None:
                live.append(next_id)
            next_id += 1
        elif op == 1:
            s = live[int(rng.integers(0, len(live)))]
            mgr.append_slots(s, int(rng.integers(0, 40)))
        elif op == 2:
            s = live[int(rng.integers(0, len(live)))]
            mgr.fork(s, next_id)
            live.append(next_id)
            next_id += 1
        else:
            s = live.pop(int(rng.integers(0, len(live))))
            mgr.free_sequence(s)
        mgr.check_invariants()
    return mgr, live


@pytest.mark.parametrize("seed", range(6))
def test_internal_waste_and_refcounts(seed):
    """Waste <= block_size - 1 per sequence [Manager, 第二部分 碎片问题的解决];
    reference counts equal table references; free <=> count 0."""
    mgr, _ = _random_run(seed)
    mgr.check_invariants()


@pytest.mark.parametrize("seed", range(6))
def test_everything_returns_to_the_pool(seed):
    """Freeing every sequence returns every block, shared ones included
    ([VM-paging, 写时复制与块共享机制], last paragraph)."""
    mgr, live = _random_run(seed)
    for s in live:
        mgr.free_sequence(s)
    assert mgr.num_free() == mgr.num_blocks
    assert sorted(mgr.free) == list(range(mgr.num_blocks))
    assert not mgr.ref.any()


def test_exhaustion_fails_without_side_effects():
    """A request the pool cannot serve returns None and changes nothing
    ([Manager, 第四部分 KVCacheManager 与 allocate_slots()])."""
    mgr = BlockManager(4, 16)
    assert mgr.add_sequence(0, 40) is not None        # 3 blocks
    snap = (list(mgr.free), mgr.ref.copy(), {k: list(v) for k, v in mgr.tables.items()},
            dict(mgr.lens))
    assert mgr.append_slots(0, 30) is None             # needs 2, 1 free
    assert mgr.add_sequence(1, 33) is None             # needs 3
    assert (list(mgr.free), mgr.tables, mgr.lens) == (snap[0], snap[2], snap[3])
    assert np.array_equal(mgr.ref, snap[1]) and 1 not in mgr.tables
    assert mgr.append_slots(0, 24) is not None         # fits exactly
    assert mgr.num_free() == 0


def test_copy_on_write_rules():
    """Count 1 -> write in place; count > 1 -> copy to a new block, remap,
    drop one reference on the original ([VM-paging, 写时复制与块共享机制];
    [Practice §4.1] steps 1-4)."""
    mgr = BlockManager(16, 4)
    mgr.add_sequence(0, 6)                              # blocks A (full), B (2 of 4)
    a, b = mgr.tables[0]
    mgr.fork(0, 1)
    mgr.fork(0, 2)
    assert mgr.ref[a] == 3 and mgr.ref[b] == 3
    slots, cow = mgr.append_slots(1, 1)
    assert len(cow) == 1 and cow[0][0] == b and mgr.ref[b] == 2
    new = cow[0][1]
    assert mgr.tables[1] == [a, new] and slots == [new * 4 + 2]
    slots, cow = mgr.append_slots(2, 1)
    assert len(cow) == 1 and mgr.ref[b] == 1
    slots, cow = mgr.append_slots(0, 1)                 # last holder: in place
    assert cow == [] and slots == [b * 4 + 2] and mgr.tables[0] == [a, b]
    mgr.check_invariants()
    slots, cow = mgr.append_slots(0, 3)                 # fills B, opens a fresh block
    assert cow == [] and len(mgr.tables[0]) == 3
    mgr.check_invariants()


def test_beam_search_workload_sharing():
    """The beam-search generator: one stored copy of each prompt, at most
    beams - 1 copies of its shared partial block, and everything returns to
    the pool afterwards.  The memory saving of sharing is reported for
    context next to the 40-70% the VM-paging page quotes for beam search."""
    wl = gen.beam_search(prompts=4, beams=4, prompt_len=1000, max_new=256, num_heads=2,
                         num_blocks=1024)
    mgr: BlockManager = wl.extra["manager"]
    mgr.check_invariants()
    n_new = wl.extra["n_new"]
    writers = (n_new > 0).sum(axis=1)
    expect = sum(max(int(w) - 1, 0) if (1000 % 16) else 0 for w in writers)
    assert wl.block_mapping.shape[0] == expect
    # shared full prompt blocks keep a count of 4
    for p in range(4):
        full = wl.block_tables[p * 4, :1000 // 16]
        assert np.all(mgr.ref[full] == 4)
    used = mgr.num_blocks - mgr.num_free()
    unshared = sum(-(-int(c) // 16) for c in wl.context_lens)
    saving = 1 - used / unshared
    assert 0.5 < saving < 0.8
    for s in list(mgr.tables):
        mgr.free_sequence(s)
    assert mgr.num_free() == mgr.num_blocks


def test_generator_pool_reproduces_logical_tokens():
    """Gathering the generator's pool through its tables (plus the step's
    appended tokens) gives back every sequence's logical K/V; every slot no
    token owns (or that no copy filled) holds the NaN sentinel."""
    for wl in (gen.tiny(), gen.beam_search(prompts=2, beams=4, prompt_len=40, max_new=24,
                                           num_heads=4, num_blocks=64, keep_logical=True)):
        from tests.oracle_pins import pool_after_step
        kc, vc = pool_after_step(wl)
        owned = np.zeros(kc.shape[:2], bool)
        for s in range(wl.num_seqs):
            c = int(wl.context_lens[s])
            pos = np.arange(c)
            blk = wl.block_tables[s, pos // wl.block_size]
            off = pos % wl.block_size
            assert np.array_equal(kc[blk, off], wl.keys[s])
            assert np.array_equal(vc[blk, off], wl.values[s])
            owned[blk, off] = True
        for src, dst in wl.block_mapping:            # copies of owned blocks
            owned[dst] |= owned[src]
        assert np.all(kc[~owned] == gen.NAN_BITS[wl.dtype])


def test_generators_are_deterministic():
    a, b = gen.tiny(), gen.tiny()
    for f in ("query", "k_cache", "v_cache", "block_tables", "slot_mapping", "block_mapping",
              "new_key"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-39, 1.0 + 2 ** -8], np.float32)
    bits = gen.f32_to_bits(x, "bf16")
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    # halfway cases go to the even neighbour
    assert back[1] == 1.0 and back[2] == 1.015625 and back[5] == 1.0
    assert back[0] == 1.0 and back[3] == -2.5
    assert np.all(np.abs(back - x) <= np.abs(x) * 2 ** -8 + 1e-40)
