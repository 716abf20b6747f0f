"""The native (C++) host block manager: differential against the Python
allocator model on random operation streams, its own invariant check, and
the prefix cache (CPU only; no GPU call is made).

Pages cited (title, then section):
  [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
  [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
"""
import numpy as np
import pytest

from workloads.block_manager import BlockManager


@pytest.fixture(scope="module")
def native():
    from paged_kv_cache_415_b200 import build
    build.build()
    from paged_kv_cache_415_b200.block_manager import NativeBlockManager
    return NativeBlockManager


@pytest.mark.parametrize("seed", range(8))
def test_matches_python_model(native, seed):
    rng = np.random.Generator(np.random.PCG64(100 + seed))
    nb, b = 96, 16
    py, cc = BlockManager(nb, b), native(nb, b)
    live, next_id = [], 0
    for _ in range(500):
        op = int(rng.integers(0, 4))
        if op == 0 or not live:
            n = int(rng.integers(0, 70))
            a = py.add_sequence(next_id, n)
            r = cc.add_sequence(next_id, n)
            assert (a is None) == (r is None)
            if a is not None:
                assert a == r[0] and r[1] == 0
                live.append(next_id)
            next_id += 1
        elif op == 1:
            s = live[int(rng.integers(0, len(live)))]
            n = int(rng.integers(0, 40))
            a, r = py.append_slots(s, n), cc.append_slots(s, n)
            assert (a is None) == (r is None)
            if a is not None:
                assert a[0] == r[0] and a[1] == r[1]
        elif op == 2:
            s = live[int(rng.integers(0, len(live)))]
            py.fork(s, next_id)
            cc.fork(s, next_id)
            live.append(next_id)
            next_id += 1
        else:
            s = live.pop(int(rng.integers(0, len(live))))
            py.free_sequence(s)
            cc.free_sequence(s)
        assert cc.check() == 0
        assert py.num_free() == cc.num_free()
    for s in live:
        assert py.tables[s] == cc.block_table(s)
        assert py.lens[s] == cc.context_len(s)
    assert [int(x) for x in py.ref] == [cc.ref(i) for i in range(nb)]
    for s in live:
        cc.free_sequence(s)
    assert cc.num_free() == nb and cc.check() == 0


def test_exhaustion_leaves_state_unchanged(native):
    cc = native(4, 16)
    assert cc.add_sequence(0, 40) is not None                 # 3 blocks
    before = (cc.num_free(), cc.block_table(0), [cc.ref(i) for i in range(4)])
    assert cc.append_slots(0, 30) is None
    assert cc.add_sequence(1, 33) is None
    assert (cc.num_free(), cc.block_table(0), [cc.ref(i) for i in range(4)]) == before
    assert cc.context_len(1) == -1 and cc.check() == 0


def test_copy_on_write_in_native(native):
    cc = native(16, 4)
    cc.add_sequence(0, 6)
    a, bb = cc.block_table(0)
    cc.fork(0, 1)
    slots, cow = cc.append_slots(1, 1)
    assert cow == [(bb, cow[0][1])] and cc.ref(bb) == 1
    slots, cow = cc.append_slots(0, 1)                          # last holder: in place
    assert cow == [] and slots == [bb * 4 + 2]
    assert cc.check() == 0


# ---- automatic prefix caching ([Manager, 第三部分]) ------------------------

def _toks(rng, n):
    return rng.integers(0, 32000, size=n).astype(np.int32)


def test_prefix_hits_share_blocks(native):
    rng = np.random.Generator(np.random.PCG64(1))
    cc = native(32, 16, prefix_caching=True)
    p = _toks(rng, 40)
    s0, c0 = cc.add_sequence(0, 40, p)
    assert c0 == 0 and cc.num_cached() == 2                     # two full blocks hashed
    s1, c1 = cc.add_sequence(1, 40, p)
    assert c1 == 32                                             # both full blocks reused
    t0, t1 = cc.block_table(0), cc.block_table(1)
    assert t0[:2] == t1[:2] and t0[2] != t1[2]
    assert cc.ref(t0[0]) == 2 and cc.ref(t0[2]) == 1
    assert cc.check() == 0


def test_whole_prompt_hit_still_computes_the_last_token(native):
    rng = np.random.Generator(np.random.PCG64(2))
    cc = native(32, 16, prefix_caching=True)
    p = _toks(rng, 32)
    cc.add_sequence(0, 32, p)
    _, c = cc.add_sequence(1, 32, p)
    assert c == 16                                              # the second block is recomputed
    assert cc.block_table(0)[0] == cc.block_table(1)[0]
    assert cc.block_table(0)[1] != cc.block_table(1)[1]


def test_freed_blocks_stay_cached_and_revive(native):
    rng = np.random.Generator(np.random.PCG64(3))
    cc = native(32, 16, prefix_caching=True)
    p = _toks(rng, 50)
    cc.add_sequence(0, 50, p)
    t0 = cc.block_table(0)
    cc.free_sequence(0)
    assert cc.num_free() == 32 and cc.num_cached() == 3
    free_before = cc.num_free()
    _, c = cc.add_sequence(1, 50, p)
    assert c == 48 and cc.block_table(1)[:3] == t0[:3]
    assert cc.num_free() == free_before - 4                     # 3 revived + 1 fresh
    assert cc.check() == 0


def test_allocation_evicts_from_the_queue_head(native):
    """Freed blocks queue up last block first, so allocation evicts a
    prompt's tail before its head: the most reusable prefix block survives."""
    rng = np.random.Generator(np.random.PCG64(4))
    cc = native(8, 16, prefix_caching=True)
    a, b = _toks(rng, 48), _toks(rng, 48)
    cc.add_sequence(0, 48, a)                                   # blocks 0, 1, 2
    cc.add_sequence(1, 48, b)                                   # blocks 3, 4, 5
    cc.free_sequence(0)                                         # queue: 6 7 2 1 0
    cc.free_sequence(1)                                         # queue: 6 7 2 1 0 5 4 3
    cc.add_sequence(2, 64, _toks(rng, 64))                      # takes 6 7 2 1: a's tail
    assert cc.num_cached() == 8                                 # a first block, b three, seq 2 four
    assert cc.add_sequence(3, 48, a)[1] == 16                   # only a's first block is left
    assert cc.check() == 0


def test_extra_key_and_chain_isolate(native):
    rng = np.random.Generator(np.random.PCG64(5))
    cc = native(32, 16, prefix_caching=True)
    p = _toks(rng, 48)
    cc.add_sequence(0, 48, p, extra_key=7)
    assert cc.add_sequence(1, 48, p, extra_key=8)[1] == 0       # other adapter: no reuse
    q = p.copy()
    q[0] += 1                                                   # first block differs ...
    assert cc.add_sequence(2, 48, q, extra_key=7)[1] == 0       # ... so later blocks miss too
    assert cc.add_sequence(3, 48, p, extra_key=7)[1] == 32
    assert cc.check() == 0


def test_appended_full_blocks_become_cached(native):
    rng = np.random.Generator(np.random.PCG64(6))
    cc = native(32, 16, prefix_caching=True)
    p = _toks(rng, 10)
    gen = _toks(rng, 30)
    cc.add_sequence(0, 10, p)
    assert cc.num_cached() == 0
    cc.append_slots(0, 30, gen)                                 # fills blocks 0 and 1
    assert cc.num_cached() == 2
    full = np.concatenate([p, gen])
    _, c = cc.add_sequence(1, 40, full)
    assert c == 32 and cc.block_table(1)[:2] == cc.block_table(0)[:2]
    assert cc.check() == 0


@pytest.mark.parametrize("seed", range(4))
def test_random_streams_with_caching_keep_invariants(native, seed):
    rng = np.random.Generator(np.random.PCG64(200 + seed))
    cc = native(64, 16, prefix_caching=True)
    prompts = [_toks(rng, int(rng.integers(1, 90))) for _ in range(6)]
    live, next_id = [], 0
    for _ in range(400):
        op = int(rng.integers(0, 4))
        if op == 0 or not live:
            p = prompts[int(rng.integers(0, len(prompts)))]
            n = int(rng.integers(1, len(p) + 1))
            r = cc.add_sequence(next_id, n, p[:n], extra_key=int(rng.integers(0, 2)))
            if r is not None:
                assert r[1] < n
                live.append(next_id)
            next_id += 1
        elif op == 1:
            s = live[int(rng.integers(0, len(live)))]
            n = int(rng.integers(0, 30))
            cc.append_slots(s, n, _toks(rng, n))
        elif op == 2:
            s = live[int(rng.integers(0, len(live)))]
            cc.fork(s, next_id)
            live.append(next_id)
            next_id += 1
        else:
            cc.free_sequence(live.pop(int(rng.integers(0, len(live)))))
        assert cc.check() == 0
    for s in live:
        cc.free_sequence(s)
    assert cc.num_free() == 64 and cc.check() == 0
