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


# ---- swapping to a host pool ([VM-paging, 显存管理与调度策略设计], eviction) ------

def _tag(extra, tokens):
    """The bytes a token's K/V stands for: a function of its whole prefix
    (and the extra key), so prefix-cache hits and revived blocks must already
    hold them."""
    h = (extra * 1000003 + 7) & 0xFFFFFFFF
    for t in tokens:
        h = (h * 31 + int(t) + 1) & 0xFFFFFFFF
    return h


class _Pools:
    """Device and host pools of 32-bit tags (two uint16 per slot), moved
    only by the oracle's copy_blocks and swap_blocks."""

    def __init__(self, nb, nh, b):
        self.b = b
        self.dev = np.zeros((nb, b, 1, 2), np.uint16)
        self.host = np.zeros((nh, b, 1, 2), np.uint16)
        self.scratch_dev = np.zeros_like(self.dev)
        self.scratch_host = np.zeros_like(self.host)

    def write(self, slot, tag):
        self.dev[slot // self.b, slot % self.b, 0] = (tag & 0xFFFF, tag >> 16)

    def read(self, table, n):
        out = []
        for p in range(n):
            lo, hi = self.dev[table[p // self.b], p % self.b, 0]
            out.append(int(lo) | (int(hi) << 16))
        return out

    def cow(self, pairs):
        import oracle
        if pairs:
            assert oracle.copy_blocks(self.dev, self.scratch_dev, np.array(pairs)) == 0

    def swap_out(self, pairs):
        import oracle
        if pairs:
            assert oracle.swap_blocks(self.dev, self.scratch_dev, self.host, self.scratch_host,
                                      np.array(pairs)) == 0

    def swap_in(self, pairs):
        import oracle
        if pairs:
            assert oracle.swap_blocks(self.host, self.scratch_host, self.dev, self.scratch_dev,
                                      np.array(pairs)) == 0


@pytest.mark.parametrize("caching", [False, True])
@pytest.mark.parametrize("seed", range(4))
def test_swap_stream_keeps_every_sequence_intact(native, seed, caching):
    """Random add / append / fork / free / swap-out / swap-in streams over a
    small pool: after every operation each resident sequence reads back its
    own tokens through its block table, with copy-on-write copies and swap
    copies applied by the oracle, and every invariant of pa_bm_check holds."""
    rng = np.random.Generator(np.random.PCG64(300 + seed))
    nb, nh, b = 40, 48, 4
    cc = native(nb, b, prefix_caching=caching)
    cc.attach_host_pool(nh)
    pools = _Pools(nb, nh, b)
    prompts = [rng.integers(0, 50, size=int(rng.integers(4, 14))).tolist() for _ in range(3)]
    toks, extra, live, swapped, next_id = {}, {}, [], [], 0
    swaps = revivals = 0

    def expect(s):
        return [_tag(extra[s], toks[s][:p + 1]) for p in range(len(toks[s]))]

    for _ in range(400):
        op = int(rng.integers(0, 6))
        if op == 0 or not (live or swapped):
            base = list(prompts[int(rng.integers(0, 3))]) if rng.random() < 0.7 else []
            t = base + rng.integers(0, 50, size=int(rng.integers(0, 9))).tolist()
            ek = int(rng.integers(0, 2))
            r = cc.add_sequence(next_id, len(t), t if caching else None, extra_key=ek)
            if r is not None:
                slots, cached = r
                toks[next_id], extra[next_id] = t, ek
                for p in range(cached, len(t)):
                    pools.write(slots[p], _tag(ek, t[:p + 1]))
                live.append(next_id)
            next_id += 1
        elif op == 1 and live:
            s = live[int(rng.integers(0, len(live)))]
            new = rng.integers(0, 50, size=int(rng.integers(1, 7))).tolist()
            r = cc.append_slots(s, len(new), new if caching else None)
            if r is not None:
                slots, cow = r
                pools.cow(cow)
                for i, tk in enumerate(new):
                    toks[s].append(tk)
                    pools.write(slots[i], _tag(extra[s], toks[s]))
        elif op == 2 and live:
            s = live[int(rng.integers(0, len(live)))]
            cc.fork(s, next_id)
            toks[next_id], extra[next_id] = list(toks[s]), extra[s]
            live.append(next_id)
            next_id += 1
        elif op == 3 and (live or swapped):
            pool = live if (live and (not swapped or rng.random() < 0.5)) else swapped
            s = pool.pop(int(rng.integers(0, len(pool))))
            cc.free_sequence(s)
        elif op == 4 and live:
            k = min(len(live), int(rng.integers(1, 4)))
            group = [live[i] for i in rng.permutation(len(live))[:k]]
            pairs = cc.swap_out(group)
            if pairs is not None:
                pools.swap_out(pairs)
                for s in group:
                    live.remove(s)
                    swapped.append(s)
                    assert cc.is_swapped(s) == 1
                swaps += 1
        elif op == 5 and swapped:
            k = min(len(swapped), int(rng.integers(1, 4)))
            group = [swapped[i] for i in rng.permutation(len(swapped))[:k]]
            blocks = sum(-(-len(toks[s]) // b) for s in group)
            pairs = cc.swap_in(group)
            if pairs is not None:
                pools.swap_in(pairs)
                revivals += len(pairs) < blocks
                for s in group:
                    swapped.remove(s)
                    live.append(s)
                    assert cc.is_swapped(s) == 0
        assert cc.check() == 0
        for s in live:
            assert cc.context_len(s) == len(toks[s])
            assert pools.read(cc.block_table(s), len(toks[s])) == expect(s), s
    assert swaps > 5
    assert revivals > 0 or not caching      # swap-ins that copied fewer blocks than they hold
    for s in live + swapped:
        cc.free_sequence(s)
    assert cc.num_free() == nb and cc.num_free_host() == nh and cc.check() == 0


def test_swap_keeps_a_group_shared(native):
    """Three beams sharing a prompt leave as one host copy per distinct
    block and come back sharing again."""
    cc = native(32, 4)
    cc.attach_host_pool(32)
    cc.add_sequence(0, 10)                   # blocks: 2 full + 1 partial
    cc.fork(0, 1)
    cc.fork(0, 2)
    cc.append_slots(1, 1)                    # copy-on-write of the partial block
    out = cc.swap_out([0, 1, 2])
    assert len(out) == 4 and len({h for _, h in out}) == 4     # 3 shared + beam 1's copy
    assert cc.num_free() == 32 and cc.num_free_host() == 28 and cc.check() == 0
    assert cc.is_swapped(0) == cc.is_swapped(1) == cc.is_swapped(2) == 1
    back = cc.swap_in([0, 1, 2])
    assert len(back) == 4 and cc.num_free_host() == 32 and cc.check() == 0
    t0, t1, t2 = cc.block_table(0), cc.block_table(1), cc.block_table(2)
    assert t0 == t2 and t0[:2] == t1[:2] and t0[2] != t1[2]
    assert [cc.ref(b) for b in t0] == [3, 3, 2] and cc.ref(t1[2]) == 1


def test_swap_in_revives_cached_blocks(native):
    """With prefix caching, full blocks freed by a swap-out keep their
    hashes; swapping back in revives them without a copy while they have not
    been reused, and copies only the partial block and reused ones."""
    cc = native(16, 4, prefix_caching=True)
    cc.attach_host_pool(8)
    toks = list(range(14))                                     # 3 full blocks + 2 tokens
    cc.add_sequence(0, 14, toks)
    table = cc.block_table(0)
    assert len(cc.swap_out([0])) == 4 and cc.num_cached() == 3
    back = cc.swap_in([0])
    assert len(back) == 1 and back[0][1] not in table[:3]
    assert cc.block_table(0)[:3] == table[:3] and cc.check() == 0
    # reuse the freed blocks before swapping in: now every block is copied
    assert len(cc.swap_out([0])) == 4
    cc.add_sequence(1, 64, list(range(100, 164)))             # takes the whole pool
    assert cc.swap_in([0]) is None                             # no room: nothing changes
    assert cc.is_swapped(0) == 1 and cc.check() == 0
    cc.free_sequence(1)
    assert len(cc.swap_in([0])) == 4 and cc.check() == 0


def test_swap_refusals_change_nothing(native):
    cc = native(8, 4)
    with pytest.raises(ValueError):
        cc.swap_out([0])                                       # no host pool yet
    cc.attach_host_pool(2)
    with pytest.raises(ValueError):
        cc.attach_host_pool(4)                                 # only once
    cc.add_sequence(0, 12)                                     # 3 blocks
    cc.add_sequence(1, 4)
    state = (cc.num_free(), cc.num_free_host(), cc.block_table(0), cc.block_table(1))
    assert cc.swap_out([0]) is None                            # 3 blocks > 2 host blocks
    for bad in ([0, 0], [7], []):
        with pytest.raises(ValueError):
            cc.swap_out(bad)
    with pytest.raises(ValueError):
        cc.swap_in([1])                                        # resident
    assert (cc.num_free(), cc.num_free_host(), cc.block_table(0), cc.block_table(1)) == state
    assert len(cc.swap_out([1])) == 1
    for call in (lambda: cc.append_slots(1, 1), lambda: cc.fork(1, 5), lambda: cc.block_table(1)):
        with pytest.raises(ValueError):
            call()
    assert cc.context_len(1) == 4 and cc.check() == 0
    cc.free_sequence(1)                                        # releases its host block
    assert cc.num_free_host() == 2 and cc.is_swapped(1) == -1 and cc.check() == 0


def test_watermark_holds_back_admissions_not_appends(native):
    """With 2 of 10 blocks reserved, a new request (or a swapped group
    coming back) may not take the last 2 free blocks; a running sequence
    may."""
    cc = native(10, 4)
    cc.attach_host_pool(8)
    for bad in (-1, 11):
        with pytest.raises(ValueError):
            cc.set_watermark(bad)
    cc.set_watermark(2)
    assert cc.add_sequence(0, 24) is not None                  # 6 blocks, 4 left
    assert cc.add_sequence(1, 12) is None                      # would leave 1 < 2
    assert cc.add_sequence(1, 8) is not None                   # leaves exactly 2
    assert cc.append_slots(0, 8) is not None and cc.num_free() == 0   # the reserve is usable
    cc.free_sequence(1)
    assert len(cc.swap_out([0])) == 8 and cc.num_free() == 10
    cc.add_sequence(2, 4)                                      # 9 free
    assert cc.swap_in([0]) is None                             # 8 of 9 would leave 1 < 2
    cc.set_watermark(1)
    assert cc.swap_in([0]) is not None and cc.num_free() == 1 and cc.check() == 0


def test_stats_utilisation_and_hit_rate(native):
    """Utilisation counts each stored token once (shared blocks once) over
    the capacity of the blocks in use; the hit rate counts full prompt
    blocks found in the prefix cache."""
    cc = native(32, 4, prefix_caching=True)
    st = cc.stats()
    assert (st.used_blocks, st.stored_tokens, st.prefix_queries) == (0, 0, 0)
    assert st.utilisation == 1.0 and st.hit_rate == 0.0
    prompt = list(range(10))                         # 2 full blocks + 2 tokens
    cc.add_sequence(0, 10, prompt)
    cc.fork(0, 1)                                    # shares all 3 blocks
    st = cc.stats()
    assert (st.used_blocks, st.stored_tokens) == (3, 10) and abs(st.utilisation - 10 / 12) < 1e-12
    cc.append_slots(1, 1, [99])                      # copy-on-write: 3 + 1 blocks, 10 + 3 tokens
    st = cc.stats()
    assert (st.used_blocks, st.stored_tokens, st.num_seqs) == (4, 13, 2)
    cc.add_sequence(2, 13, prompt + [5, 6, 7])       # 3 full blocks: 2 cached, 1 new
    st = cc.stats()
    assert (st.prefix_queries, st.prefix_hits) == (2 + 3, 2) and abs(st.hit_rate - 0.4) < 1e-12
    # the pages' waste bound: every sequence wastes at most block_size - 1 slots
    assert st.used_blocks * 4 - st.stored_tokens <= 3 * st.num_seqs
    assert cc.add_sequence(3, 1000, list(range(1000))) is None      # refused: counters unchanged
    assert cc.stats().prefix_queries == 5


def test_paged_waste_matches_the_pages_figure(native):
    """The page's worked case: LLaMA-7B requests averaging 256 tokens waste
    93.75% of a 4096-token contiguous reservation and under 5% with 16-token
    blocks allocated on demand (utilisation above the 90% target).  Seeded
    lengths uniform in [1, 511] (mean 256), prompts plus appended tokens,
    through the native manager."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "page_figures.json")))["paged_waste_below_5pct"]
    rng = np.random.Generator(np.random.PCG64(415))
    b, n = g["block_size"], 200
    lens = rng.integers(1, 2 * g["mean_tokens"], size=n)
    cc = native(int(sum(-(-int(x) // b) for x in lens)), b)
    for s, total in enumerate(lens):
        prompt = int(rng.integers(1, total + 1))
        assert cc.add_sequence(s, prompt) is not None
        if total > prompt:
            assert cc.append_slots(s, int(total - prompt)) is not None
    st = cc.stats()
    assert st.stored_tokens == int(lens.sum()) and st.free_blocks == 0
    contiguous_waste = 1 - int(lens.sum()) / (n * 4096)
    assert abs(contiguous_waste * 100 - g["contiguous_waste_pct"]) < 1.0
    assert (1 - st.utilisation) * 100 < g["paged_waste_pct_below"]
    assert st.utilisation * 100 > g["utilisation_target_pct"]


def test_high_priority_requests_use_the_reserve(native):
    """Two-level allocation: with 2 of 8 blocks held back, an ordinary request
    is refused where a high-priority one is admitted from the reserve; the
    priority call without priority behaves as pa_bm_add_sequence."""
    cc = native(8, 4)
    cc.set_watermark(2)
    assert cc.add_sequence(0, 24) is not None                  # 6 blocks, 2 left
    assert cc.add_sequence(1, 4) is None                       # ordinary: reserve untouchable
    assert cc.add_sequence(1, 4, high_priority=False) is None
    assert cc.add_sequence(1, 8, high_priority=True) is not None and cc.num_free() == 0
    assert cc.add_sequence(2, 1, high_priority=True) is None   # nothing left at all
    assert cc.check() == 0
