"""Seeded synthetic inputs for the paged decode step.

Holds none of the method's arithmetic: it draws values, lays the logical
per-sequence K/V into the physical pool through the block tables the
allocator model hands out, and records what one decode step must do.

One decode step (every workload):
  1. copy_blocks(block_mapping)           -- copy-on-write copies, if any
  2. reshape_and_cache(new K/V, slots)    -- append this step's tokens
  3. paged_decode(query, ...)             -- attend over context_lens tokens,
                                             the appended tokens included
(the new token is written before attention and is part of the context:
"深入解析 vLLM 的 KV Cache 管理器", 第一部分 KV Cache 的核心价值).

Values are N(0, 1) rounded to the element type.  Physical blocks come from a
seeded permutation of the pool.  Pool slots that hold no token (free blocks,
the tail of a sequence's last block, and the slots this step's tokens will
be written to) hold a NaN bit pattern, so a kernel that reads a slot it must
not read poisons its output.

Random streams: numpy ``Generator(PCG64(4150 + config number))``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from .block_manager import BlockManager

SEED_BASE = 4150
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


def f32_to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to fp16 / bf16 (round to nearest even) and return
    the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def normal_bits(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    return f32_to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)


@dataclass
class DecodeWorkload:
    name: str
    dtype: str                     # "f16" or "bf16"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float                   # an fp32 value
    context_lens: np.ndarray       # int32 [S], after this step's appends
    block_tables: np.ndarray       # int32 [S][max_blocks_per_seq], -1 = unused
    query: np.ndarray              # uint16 [S][Hq][D]
    k_cache: np.ndarray            # uint16 [num_blocks][B][Hkv][D], before the step
    v_cache: np.ndarray
    new_key: np.ndarray            # uint16 [T][Hkv][D]
    new_value: np.ndarray
    slot_mapping: np.ndarray       # int64 [T]
    block_mapping: np.ndarray      # int64 [P][2] (src, dst) copies before the appends
    partition_size: int = 0        # 0 = library's choice
    keys: list | None = None       # logical per-sequence K [ctx][Hkv][D] (small cases)
    values: list | None = None
    extra: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def num_new_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])


def _empty_pool(num_blocks, block_size, hkv, d, dtype):
    shape = (num_blocks, block_size, hkv, d)
    k = np.full(shape, NAN_BITS[dtype], dtype=np.uint16)
    v = np.full(shape, NAN_BITS[dtype], dtype=np.uint16)
    return k, v


def _scatter(pool: np.ndarray, slots: np.ndarray, rows: np.ndarray, block_size: int):
    """pool[slot // B, slot % B] = rows (one [Hkv][D] row per slot)."""
    slots = np.asarray(slots, dtype=np.int64)
    pool[slots // block_size, slots % block_size] = rows


def make_decode(name, *, seed, dtype, context_lens, num_q_heads, num_kv_heads, head_dim,
                block_size, num_blocks, scale, partition_size=0, keep_logical=False,
                max_blocks_per_seq=None):
    """Independent sequences, one new token each (at position ctx - 1).

    Blocks are handed out by the allocator model from a seeded permutation of
    the pool, so every sequence's blocks are scattered."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(context_lens, dtype=np.int32)
    s_n = ctx.shape[0]
    order = rng.permutation(num_blocks)
    mgr = BlockManager(num_blocks, block_size, free_order=order)
    for s in range(s_n):
        if mgr.add_sequence(s, int(ctx[s])) is None:
            raise ValueError(f"{name}: pool of {num_blocks} blocks is too small")
    tables = mgr.block_table_array(range(s_n), max_blocks_per_seq)
    k_cache, v_cache = _empty_pool(num_blocks, block_size, num_kv_heads, head_dim, dtype)

    total = int(ctx.sum())
    row = (num_kv_heads, head_dim)
    keys = normal_bits(rng, (total,) + row, dtype)
    vals = normal_bits(rng, (total,) + row, dtype)
    query = normal_bits(rng, (s_n, num_q_heads, head_dim), dtype)

    starts = np.concatenate([[0], np.cumsum(ctx)[:-1]]).astype(np.int64)
    hist_slots, hist_rows, new_slots, new_rows = [], [], [], []
    for s in range(s_n):
        c = int(ctx[s])
        if c == 0:
            continue
        table = np.asarray(mgr.tables[s], dtype=np.int64)
        pos = np.arange(c, dtype=np.int64)
        slots = table[pos // block_size] * block_size + pos % block_size
        hist_slots.append(slots[:-1])
        hist_rows.append(np.arange(starts[s], starts[s] + c - 1))
        new_slots.append(slots[-1])
        new_rows.append(starts[s] + c - 1)
    if hist_slots:
        hs = np.concatenate(hist_slots)
        hr = np.concatenate(hist_rows)
        _scatter(k_cache, hs, keys[hr], block_size)
        _scatter(v_cache, hs, vals[hr], block_size)
    new_rows = np.asarray(new_rows, dtype=np.int64)
    wl = DecodeWorkload(
        name=name, dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, num_blocks=num_blocks,
        scale=float(np.float32(scale)), context_lens=ctx, block_tables=tables, query=query,
        k_cache=k_cache, v_cache=v_cache,
        new_key=np.ascontiguousarray(keys[new_rows]), new_value=np.ascontiguousarray(vals[new_rows]),
        slot_mapping=np.asarray(new_slots, dtype=np.int64),
        block_mapping=np.zeros((0, 2), dtype=np.int64), partition_size=partition_size)
    if keep_logical:
        wl.keys = [keys[starts[s]:starts[s] + ctx[s]] for s in range(s_n)]
        wl.values = [vals[starts[s]:starts[s] + ctx[s]] for s in range(s_n)]
    wl.extra["manager"] = mgr
    # every sequence appends exactly one token, at position ctx - 1
    wl.extra["one_token_per_seq"] = bool(np.all(ctx > 0))
    return wl


# ---------------------------------------------------------------------------
# FP8 (e4m3) pools: the same workload with its cached K/V held as one-byte
# codes.  The codes are drawn directly (sign, exponent field, mantissa field
# uniform), so nothing here quantises; the step's new tokens stay in the
# 16-bit element type and are quantised by the cache write under test.
# ---------------------------------------------------------------------------

E4M3_NAN = 0x7F


def e4m3_codes(rng: np.random.Generator, shape, max_exponent_field: int = 14) -> np.ndarray:
    """Random e4m3 codes: sign and mantissa uniform, exponent field uniform in
    [0, max_exponent_field] (14 keeps clear of the NaN code 0x7F / 0xFF)."""
    sign = rng.integers(0, 2, size=shape, dtype=np.uint8) << 7
    exp = rng.integers(0, max_exponent_field + 1, size=shape, dtype=np.uint8) << 3
    mant = rng.integers(0, 8, size=shape, dtype=np.uint8)
    return (sign | exp | mant).astype(np.uint8)


def int8_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """Random int8 codes, uniform in [-127, 127]."""
    return rng.integers(-127, 128, size=shape, dtype=np.int8)


# The code every slot without a history token holds: NaN for e4m3 (reading it
# poisons the output), the most negative code for int8 (no NaN exists).
INT8_POISON = -128


def _with_code_pools(wl: DecodeWorkload, seed: int, kv_dtype: str, draw, poison, np_dtype,
                     k_scale: float, v_scale: float) -> DecodeWorkload:
    rng = np.random.Generator(np.random.PCG64(seed))
    b = wl.block_size
    shape = (wl.num_blocks, b, wl.num_kv_heads, wl.head_dim)
    k_cache = np.full(shape, poison, dtype=np_dtype)
    v_cache = np.full(shape, poison, dtype=np_dtype)
    new = set(int(x) for x in wl.slot_mapping if x >= 0)
    slots = []
    for s in range(wl.num_seqs):
        c = int(wl.context_lens[s])
        pos = np.arange(c, dtype=np.int64)
        table = wl.block_tables[s].astype(np.int64)
        slots.extend(int(x) for x in table[pos // b] * b + pos % b if int(x) not in new)
    slots = np.asarray(sorted(set(slots)), dtype=np.int64)
    row = (wl.num_kv_heads, wl.head_dim)
    if slots.size:
        _scatter(k_cache, slots, draw(rng, (slots.size,) + row), b)
        _scatter(v_cache, slots, draw(rng, (slots.size,) + row), b)
    out = DecodeWorkload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    out.name = f"{wl.name}-{kv_dtype}"
    out.k_cache, out.v_cache = k_cache, v_cache
    out.keys = out.values = None
    out.extra = dict(wl.extra, kv_dtype=kv_dtype, k_scale=float(np.float32(k_scale)),
                     v_scale=float(np.float32(v_scale)))
    return out


def with_fp8_pools(wl: DecodeWorkload, seed: int, k_scale: float = 1.0 / 64.0,
                   v_scale: float = 1.0 / 64.0) -> DecodeWorkload:
    """A copy of a make_decode workload whose pools are e4m3 codes: every
    slot that holds a history token gets random codes, every other slot the
    NaN code (so reading a slot the kernel must not read poisons the
    output).  Scales are per pool; with 1/64 the largest code (240) stands
    for 3.75.  extra: kv_dtype = "fp8", k_scale, v_scale."""
    return _with_code_pools(wl, seed, "fp8", e4m3_codes, E4M3_NAN, np.uint8, k_scale, v_scale)


def with_int8_pools(wl: DecodeWorkload, seed: int, k_scale: float = 1.0 / 64.0,
                    v_scale: float = 1.0 / 64.0) -> DecodeWorkload:
    """As with_fp8_pools with int8 codes (uniform in [-127, 127]; slots
    without a history token hold -128).  With scale 1/64 the codes stand for
    values up to about 2.  extra: kv_dtype = "int8", k_scale, v_scale."""
    return _with_code_pools(wl, seed, "int8", int8_codes, INT8_POISON, np.int8, k_scale, v_scale)


def with_rowscale_pools(wl: DecodeWorkload, kv_dtype: str, seed: int) -> DecodeWorkload:
    """A copy of a make_decode workload with one-byte code pools (as
    with_code_pools) and fp32 row-scale pools [num_blocks][Hkv][B]: each
    history row's scale is drawn uniform in [0.5, 2] times a per-kv-head
    magnitude spread geometrically over [1e-2, 1e2], divided by the format's
    top code (448 or 127), so the kv heads differ in magnitude by 10^4.  Every
    scale of a slot without a history token is NaN (reading one poisons the
    output).  The step's new tokens stay N(0,1) in the 16-bit type.
    extra: kv_dtype, rowscale = True, k_scales, v_scales."""
    out = with_code_pools(wl, kv_dtype, seed)
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    nb, b, h = wl.num_blocks, wl.block_size, wl.num_kv_heads
    top = {"fp8": 448.0, "int8": 127.0}[kv_dtype]
    mags = np.geomspace(1e-2, 1e2, h) if h > 1 else np.ones(1)
    history = np.zeros((nb, b), bool)
    new = set(int(x) for x in wl.slot_mapping if x >= 0)
    for s in range(wl.num_seqs):
        c = int(wl.context_lens[s])
        pos = np.arange(c, dtype=np.int64)
        slots = wl.block_tables[s].astype(np.int64)[pos // b] * b + pos % b
        slots = np.asarray([x for x in slots.tolist() if x not in new], dtype=np.int64)
        history[slots // b, slots % b] = True
    scales = []
    for _ in range(2):
        sc = (rng.uniform(0.5, 2.0, (nb, h, b)) * mags[None, :, None] / top).astype(np.float32)
        sc[np.broadcast_to(~history[:, None, :], sc.shape)] = np.nan
        scales.append(np.ascontiguousarray(sc))
    out.name = f"{wl.name}-{kv_dtype}-rows"
    out.extra = dict(out.extra, rowscale=True, k_scales=scales[0], v_scales=scales[1])
    return out


def with_code_pools(wl: DecodeWorkload, kv_dtype: str, seed: int) -> DecodeWorkload:
    """with_fp8_pools or with_int8_pools by name ("fp8" / "int8")."""
    return {"fp8": with_fp8_pools, "int8": with_int8_pools}[kv_dtype](wl, seed=seed)


# ---------------------------------------------------------------------------
# The five workloads.  ``seqs`` shrinks the batch (and ``max_ctx`` the
# contexts) for oracle-sized parity cases; the head layout is unchanged.
# ---------------------------------------------------------------------------

def tiny(keep_logical=True) -> DecodeWorkload:
    """4 sequences, contexts {5, 16, 17, 40}, 2/2 heads, head_dim 64, block 16,
    fp16, 64-block pool, scale 1/8; 4 new tokens; 2 block copies of full,
    untouched blocks into free blocks, with the tables remapped to the copies
    in ``extra['remapped_block_tables']``."""
    wl = make_decode("tiny", seed=SEED_BASE + 1, dtype="f16", context_lens=[5, 16, 17, 40],
                     num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                     num_blocks=64, scale=1.0 / 8.0, keep_logical=keep_logical)
    mgr: BlockManager = wl.extra["manager"]
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + 101))
    # full blocks that this step's new tokens do not touch
    cands = []
    for s in range(wl.num_seqs):
        c = int(wl.context_lens[s])
        for j in range(c // wl.block_size):
            if j != (c - 1) // wl.block_size:
                cands.append((s, j))
    pick = rng.choice(len(cands), size=2, replace=False)
    pairs, remapped = [], wl.block_tables.copy()
    for i in pick:
        s, j = cands[int(i)]
        src = int(wl.block_tables[s, j])
        dst = mgr._take()
        pairs.append((src, dst))
        remapped[s, j] = dst
    wl.block_mapping = np.asarray(pairs, dtype=np.int64)
    wl.extra["remapped_block_tables"] = remapped
    return wl


def llama7b(seqs=64, max_ctx=2048, min_ctx=128, num_blocks=16384,
            keep_logical=False) -> DecodeWorkload:
    """LLaMA-7B-shaped MHA decode: 32/32 heads, head_dim 128, block 16, fp16,
    contexts uniform in [128, 2048], 16384-block pool, scale 1/sqrt(128),
    one new token per sequence."""
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + 2 + 1000))
    ctx = rng.integers(min_ctx, max_ctx, size=seqs, endpoint=True)
    return make_decode("llama7b", seed=SEED_BASE + 2, dtype="f16", context_lens=ctx,
                       num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=16,
                       num_blocks=num_blocks, scale=1.0 / math.sqrt(128.0),
                       keep_logical=keep_logical)


def mistral7b(seqs=256, cap=8192, median=1000.0, sigma=0.6, num_blocks=65536,
              keep_logical=False) -> DecodeWorkload:
    """Mistral-7B-shaped GQA decode: 32 q / 8 kv heads, head_dim 128, block 16,
    bf16, contexts lognormal (median 1000, sigma 0.6, capped at 8192),
    65536-block pool, scale 1/sqrt(128), one new token per sequence."""
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + 3 + 1000))
    ctx = np.clip(np.rint(median * np.exp(sigma * rng.standard_normal(seqs))), 1, cap)
    return make_decode("mistral7b", seed=SEED_BASE + 3, dtype="bf16",
                       context_lens=ctx.astype(np.int32), num_q_heads=32, num_kv_heads=8,
                       head_dim=128, block_size=16, num_blocks=num_blocks,
                       scale=1.0 / math.sqrt(128.0), keep_logical=keep_logical)


def long_context(seqs=16, ctx=32768, num_blocks=40000, partition_size=512,
                 keep_logical=False) -> DecodeWorkload:
    """Long-context split-context decode: contexts of 32768, 32 q / 8 kv heads,
    head_dim 128, block 16, bf16, fully shuffled 40000-block pool, partitions
    of 512 tokens merged by the reduction kernel."""
    return make_decode("long_context", seed=SEED_BASE + 5, dtype="bf16",
                       context_lens=np.full(seqs, ctx, dtype=np.int32), num_q_heads=32,
                       num_kv_heads=8, head_dim=128, block_size=16, num_blocks=num_blocks,
                       scale=1.0 / math.sqrt(128.0), partition_size=partition_size,
                       keep_logical=keep_logical)


def beam_search(prompts=32, beams=4, prompt_len=1000, max_new=256, num_heads=40,
                num_blocks=8192, keep_logical=False) -> DecodeWorkload:
    """LLaMA-2-13B-shaped beam search with block sharing: each prompt's K/V
    is stored once and shared by its beams (reference count = beams); each
    beam then appends 0..max_new divergent tokens.  The writing beams are
    served in order; one that finds the shared partial last block with a
    count above 1 copies it first (the (src, dst) pairs land in
    block_mapping), the last writer finds a count of 1 and writes in place.
    fp16, 40/40 heads, head_dim 128, block 16, scale 1/sqrt(128)."""
    seed = SEED_BASE + 4
    rng = np.random.Generator(np.random.PCG64(seed))
    dtype, b, d = "f16", 16, 128
    mgr = BlockManager(num_blocks, b, free_order=rng.permutation(num_blocks))
    k_cache, v_cache = _empty_pool(num_blocks, b, num_heads, d, dtype)
    row = (num_heads, d)
    n_new = rng.integers(0, max_new, size=(prompts, beams), endpoint=True)
    keys_l, vals_l = [], []
    new_slots, new_k, new_v, cow_pairs = [], [], [], []
    for p in range(prompts):
        base = p * beams
        slots = mgr.add_sequence(base, prompt_len)
        pk = normal_bits(rng, (prompt_len,) + row, dtype)
        pv = normal_bits(rng, (prompt_len,) + row, dtype)
        _scatter(k_cache, np.asarray(slots), pk, b)
        _scatter(v_cache, np.asarray(slots), pv, b)
        for j in range(1, beams):
            mgr.fork(base, base + j)
        for j in range(beams):
            n = int(n_new[p, j])
            res = mgr.append_slots(base + j, n)
            if res is None:
                raise ValueError("beam_search: pool too small")
            sl, cow = res
            cow_pairs.extend(cow)
            nk = normal_bits(rng, (n,) + row, dtype)
            nv = normal_bits(rng, (n,) + row, dtype)
            new_slots.extend(sl)
            new_k.append(nk)
            new_v.append(nv)
            if keep_logical:
                keys_l.append(np.concatenate([pk, nk]))
                vals_l.append(np.concatenate([pv, nv]))
    s_n = prompts * beams
    ctx = np.array([mgr.lens[s] for s in range(s_n)], dtype=np.int32)
    query = normal_bits(rng, (s_n, num_heads, d), dtype)
    wl = DecodeWorkload(
        name="beam_search", dtype=dtype, num_q_heads=num_heads, num_kv_heads=num_heads,
        head_dim=d, block_size=b, num_blocks=num_blocks, scale=float(np.float32(1 / math.sqrt(d))),
        context_lens=ctx, block_tables=mgr.block_table_array(range(s_n)), query=query,
        k_cache=k_cache, v_cache=v_cache,
        new_key=np.concatenate(new_k) if new_k else np.zeros((0,) + row, np.uint16),
        new_value=np.concatenate(new_v) if new_v else np.zeros((0,) + row, np.uint16),
        slot_mapping=np.asarray(new_slots, dtype=np.int64),
        block_mapping=np.asarray(cow_pairs, dtype=np.int64).reshape(-1, 2))
    if keep_logical:
        wl.keys, wl.values = keys_l, vals_l
    wl.extra["manager"] = mgr
    wl.extra["n_new"] = n_new
    # the beams of a prompt share its full blocks (the partial last block is
    # copied on write by every beam but the last writer)
    wl.extra["group_size"] = beams
    wl.extra["prefix_lens"] = np.full(prompts, (prompt_len // b) * b, dtype=np.int32)
    return wl


CONFIGS = {
    "tiny": tiny,
    "llama7b": llama7b,
    "mistral7b": mistral7b,
    "beam_search": beam_search,
    "long_context": long_context,
}
