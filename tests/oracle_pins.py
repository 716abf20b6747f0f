"""Pins of the fp64 oracle: checks against things other than the oracle
itself (numpy / scipy library routines, brute-force loops, closed forms,
invariances the mathematics fixes).  Each pin takes an oracle library handle
so the same battery can run against deliberately broken builds of the
oracle (tests/test_oracle_mutants.py) and must catch every one of them.

Pages cited (title, then section):
  [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
  [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
  [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from oracle import brute
from workloads import generators as gen

F16_ONE = 0x3C00


# ---------------------------------------------------------------- helpers
def pool_after_step(wl):
    """numpy-only: the pools after the step's copies and appends."""
    kc, vc = wl.k_cache.copy(), wl.v_cache.copy()
    for src, dst in wl.block_mapping:
        if src != dst:
            kc[dst] = kc[src]
            vc[dst] = vc[src]
    b = wl.block_size
    sl = wl.slot_mapping
    keep = sl >= 0
    kc[sl[keep] // b, sl[keep] % b] = wl.new_key[keep]
    vc[sl[keep] // b, sl[keep] % b] = wl.new_value[keep]
    return kc, vc


def small_llama(seed_shift=0, seqs=4, max_ctx=300, keep_logical=True):
    return gen.make_decode("llama7b-small", seed=gen.SEED_BASE + 2 + seed_shift, dtype="f16",
                           context_lens=np.random.Generator(np.random.PCG64(7 + seed_shift))
                           .integers(1, max_ctx, size=seqs, endpoint=True),
                           num_q_heads=8, num_kv_heads=8, head_dim=128, block_size=16,
                           num_blocks=160, scale=1 / math.sqrt(128), keep_logical=keep_logical)


def small_gqa(block_size=16, dtype="bf16", seqs=5, head_dim=128, keep_logical=True, kv_heads=2):
    ctx = np.random.Generator(np.random.PCG64(11)).integers(1, 260, size=seqs, endpoint=True)
    nb = int(sum(-(-int(c) // block_size) for c in ctx)) + 16
    return gen.make_decode("gqa-small", seed=gen.SEED_BASE + 3, dtype=dtype, context_lens=ctx,
                           num_q_heads=4 * kv_heads, num_kv_heads=kv_heads, head_dim=head_dim,
                           block_size=block_size, num_blocks=nb, scale=1 / math.sqrt(head_dim),
                           keep_logical=keep_logical)


def small_beams():
    return gen.beam_search(prompts=2, beams=4, prompt_len=40, max_new=24, num_heads=4,
                           num_blocks=64, keep_logical=True)


def run_decode(lib, wl, kc=None, vc=None, tables=None, query=None, ctx=None, blocked=False):
    if kc is None:
        kc, vc = pool_after_step(wl)
    return oracle.paged_decode(wl.query if query is None else query, kc, vc,
                               wl.block_tables if tables is None else tables,
                               wl.context_lens if ctx is None else ctx, wl.scale, wl.dtype,
                               blocked=blocked, lib=lib)


def close(a, b, tol=1e-12):
    assert np.all(np.isfinite(a)), "non-finite oracle output"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol * (1 + np.max(np.abs(b))), f"max abs diff {err:g}"


# ------------------------------------------------------------------- pins
def pin_decode_bits_f16(lib):
    """Every binary16 pattern decodes to numpy's float16 value."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode_bits(bits, "f16", lib=lib)
    assert np.array_equal(got, bits.view(np.float16).astype(np.float64), equal_nan=True)


def pin_decode_bits_bf16(lib):
    """Every bfloat16 pattern decodes to the binary32 with the same upper half."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode_bits(bits, "bf16", lib=lib)
    with np.errstate(invalid="ignore"):
        ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(got, ref, equal_nan=True)


def pin_reshape_layout(lib):
    """One token lands at element ((block*B + offset)*Hkv + h)*D + d of the
    [num_blocks][B][Hkv][D] pool, K from key and V from value; nothing else
    changes; negative slots write nothing; slots past the pool raise bit 2."""
    nb, b, h, d = 5, 4, 3, 8
    kc = np.full((nb, b, h, d), 0xAAAA, np.uint16)
    vc = np.full((nb, b, h, d), 0x5555, np.uint16)
    key = (np.arange(h * d, dtype=np.uint16) + 1).reshape(1, h, d)
    value = key + 1000
    st = oracle.reshape_and_cache(key, value, kc, vc, np.array([2 * b + 3]), b, lib=lib)
    assert st == 0
    fk, fv = kc.reshape(-1), vc.reshape(-1)
    for hh in range(h):
        for dd in range(d):
            off = ((2 * b + 3) * h + hh) * d + dd
            assert fk[off] == key[0, hh, dd] and fv[off] == value[0, hh, dd]
    assert int((fk != 0xAAAA).sum()) == h * d and int((fv != 0x5555).sum()) == h * d
    before_k, before_v = kc.copy(), vc.copy()
    assert oracle.reshape_and_cache(key, value, kc, vc, np.array([-1]), b, lib=lib) == 0
    assert oracle.reshape_and_cache(key, value, kc, vc, np.array([nb * b]), b, lib=lib) == 2
    assert np.array_equal(kc, before_k) and np.array_equal(vc, before_v)


def pin_reshape_matches_scatter(lib):
    """The oracle's cache write of the step's tokens equals numpy fancy-index
    assignment of the same rows into the same slots."""
    for wl in (gen.tiny(), small_beams()):
        kc, vc = wl.k_cache.copy(), wl.v_cache.copy()
        for src, dst in wl.block_mapping:
            kc[dst], vc[dst] = kc[src], vc[src]
        st = oracle.reshape_and_cache(wl.new_key, wl.new_value, kc, vc, wl.slot_mapping,
                                      wl.block_size, lib=lib)
        ek, ev = pool_after_step(wl)
        assert st == 0 and np.array_equal(kc, ek) and np.array_equal(vc, ev)


def pin_copy_blocks(lib):
    """Pairs copy whole K and V blocks in order; src == dst is a no-op; a
    destination used twice, or also used as a source, raises bit 8."""
    rng = np.random.Generator(np.random.PCG64(5))
    kc = rng.integers(0, 65535, size=(6, 4, 2, 8), dtype=np.uint16)
    vc = rng.integers(0, 65535, size=(6, 4, 2, 8), dtype=np.uint16)
    ek, ev = kc.copy(), vc.copy()
    ek[4], ev[4] = kc[1], vc[1]
    ek[3], ev[3] = kc[0], vc[0]
    st = oracle.copy_blocks(kc, vc, np.array([[1, 4], [2, 2], [0, 3]]), lib=lib)
    assert st == 0 and np.array_equal(kc, ek) and np.array_equal(vc, ev)
    assert oracle.copy_blocks(kc.copy(), vc.copy(), np.array([[1, 4], [2, 4]]), lib=lib) & 8
    assert oracle.copy_blocks(kc.copy(), vc.copy(), np.array([[1, 4], [4, 2]]), lib=lib) & 8


def pin_copy_blocks_of_code_pools(lib):
    """One-byte pools (e4m3 or int8 codes) copy whole blocks byte for byte,
    and nothing past the pool: the last block is a destination."""
    rng = np.random.Generator(np.random.PCG64(6))
    for dt in (np.uint8, np.int8):
        kc = rng.integers(0, 256, size=(5, 4, 2, 8), dtype=np.uint8).view(dt)
        vc = rng.integers(0, 256, size=(5, 4, 2, 8), dtype=np.uint8).view(dt)
        ek, ev = kc.copy(), vc.copy()
        ek[4], ev[4] = kc[0], vc[0]
        ek[1], ev[1] = kc[3], vc[3]
        st = oracle.copy_blocks(kc, vc, np.array([[0, 4], [3, 1]]), lib=lib)
        assert st == 0 and np.array_equal(kc, ek) and np.array_equal(vc, ev)


def pin_brute_force_tiny(lib):
    """The tiny workload against element-by-element Python loops."""
    wl = gen.tiny()
    kc, vc = pool_after_step(wl)
    out, st = run_decode(lib, wl, kc, vc)
    ref = brute.brute_paged_decode(wl.query, kc, vc, wl.block_tables, wl.context_lens,
                                   wl.scale, wl.dtype)
    assert st == 0
    close(out, ref)


def pin_contiguous(lib):
    """Paged attention equals textbook softmax(scale q K^T) V (numpy einsum +
    scipy softmax) on the un-paged per-sequence K/V: paging changes only
    where the bytes are ([Manager, 第二部分 PagedAttention 的核心思想])."""
    for wl in (gen.tiny(), small_llama(), small_gqa(), small_gqa(block_size=8, dtype="f16"),
               small_gqa(block_size=32, head_dim=64), small_beams()):
        out, st = run_decode(lib, wl)
        ref = brute.contiguous_attention(wl.query, wl.keys, wl.values, wl.context_lens,
                                         wl.scale, wl.dtype)
        assert st == 0
        close(out, ref)


def pin_permutation_invariance(lib):
    """Relabelling physical blocks (moving every block to pi(b) and mapping
    the tables through pi) leaves the output bit-identical."""
    wl = small_gqa()
    kc, vc = pool_after_step(wl)
    pi = np.random.Generator(np.random.PCG64(3)).permutation(wl.num_blocks)
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[pi], vc2[pi] = kc, vc
    t2 = np.where(wl.block_tables >= 0, pi[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    a, _ = run_decode(lib, wl, kc, vc)
    b, _ = run_decode(lib, wl, kc2, vc2, tables=t2)
    assert np.array_equal(a, b)


def pin_gqa_equals_repeated_mha(lib):
    """Query head h reads kv head h // (Hq/Hkv): GQA equals MHA over K/V with
    every kv head repeated Hq/Hkv times consecutively."""
    wl = small_gqa()
    kc, vc = pool_after_step(wl)
    g = wl.num_q_heads // wl.num_kv_heads
    a, _ = run_decode(lib, wl, kc, vc)
    b, _ = run_decode(lib, wl, np.ascontiguousarray(np.repeat(kc, g, axis=2)),
                      np.ascontiguousarray(np.repeat(vc, g, axis=2)))
    assert np.array_equal(a, b)


def pin_single_token(lib):
    """A one-token context returns that token's V row exactly."""
    wl = small_llama()
    kc, vc = pool_after_step(wl)
    ctx = np.ones(wl.num_seqs, dtype=np.int32)
    out, _ = run_decode(lib, wl, kc, vc, ctx=ctx)
    b = wl.block_size
    for s in range(wl.num_seqs):
        blk = wl.block_tables[s, 0]
        v0 = vc[blk, 0].view(np.float16).astype(np.float64)           # [Hkv][D]
        g = wl.num_q_heads // wl.num_kv_heads
        assert np.array_equal(out[s], np.repeat(v0, g, axis=0)), b


def pin_equal_keys_mean(lib):
    """When every key is the same, the weights are uniform and the output is
    the mean of the V rows."""
    wl = small_llama(seqs=3)
    kc, vc = pool_after_step(wl)
    kc[:] = kc[wl.block_tables[0, 0], 0]
    out, _ = run_decode(lib, wl, kc, vc)
    for s in range(wl.num_seqs):
        v = brute._f64(wl.values[s], wl.dtype)                         # [ctx][Hkv][D]
        close(out[s], v.mean(0))


def pin_closed_form_weights(lib):
    """q = e_0, K_t = a_t e_0, V_t = e_t, scale 1: the output row is the
    softmax of (a_t), i.e. exp(a_t) / sum exp(a_u), in closed form."""
    a = [0.0, 1.0, 2.0, -1.5, 0.5, 3.0, 2.0, -4.0, 0.0, 1.0, 1.25, -0.75, 2.5, 0.0, 0.0, 1.0,
         0.5, -2.0, 3.5]                                              # 19 tokens: ragged tail
    n, d, b = len(a), 32, 16
    kc = np.zeros((4, b, 1, d), np.uint16)
    vc = np.zeros((4, b, 1, d), np.uint16)
    table = np.array([[2, 0, -1]], np.int32)
    for t in range(n):
        blk, off = table[0, t // b], t % b
        kc[blk, off, 0, 0] = np.float16(a[t]).view(np.uint16)
        vc[blk, off, 0, t] = F16_ONE
    q = np.zeros((1, 1, d), np.uint16)
    q[0, 0, 0] = F16_ONE
    out, st = oracle.paged_decode(q, kc, vc, table, np.array([n], np.int32), 1.0, "f16", lib=lib)
    z = sum(math.exp(x) for x in a)
    ref = np.zeros(d)
    ref[:n] = [math.exp(x) / z for x in a]
    assert st == 0
    close(out[0, 0], ref, tol=1e-14)


def pin_blocked_equals_direct(lib):
    """The five blocked-softmax steps of [Practice §5.1 分块Softmax算法] give
    the direct softmax result."""
    for wl in (small_gqa(block_size=8), small_gqa(block_size=32), small_llama()):
        a, _ = run_decode(lib, wl)
        b, _ = run_decode(lib, wl, blocked=True)
        close(b, a)


def pin_large_magnitude(lib):
    """Scores of several thousand (q scaled by 1000) stay finite thanks to the
    max subtraction, and each output is a convex combination of V rows.  The
    blocked form agrees there too: only at such scores does a global max
    that misses a block (or part of one) change the result, by overflow."""
    wl = small_llama(seqs=3)
    q = (wl.query.view(np.float16).astype(np.float32) * 1000).astype(np.float16).view(np.uint16)
    kc, vc = pool_after_step(wl)
    out, _ = run_decode(lib, wl, kc, vc, query=q)
    assert np.all(np.isfinite(out))
    for s in range(wl.num_seqs):
        v = brute._f64(wl.values[s], wl.dtype)
        assert np.all(out[s] >= v.min(0) - 1e-9) and np.all(out[s] <= v.max(0) + 1e-9)
    blocked, _ = run_decode(lib, wl, kc, vc, query=q, blocked=True)
    assert np.all(np.isfinite(blocked))
    close(blocked, out)


def pin_blocked_max_in_last_block(lib):
    """The blocked form's global max must cover every block and every token
    of a block: each head's query points along its sequence's newest key
    (x 100, so its score is in the thousands and every other far below),
    which sits in the last block and not at a block's first position.  A
    max that missed it would overflow; blocked and direct agree instead."""
    wl = gen.make_decode("blocked-max", seed=gen.SEED_BASE + 9, dtype="f16",
                         context_lens=[37, 70, 100], num_q_heads=4, num_kv_heads=4,
                         head_dim=128, block_size=16, num_blocks=24, scale=1 / math.sqrt(128),
                         keep_logical=False)
    assert wl.extra["one_token_per_seq"] and all((c - 1) % 16 for c in wl.context_lens)
    kc, vc = pool_after_step(wl)
    q = (wl.new_key.view(np.float16).astype(np.float32) * 100).astype(np.float16).view(np.uint16)
    direct, _ = run_decode(lib, wl, kc, vc, query=q)
    blocked, _ = run_decode(lib, wl, kc, vc, query=q, blocked=True)
    assert np.all(np.isfinite(direct)) and np.all(np.isfinite(blocked))
    close(blocked, direct)
    # the newest token dominates: the output is (about) its value row
    newest = wl.new_value.view(np.float16).astype(np.float64)
    assert np.max(np.abs(direct - newest)) < 1e-6


def pin_edge_contexts(lib):
    """Empty context -> zero row, status 0; negative or longer-than-table
    context -> zero row, bit 4; a table entry outside the pool -> bit 1 and
    that block's tokens are left out of the softmax."""
    wl = small_llama(seqs=4)
    kc, vc = pool_after_step(wl)
    ctx = wl.context_lens.copy()
    ctx[0] = 0
    out, st = run_decode(lib, wl, kc, vc, ctx=ctx)
    assert st == 0 and not out[0].any()
    ctx[0] = -3
    out, st = run_decode(lib, wl, kc, vc, ctx=ctx)
    assert st == 4 and not out[0].any()
    ctx[0] = wl.max_blocks_per_seq * wl.block_size + 1
    out, st = run_decode(lib, wl, kc, vc, ctx=ctx)
    assert st == 4 and not out[0].any()
    # drop block 0 of the longest sequence
    s = int(np.argmax(wl.context_lens))
    tables = wl.block_tables.copy()
    tables[s, 0] = wl.num_blocks + 7
    out, st = run_decode(lib, wl, kc, vc, tables=tables)
    assert st == 1
    b = wl.block_size
    keys = [k[b:] if i == s else k for i, k in enumerate(wl.keys)]
    vals = [v[b:] if i == s else v for i, v in enumerate(wl.values)]
    lens = np.array([len(k) for k in keys], np.int32)
    ref = brute.contiguous_attention(wl.query, keys, vals, lens, wl.scale, wl.dtype)
    close(out, ref)


def pin_rows_match_full(lib):
    """The sampled-row entry point returns exactly the full run's rows."""
    wl = small_gqa()
    kc, vc = pool_after_step(wl)
    full, _ = run_decode(lib, wl, kc, vc)
    rows = np.array([[0, 0], [2, 5], [4, 7], [1, 3]], np.int32)
    got, _ = oracle.paged_decode_rows(rows, wl.query, kc, vc, wl.block_tables,
                                      wl.context_lens, wl.scale, wl.dtype, lib=lib)
    assert np.array_equal(got, full[rows[:, 0], rows[:, 1]])


# ---- FP8 (e4m3) caches ------------------------------------------------------

def _torch_e4m3():
    import torch
    return torch


def pin_e4m3_decode_all_codes(lib):
    """Every e4m3 code decodes to torch.float8_e4m3fn's value."""
    torch = _torch_e4m3()
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.decode_e4m3(codes, lib=lib), ref, equal_nan=True)


def pin_e4m3_encode_rounding(lib):
    """fp32 -> e4m3 rounds to nearest, ties to even (torch.float8_e4m3fn for
    in-range values, including every exact midpoint); saturates at +-448;
    keeps the sign of zero; NaN -> 0x7F."""
    torch = _torch_e4m3()
    codes = np.arange(0, 0x7f, dtype=np.uint8)                 # finite non-negative codes
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.Generator(np.random.PCG64(8))
    x = np.concatenate([vals, mids, rng.uniform(-447, 447, 4000), rng.normal(0, 0.01, 2000)])
    x = np.concatenate([x, -x]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.encode_e4m3(x, lib=lib), ref)
    sat = np.array([448.0, 449.0, 1e6, -500.0, np.inf, -np.inf, np.nan, -0.0, 0.0], np.float32)
    assert oracle.encode_e4m3(sat, lib=lib).tolist() == [0x7e, 0x7e, 0x7e, 0xfe, 0x7e, 0xfe,
                                                         0x7f, 0x80, 0x00]


def pin_fp8_cache_write(lib):
    """The quantising write stores e4m3(fp32(x) * fp32(1/scale)) at the slot's
    offset; other bytes unchanged."""
    rng = np.random.Generator(np.random.PCG64(9))
    nb, b, h, d = 6, 4, 2, 8
    kc = np.full((nb, b, h, d), 0x7f, np.uint8)
    vc = np.full((nb, b, h, d), 0x7f, np.uint8)
    key = gen.normal_bits(rng, (3, h, d), "f16")
    val = gen.normal_bits(rng, (3, h, d), "f16")
    slots = np.array([5, -1, 17])
    st = oracle.reshape_and_cache_fp8(key, val, kc, vc, slots, b, "f16", 0.05, 0.03, lib=lib)
    assert st == 0
    inv_k, inv_v = np.float32(1) / np.float32(0.05), np.float32(1) / np.float32(0.03)
    for t, sl in ((0, 5), (2, 17)):
        kx = key[t].view(np.float16).astype(np.float32) * inv_k
        vx = val[t].view(np.float16).astype(np.float32) * inv_v
        assert np.array_equal(kc[sl // b, sl % b], oracle.encode_e4m3(kx, lib=lib))
        assert np.array_equal(vc[sl // b, sl % b], oracle.encode_e4m3(vx, lib=lib))
    touched = np.zeros((nb, b), bool)
    touched[1, 1] = touched[4, 1] = True
    assert np.all(kc[~touched] == 0x7f) and np.all(vc[~touched] == 0x7f)


def pin_fp8_decode_equals_dequantised_fp16(lib):
    """With power-of-two scales the dequantised cache is exact in fp16, so the
    fp8 decode must equal the (pinned) fp16 decode of the dequantised pools."""
    rng = np.random.Generator(np.random.PCG64(10))
    wl = small_gqa(dtype="f16")
    codes_k = rng.integers(0, 256, size=wl.k_cache.shape).astype(np.uint8)
    codes_v = rng.integers(0, 256, size=wl.v_cache.shape).astype(np.uint8)
    for c in (codes_k, codes_v):
        c[(c & 0x7f) == 0x7f] = 0x3c                            # no NaN codes
    ks, vs = 0.25, 0.5
    deq_k = (oracle.decode_e4m3(codes_k, lib=lib) * ks).astype(np.float16).view(np.uint16)
    deq_v = (oracle.decode_e4m3(codes_v, lib=lib) * vs).astype(np.float16).view(np.uint16)
    a, sa = oracle.paged_decode_fp8(wl.query, codes_k, codes_v, wl.block_tables, wl.context_lens,
                                    wl.scale, "f16", ks, vs, lib=lib)
    b, sb = oracle.paged_decode(wl.query, deq_k, deq_v, wl.block_tables, wl.context_lens,
                                wl.scale, "f16", lib=lib)
    assert sa == sb == 0
    assert np.array_equal(a, b)


def pin_fp8_decode_matches_numpy_attention(lib):
    """Scales that are not powers of two: the fp8 decode equals numpy
    softmax attention over K/V gathered through the tables and dequantised
    with torch's e4m3 decoding times the scales (<= 1e-12)."""
    torch = _torch_e4m3()
    from scipy.special import softmax
    wl = small_gqa(dtype="bf16", seqs=4, head_dim=64)
    rng = np.random.Generator(np.random.PCG64(15))
    kc = rng.integers(0, 256, size=wl.k_cache.shape).astype(np.uint8)
    vc = rng.integers(0, 256, size=wl.v_cache.shape).astype(np.uint8)
    for c in (kc, vc):
        c[(c & 0x7f) == 0x7f] = 0x11                             # no NaN codes
    ks, vs = 0.0371, 0.2113
    got, st = oracle.paged_decode_fp8(wl.query, kc, vc, wl.block_tables, wl.context_lens,
                                      wl.scale, wl.dtype, ks, vs, lib=lib)
    assert st == 0
    deq = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    q = (torch.from_numpy(wl.query.view(np.int16)).view(torch.bfloat16)
         .to(torch.float64).numpy())
    b, group = wl.block_size, wl.num_q_heads // wl.num_kv_heads
    for s in range(wl.num_seqs):
        c = int(wl.context_lens[s])
        pos = np.arange(c)
        phys = wl.block_tables[s][pos // b]
        k = np.repeat(deq(kc[phys, pos % b]) * ks, group, axis=1)      # scales as given
        v = np.repeat(deq(vc[phys, pos % b]) * vs, group, axis=1)
        w = softmax(wl.scale * np.einsum("hd,thd->ht", q[s], k), axis=1)
        close(got[s], np.einsum("ht,thd->hd", w, v), 1e-12)


# ---- INT8 caches ---------------------------------------------------------------

def pin_int8_decode_all_codes(lib):
    """Every byte decodes to its two's-complement value (numpy's int8 view)."""
    codes = np.arange(256, dtype=np.uint8)
    assert np.array_equal(oracle.decode_int8(codes, lib=lib),
                          codes.view(np.int8).astype(np.float64))


def pin_int8_encode_rounding(lib):
    """fp32 -> int8 agrees with torch.round (ties to even) clamped to
    [-128, 127] on random values, every integer and every midpoint of the
    range; beyond it saturates (inf too) and NaN gives 0."""
    import torch
    rng = np.random.Generator(np.random.PCG64(16))
    ints = np.arange(-128, 128, dtype=np.float64)
    x = np.concatenate([ints, ints[:-1] + 0.5, rng.uniform(-130, 130, 4000),
                        rng.normal(0, 2, 2000)]).astype(np.float32)
    ref = torch.clamp(torch.round(torch.from_numpy(x)), -128, 127).to(torch.int8).numpy()
    assert np.array_equal(oracle.encode_int8(x, lib=lib), ref)
    assert np.array_equal(oracle.encode_int8(ints.astype(np.float32), lib=lib),
                          ints.astype(np.int8))
    special = np.array([127.4, 127.5, 127.6, 128.0, 1e6, np.inf, -128.4, -128.5, -129.0, -np.inf,
                        np.nan, 0.5, -0.5, 1.5, -2.5], np.float32)
    assert oracle.encode_int8(special, lib=lib).tolist() == [127, 127, 127, 127, 127, 127, -128,
                                                             -128, -128, -128, 0, 0, 0, 2, -2]


def pin_int8_cache_write(lib):
    """The quantising write stores int8(fp32(x) * fp32(1/scale)) at the slot's
    offset; other bytes unchanged; a slot past the pool is flagged."""
    rng = np.random.Generator(np.random.PCG64(17))
    nb, b, h, d = 6, 4, 2, 8
    kc = np.full((nb, b, h, d), 0x55, np.uint8).view(np.int8)
    vc = np.full((nb, b, h, d), 0x55, np.uint8).view(np.int8)
    key = gen.normal_bits(rng, (3, h, d), "bf16")
    val = gen.normal_bits(rng, (3, h, d), "bf16")
    slots = np.array([5, -1, 17])
    st = oracle.reshape_and_cache_int8(key, val, kc, vc, slots, b, "bf16", 0.02, 0.03, lib=lib)
    assert st == 0
    inv_k, inv_v = np.float32(1) / np.float32(0.02), np.float32(1) / np.float32(0.03)
    as_f32 = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32)   # bf16 -> fp32, exact
    for t, sl in ((0, 5), (2, 17)):
        assert np.array_equal(kc[sl // b, sl % b], oracle.encode_int8(as_f32(key[t]) * inv_k, lib=lib))
        assert np.array_equal(vc[sl // b, sl % b], oracle.encode_int8(as_f32(val[t]) * inv_v, lib=lib))
    touched = np.zeros((nb, b), bool)
    touched[1, 1] = touched[4, 1] = True
    assert np.all(kc[~touched] == 0x55) and np.all(vc[~touched] == 0x55)
    assert oracle.reshape_and_cache_int8(key, val, kc, vc, np.array([nb * b, 0, 1]), b, "bf16",
                                         0.02, 0.03, lib=lib) == 2


def pin_int8_decode_equals_dequantised_fp16(lib):
    """With power-of-two scales every code x scale is exact in fp16, so the
    int8 decode must equal the (pinned) fp16 decode of the dequantised pools."""
    rng = np.random.Generator(np.random.PCG64(18))
    wl = small_gqa(dtype="f16")
    codes_k = rng.integers(-128, 128, size=wl.k_cache.shape).astype(np.int8)
    codes_v = rng.integers(-128, 128, size=wl.v_cache.shape).astype(np.int8)
    ks, vs = 2.0 ** -6, 2.0 ** -5
    deq_k = (codes_k.astype(np.float64) * ks).astype(np.float16).view(np.uint16)
    deq_v = (codes_v.astype(np.float64) * vs).astype(np.float16).view(np.uint16)
    a, sa = oracle.paged_decode_int8(wl.query, codes_k, codes_v, wl.block_tables, wl.context_lens,
                                     wl.scale, "f16", ks, vs, lib=lib)
    b, sb = oracle.paged_decode(wl.query, deq_k, deq_v, wl.block_tables, wl.context_lens,
                                wl.scale, "f16", lib=lib)
    assert sa == sb == 0
    assert np.array_equal(a, b)


def pin_int8_decode_matches_numpy_attention(lib):
    """Scales that are not powers of two: the int8 decode equals numpy
    softmax attention over K/V gathered through the tables, dequantised as
    code x scale (<= 1e-12)."""
    from scipy.special import softmax
    wl = small_gqa(dtype="f16", seqs=4, head_dim=64)
    rng = np.random.Generator(np.random.PCG64(19))
    kc = rng.integers(-128, 128, size=wl.k_cache.shape).astype(np.int8)
    vc = rng.integers(-128, 128, size=wl.v_cache.shape).astype(np.int8)
    ks, vs = 0.0173, 0.0291
    got, st = oracle.paged_decode_int8(wl.query, kc, vc, wl.block_tables, wl.context_lens,
                                       wl.scale, wl.dtype, ks, vs, lib=lib)
    assert st == 0
    q = wl.query.view(np.float16).astype(np.float64)
    b, group = wl.block_size, wl.num_q_heads // wl.num_kv_heads
    for s in range(wl.num_seqs):
        c = int(wl.context_lens[s])
        pos = np.arange(c)
        phys = wl.block_tables[s][pos // b]
        k = np.repeat(kc[phys, pos % b].astype(np.float64) * ks, group, axis=1)
        v = np.repeat(vc[phys, pos % b].astype(np.float64) * vs, group, axis=1)
        w = softmax(wl.scale * np.einsum("hd,thd->ht", q[s], k), axis=1)
        close(got[s], np.einsum("ht,thd->hd", w, v), 1e-12)


# ---- swap_blocks (eviction to host memory and back) ---------------------------

def pin_swap_round_trip(lib):
    """Swapping blocks out to a second pool and back through the inverse
    mapping restores the first pool exactly; destination blocks outside the
    mapping keep their bytes."""
    rng = np.random.Generator(np.random.PCG64(12))
    dev_k = rng.integers(0, 65536, size=(9, 4, 2, 8), dtype=np.uint16)
    dev_v = rng.integers(0, 65536, size=(9, 4, 2, 8), dtype=np.uint16)
    host_k = rng.integers(0, 65536, size=(5, 4, 2, 8), dtype=np.uint16)
    host_v = rng.integers(0, 65536, size=(5, 4, 2, 8), dtype=np.uint16)
    out = np.array([[7, 0], [2, 3], [5, 1]])
    hk0, hv0 = host_k.copy(), host_v.copy()
    assert oracle.swap_blocks(dev_k, dev_v, host_k, host_v, out, lib=lib) == 0
    for blk in (2, 4):
        assert np.array_equal(host_k[blk], hk0[blk]) and np.array_equal(host_v[blk], hv0[blk])
    back_k = np.zeros_like(dev_k)
    back_v = np.zeros_like(dev_v)
    assert oracle.swap_blocks(host_k, host_v, back_k, back_v, out[:, ::-1], lib=lib) == 0
    for src, _ in out:
        assert np.array_equal(back_k[src], dev_k[src]) and np.array_equal(back_v[src], dev_v[src])


def pin_swap_equals_copy_on_joined_pool(lib):
    """A swap between two pools is copy_blocks on the pool made of both, with
    destination ids shifted past the source pool (copy_blocks is pinned by
    its own definition above); statuses agree, including a bad id and a
    repeated destination."""
    rng = np.random.Generator(np.random.PCG64(13))
    a_k = rng.integers(0, 65536, size=(6, 4, 2, 8), dtype=np.uint16)
    a_v = rng.integers(0, 65536, size=(6, 4, 2, 8), dtype=np.uint16)
    b_k = rng.integers(0, 65536, size=(4, 4, 2, 8), dtype=np.uint16)
    b_v = rng.integers(0, 65536, size=(4, 4, 2, 8), dtype=np.uint16)
    for pairs, want in (([[0, 3], [5, 0], [2, 1]], 0), ([[1, 2], [4, 2]], 8), ([[-1, 0], [3, 1]], 1)):
        m = np.array(pairs, dtype=np.int64)
        jk, jv = np.concatenate([a_k, b_k]), np.concatenate([a_v, b_v])
        mj = m.copy()
        mj[:, 1] += a_k.shape[0]
        st_copy = oracle.copy_blocks(jk, jv, mj, lib=lib)
        dk, dv = b_k.copy(), b_v.copy()
        st_swap = oracle.swap_blocks(a_k, a_v, dk, dv, m, lib=lib)
        assert st_swap == st_copy == want
        assert np.array_equal(dk, jk[a_k.shape[0]:]) and np.array_equal(dv, jv[a_k.shape[0]:])


def pin_swap_bytes_of_fp8_pools(lib):
    """One-byte pools swap as bytes: the same data seen as 16-bit pairs
    swaps identically."""
    rng = np.random.Generator(np.random.PCG64(14))
    src_k = rng.integers(0, 256, size=(5, 4, 2, 16), dtype=np.uint8)
    src_v = rng.integers(0, 256, size=(5, 4, 2, 16), dtype=np.uint8)
    dst_k = rng.integers(0, 256, size=(3, 4, 2, 16), dtype=np.uint8)
    dst_v = rng.integers(0, 256, size=(3, 4, 2, 16), dtype=np.uint8)
    m = np.array([[4, 0], [1, 2]])
    w_k, w_v = dst_k.copy().view(np.uint16), dst_v.copy().view(np.uint16)
    assert oracle.swap_blocks(src_k, src_v, dst_k, dst_v, m, lib=lib) == 0
    assert oracle.swap_blocks(src_k.view(np.uint16), src_v.view(np.uint16), w_k, w_v, m,
                              lib=lib) == 0
    assert np.array_equal(dst_k, w_k.view(np.uint8)) and np.array_equal(dst_v, w_v.view(np.uint8))
    assert np.array_equal(dst_k[0], src_k[4]) and np.array_equal(dst_v[2], src_v[1])
    # an id past either pool is flagged and its pair skipped
    before = dst_k.copy()
    assert oracle.swap_blocks(src_k, src_v, dst_k, dst_v, np.array([[0, 3]]), lib=lib) == 1
    assert oracle.swap_blocks(src_k, src_v, dst_k, dst_v, np.array([[5, 0]]), lib=lib) == 1
    assert np.array_equal(dst_k, before)


# ---- Row-scaled one-byte caches: one fp32 scale per (token, kv head) row ---------

_CODE_MAX = {"fp8": 448.0, "int8": 127.0}


def _dec_codes(codes, fmt):
    """Codes -> float64 with torch's e4m3 decoding or numpy's int8 view."""
    if fmt == "int8":
        return np.ascontiguousarray(codes).view(np.int8).astype(np.float64)
    torch = _torch_e4m3()
    return (torch.from_numpy(np.ascontiguousarray(codes).view(np.uint8))
            .view(torch.float8_e4m3fn).to(torch.float64).numpy())


def _rows_of_mixed_magnitude(rng, t, h, d, dtype="f16"):
    """[t][h][d] 16-bit values whose kv heads differ in magnitude by up to
    10^4 (x1, x0.01, x100, ...), with one all-zero row."""
    mags = np.array([1.0, 0.01, 100.0, 3.0])[:h].astype(np.float32)
    x = rng.standard_normal((t, h, d)).astype(np.float32) * mags[None, :, None]
    x[-1, 1 % h] = 0.0
    return gen.f32_to_bits(x, dtype)


def pin_rowscale_cache_write(lib):
    """The row-scaled write, both code formats: each written row's scale is
    fp32(max |x| / code_max); its codes are those of the (pinned) per-pool
    write with that scale; its largest element takes the top code; the
    dequantised row is within half a code step of the input; an all-zero
    row stores scale 0 and zero codes; a slot past the pool sets bit 2;
    every other code and scale byte is unchanged."""
    rng = np.random.Generator(np.random.PCG64(31))
    nb, b, h, d = 6, 4, 3, 16
    for fmt in ("fp8", "int8"):
        np_t = np.uint8 if fmt == "fp8" else np.int8
        write = getattr(oracle, f"reshape_and_cache_{fmt}_rowscale")
        pool_write = getattr(oracle, f"reshape_and_cache_{fmt}")
        poison = np.array(0x7f, np.uint8).view(np_t)
        kc = np.full((nb, b, h, d), poison, np_t)
        vc = kc.copy()
        ks = np.full((nb, h, b), -7.0, np.float32)
        vs = ks.copy()
        key = _rows_of_mixed_magnitude(rng, 4, h, d)
        val = _rows_of_mixed_magnitude(rng, 4, h, d)
        slots = np.array([5, -1, 17, 22])
        st = write(key, val, kc, vc, ks, vs, slots, b, "f16", lib=lib)
        assert st == 0
        assert write(key[:1], val[:1], kc.copy(), vc.copy(), ks.copy(), vs.copy(),
                     np.array([nb * b]), b, "f16", lib=lib) == 2
        top = _CODE_MAX[fmt]
        for t, sl in ((0, 5), (2, 17), (3, 22)):
            blk, off = sl // b, sl % b
            for src, pool, scales in ((key, kc, ks), (val, vc, vs)):
                for g in range(h):
                    x = src[t, g].view(np.float16).astype(np.float32)
                    s = scales[blk, g, off]
                    amax = np.float32(np.max(np.abs(x)))
                    if amax == 0:
                        assert s == 0 and not pool[blk, off, g].view(np.uint8).any()
                        continue
                    assert s == amax / np.float32(top), (fmt, t, g)
                    one = np.full((1, 1, 1, d), poison, np_t)
                    pool_write(src[t:t + 1, g:g + 1], src[t:t + 1, g:g + 1], one, one.copy(),
                               np.array([0]), 1, "f16", float(s), float(s), lib=lib)
                    assert np.array_equal(pool[blk, off, g], one[0, 0, 0]), (fmt, t, g)
                    deq = _dec_codes(pool[blk, off, g], fmt) * float(s)
                    assert abs(deq[np.argmax(np.abs(x))]) == top * float(s)
                    step = float(s) * (1.0 if fmt == "int8" else 2.0 ** -9)
                    rel = 0.0 if fmt == "int8" else 2.0 ** -4
                    bound = step / 2 + rel * np.abs(x) + 1e-6 * np.abs(x)
                    assert np.all(np.abs(deq - x) <= bound), (fmt, t, g)
        touched = np.zeros((nb, b), bool)
        for sl in (5, 17, 22):
            touched[sl // b, sl % b] = True
        assert np.all(kc[~touched].view(np.uint8) == 0x7f)
        assert np.all(vc[~touched].view(np.uint8) == 0x7f)
        untouched = np.ones((nb, h, b), bool)
        for sl in (5, 17, 22):
            untouched[sl // b, :, sl % b] = False
        assert np.all(ks[untouched] == -7.0) and np.all(vs[untouched] == -7.0)


def _random_rowscale_pools(rng, wl, fmt):
    """Random codes (no NaN) and positive row scales spanning four orders of
    magnitude across kv heads."""
    shape = wl.k_cache.shape
    pools = []
    for _ in range(2):
        c = rng.integers(0, 256, size=shape).astype(np.uint8)
        if fmt == "fp8":
            c[(c & 0x7f) == 0x7f] = 0x35
        pools.append(c.view(np.uint8 if fmt == "fp8" else np.int8))
    nb, b, h, _ = shape
    mags = np.geomspace(1e-2, 1e2, h).astype(np.float32)
    scales = [(rng.uniform(0.5, 2.0, (nb, h, b)).astype(np.float32) * mags[None, :, None]
               / np.float32(_CODE_MAX[fmt])).astype(np.float32) for _ in range(2)]
    return pools, scales


def pin_rowscale_decode_matches_numpy_attention(lib):
    """Row-scaled decode, both formats: numpy softmax attention over K/V
    gathered through the tables, each row dequantised with its own scale
    from [block][kv head][offset] (<= 1e-12)."""
    from scipy.special import softmax
    rng = np.random.Generator(np.random.PCG64(32))
    for fmt in ("fp8", "int8"):
        wl = small_gqa(dtype="bf16", seqs=4, head_dim=64)
        (kc, vc), (ks, vs) = _random_rowscale_pools(rng, wl, fmt)
        decode = getattr(oracle, f"paged_decode_{fmt}_rowscale")
        got, st = decode(wl.query, kc, vc, ks, vs, wl.block_tables, wl.context_lens, wl.scale,
                         wl.dtype, lib=lib)
        assert st == 0
        q = oracle.decode_bits(wl.query, "bf16", lib=lib)
        b, group = wl.block_size, wl.num_q_heads // wl.num_kv_heads
        for s in range(wl.num_seqs):
            c = int(wl.context_lens[s])
            pos = np.arange(c)
            phys = wl.block_tables[s][pos // b]
            k = _dec_codes(kc[phys, pos % b], fmt) * ks[phys, :, pos % b][:, :, None]
            v = _dec_codes(vc[phys, pos % b], fmt) * vs[phys, :, pos % b][:, :, None]
            k, v = np.repeat(k, group, axis=1), np.repeat(v, group, axis=1)
            w = softmax(wl.scale * np.einsum("hd,thd->ht", q[s], k), axis=1)
            close(got[s], np.einsum("ht,thd->hd", w, v), 1e-12)


def pin_rowscale_constant_scales_equal_pool_scales(lib):
    """Scale pools holding one value everywhere give exactly the (pinned)
    per-pool decode with that scale, and the row-scaled write of rows whose
    scales all come out equal gives the per-pool write's codes."""
    rng = np.random.Generator(np.random.PCG64(33))
    for fmt in ("fp8", "int8"):
        wl = small_gqa(dtype="f16")
        (kc, vc), _ = _random_rowscale_pools(rng, wl, fmt)
        nb, b, h, _ = kc.shape
        ks = np.full((nb, h, b), 0.0371, np.float32)
        vs = np.full((nb, h, b), 0.2113, np.float32)
        a, sa = getattr(oracle, f"paged_decode_{fmt}_rowscale")(
            wl.query, kc, vc, ks, vs, wl.block_tables, wl.context_lens, wl.scale, "f16", lib=lib)
        p, sp = getattr(oracle, f"paged_decode_{fmt}")(
            wl.query, kc, vc, wl.block_tables, wl.context_lens, wl.scale, "f16",
            float(ks[0, 0, 0]), float(vs[0, 0, 0]), lib=lib)
        assert sa == sp == 0 and np.array_equal(a, p)


def pin_rowscale_permutation_invariance(lib):
    """Relabelling physical blocks -- codes and scales moved together, tables
    remapped -- leaves the row-scaled decode bit-identical."""
    rng = np.random.Generator(np.random.PCG64(34))
    for fmt in ("fp8", "int8"):
        wl = small_gqa(dtype="bf16")
        (kc, vc), (ks, vs) = _random_rowscale_pools(rng, wl, fmt)
        decode = getattr(oracle, f"paged_decode_{fmt}_rowscale")
        a, _ = decode(wl.query, kc, vc, ks, vs, wl.block_tables, wl.context_lens, wl.scale,
                      wl.dtype, lib=lib)
        perm = rng.permutation(kc.shape[0])            # new id of old block i is perm[i]
        inv = np.argsort(perm)
        tables = np.where(wl.block_tables >= 0, perm[np.maximum(wl.block_tables, 0)], -1)
        moved = [np.ascontiguousarray(x[inv]) for x in (kc, vc, ks, vs)]
        b2, _ = decode(wl.query, *moved, tables.astype(np.int32), wl.context_lens, wl.scale,
                       wl.dtype, lib=lib)
        assert np.array_equal(a, b2)


def pin_rowscale_pools_copy_and_swap_as_blocks(lib):
    """Scale pools move with their blocks: copy_blocks and swap_blocks on a
    [num_blocks][Hkv][B] fp32 pool copy whole blocks of scales."""
    rng = np.random.Generator(np.random.PCG64(35))
    ks = rng.uniform(0, 1, (6, 3, 4)).astype(np.float32)
    vs = rng.uniform(0, 1, (6, 3, 4)).astype(np.float32)
    k0, v0 = ks.copy(), vs.copy()
    assert oracle.copy_blocks(ks, vs, np.array([[1, 4], [2, 5]]), lib=lib) == 0
    assert np.array_equal(ks[4], k0[1]) and np.array_equal(vs[5], v0[2])
    assert np.array_equal(ks[:4], k0[:4])
    hk, hv = np.zeros((2, 3, 4), np.float32), np.zeros((2, 3, 4), np.float32)
    assert oracle.swap_blocks(ks, vs, hk, hv, np.array([[3, 1]]), lib=lib) == 0
    assert np.array_equal(hk[1], ks[3]) and np.array_equal(hv[1], vs[3]) and not hk[0].any()


PINS = {name: fn for name, fn in globals().items() if name.startswith("pin_")}
