"""The byte model against the figures the pages print (tests/golden/page_figures.json)."""
import json
import math
import os

import numpy as np

from workloads import byte_model as bm
from workloads import generators as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def _g():
    with open(GOLDEN) as f:
        return json.load(f)


def test_block_size_figure():
    g = _g()["block_elements"]
    n = bm.block_elements(g["block_size"], g["num_heads"], g["head_dim"])
    assert n == g["elements"]
    assert n * 2 == g["fp16_kib"] * 1024


def test_kv_per_token_llama2_13b():
    g = _g()["kv_per_token_llama2_13b"]
    per_tok = bm.kv_bytes_per_token(g["num_layers"], g["num_heads"], g["head_dim"], g["elem_bytes"])
    assert per_tok == 819200                                   # exactly 0.78125 MiB
    assert round(per_tok / 2 ** 20, 2) == g["per_token_mib_approx"]
    assert round(per_tok * g["seq_tokens"] / 2 ** 30, 1) == g["per_seq_gib_approx"]


def test_a100_budget_is_about_14k_tokens():
    g = _g()
    kv = g["a100_kv_budget"]["kv_gb_approx"] * 1e9
    per_tok = bm.kv_bytes_per_token(40, 40, 128, 2)
    assert 14000 < kv / per_tok < 15000


def test_contiguous_waste_figures():
    g = _g()["llama7b_contiguous_utilisation"]
    u = bm.contiguous_utilisation(g["used_tokens"], g["reserved_tokens"])
    assert u * 100 == g["utilisation_pct"] and (1 - u) * 100 == g["waste_pct"]
    g = _g()["fifty_of_2048_waste"]
    u = bm.contiguous_utilisation(g["used_tokens"], g["reserved_tokens"])
    # 1 - 50/2048 = 97.56%: the page quotes it truncated to one decimal
    assert math.floor((1 - u) * 1000) / 10 == g["waste_pct_approx"]


def test_paged_waste_bound():
    for b in (8, 16, 32):
        w = [bm.paged_waste_slots(c, b) for c in range(1, 200)]
        assert max(w) == b - 1 and min(w) == 0


def test_decode_bytes_by_hand():
    # two sequences, 17 and 16 tokens, 2 kv heads, 4 q heads, D = 8, B = 16, 2-byte elements
    b = bm.decode_bytes(np.array([17, 16]), 4, 2, 8, 16, 2)
    assert b["kv"] == (17 + 16) * 2 * 8 * 2 * 2
    assert b["query"] == b["out"] == 2 * 4 * 8 * 2
    assert b["block_table"] == (2 + 1) * 4 and b["context_lens"] == 8
    assert b["total"] == b["kv"] + 2 * b["query"] + 12 + 8


def test_unique_bytes_of_shared_prefixes():
    wl = gen.beam_search(prompts=2, beams=4, prompt_len=40, max_new=24, num_heads=4,
                         num_blocks=64)
    ref = bm.decode_bytes(wl.context_lens, 4, 4, 128, 16, 2)["kv"]
    uniq = bm.unique_kv_bytes(wl)
    assert uniq < ref
    row = 4 * 128 * 2 * 2
    # unique tokens: prompts once (2 x 40) plus every divergent token, plus the
    # prompt-tail tokens duplicated into copy-on-write blocks
    n_new = int(wl.extra["n_new"].sum())
    copies = wl.block_mapping.shape[0]
    assert uniq == (2 * 40 + n_new + copies * (40 % 16)) * row


def test_fp8_step_bytes_by_hand():
    """e4m3 pools: one byte per cached element; the appended rows are read in
    the 16-bit type and written as codes."""
    wl = gen.make_decode("b", seed=1, dtype="f16", context_lens=[17, 16], num_q_heads=4,
                         num_kv_heads=2, head_dim=8, block_size=16, num_blocks=8, scale=0.5)
    w8 = gen.with_fp8_pools(wl, seed=2)
    a, b = bm.step_bytes(wl), bm.step_bytes(w8)
    assert b["kv"] * 2 == a["kv"] == (17 + 16) * 2 * 8 * 2 * 2
    assert b["append"] == 2 * 2 * 16 * 2 + 2 * 2 * 16 + 8 * 2
    assert a["attention"] - b["attention"] == a["kv"] - b["kv"]


def test_fp8_pools_mark_every_unheld_slot():
    """with_fp8_pools: history slots hold finite codes, every other slot
    (free blocks, block tails, this step's new slots) the NaN code."""
    wl = gen.make_decode("b", seed=3, dtype="bf16", context_lens=[1, 33, 20], num_q_heads=2,
                         num_kv_heads=2, head_dim=16, block_size=16, num_blocks=12, scale=0.25)
    w8 = gen.with_fp8_pools(wl, seed=4)
    for pool in (w8.k_cache, w8.v_cache):
        assert pool.dtype == np.uint8
        held = np.zeros(pool.shape[:2], bool)
        for s, c in enumerate(w8.context_lens):
            for pos in range(int(c) - 1):
                held[w8.block_tables[s, pos // 16], pos % 16] = True
        assert np.all((pool[held] & 0x7F) != 0x7F)
        assert np.all(pool[~held] == 0x7F)
        assert ((pool[held] >> 3) & 0xF).max() <= 14


def test_int8_pools_mark_every_unheld_slot_and_count_one_byte():
    """with_int8_pools: history slots hold codes in [-127, 127], every other
    slot -128; the byte model counts one byte per cached element."""
    wl = gen.make_decode("b", seed=5, dtype="f16", context_lens=[1, 33, 20], num_q_heads=2,
                         num_kv_heads=2, head_dim=16, block_size=16, num_blocks=12, scale=0.25)
    w8 = gen.with_int8_pools(wl, seed=6)
    assert w8.extra["kv_dtype"] == "int8" and bm.kv_elem_bytes(w8) == 1
    assert bm.step_bytes(w8)["kv"] * 2 == bm.step_bytes(wl)["kv"]
    for pool in (w8.k_cache, w8.v_cache):
        assert pool.dtype == np.int8
        held = np.zeros(pool.shape[:2], bool)
        for s, c in enumerate(w8.context_lens):
            for pos in range(int(c) - 1):
                held[w8.block_tables[s, pos // 16], pos % 16] = True
        assert pool[held].min() >= -127
        assert np.all(pool[~held] == -128)
