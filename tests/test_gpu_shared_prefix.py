"""pa_paged_decode_shared_prefix against the fp64 oracle: groups of
sequences that share their first blocks (beams of a prompt) read those
blocks once; the result must be the plain paged decode's."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins
from tests.gpu_utils import DeviceWorkload, assert_close, oracle_step, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _shared(dw, prefix_lens, group_size, partition_size=0, max_prefix_len=None, tables=None):
    from paged_kv_cache_415_b200 import binding as B
    wl = dw.wl
    mpl = int(prefix_lens.max()) if max_prefix_len is None else max_prefix_len
    ws_bytes = B.pa_paged_decode_shared_prefix_workspace_size(
        wl.num_seqs, group_size, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        wl.max_context_len, mpl, partition_size)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    out = torch.full_like(dw.query, float("nan"))
    B.pa_paged_decode_shared_prefix(
        out, dw.query, dw.k_cache, dw.v_cache, dw.block_tables if tables is None else tables,
        dw.context_lens, torch.from_numpy(np.ascontiguousarray(prefix_lens, np.int32)).cuda(),
        group_size, wl.max_context_len, mpl, wl.scale, ws, partition_size, dw.d_status)
    torch.cuda.synchronize()
    return out


def _run_step_then_shared(wl, **kw):
    dw = DeviceWorkload(wl)
    dw.step(cache_ops=True)                # copies + appends (the decode output is unused)
    dw.d_status.zero_()
    out = _shared(dw, wl.extra["prefix_lens"], wl.extra["group_size"], **kw)
    _, _, ref, st = oracle_step(wl)
    return dw, out, ref, st


@pytest.mark.parametrize("partition", [0, 16, 32, 64])
def test_beams_small(partition):
    wl = gen.beam_search(prompts=3, beams=4, prompt_len=40, max_new=24, num_heads=4,
                         num_blocks=96)
    dw, out, ref, st = _run_step_then_shared(wl, partition_size=partition)
    assert st == 0 and dw.status() == 0
    assert_close(to_f64(out), ref, f"shared prefix, partition {partition}")


def test_beams_prompt_longer_than_partition():
    wl = gen.beam_search(prompts=2, beams=4, prompt_len=300, max_new=60, num_heads=8,
                         num_blocks=256)
    dw, out, ref, st = _run_step_then_shared(wl, partition_size=64)
    assert dw.status() == 0
    assert_close(to_f64(out), ref, "shared prefix over several partitions")


@pytest.mark.parametrize("dtype,group,beams", [("bf16", 2, 4), ("f16", 4, 2), ("bf16", 8, 1)])
def test_gqa_groups(dtype, group, beams):
    """GQA heads and group members share the 8 rows of the tile."""
    rng = np.random.Generator(np.random.PCG64(group * 10 + beams))
    prompts, b = 3, 16
    ctx = []
    for _ in range(prompts):
        base = int(rng.integers(20, 120))
        ctx += [base + int(rng.integers(0, 40)) for _ in range(beams)]
    wl = gen.make_decode("gqa-groups", seed=5, dtype=dtype, context_lens=ctx,
                         num_q_heads=2 * group, num_kv_heads=2, head_dim=128, block_size=b,
                         num_blocks=256, scale=1 / math.sqrt(128))
    # make every group's members share the first block(s) of member 0
    tables = wl.block_tables.copy()
    prefix = []
    kc, vc = oracle_pins.pool_after_step(wl)
    wl.k_cache, wl.v_cache = kc, vc
    wl.slot_mapping = wl.slot_mapping[:0]
    wl.new_key, wl.new_value = wl.new_key[:0], wl.new_value[:0]
    for p in range(prompts):
        members = range(p * beams, (p + 1) * beams)
        shared_blocks = min(int(wl.context_lens[m]) for m in members) // b
        shared_blocks = max(0, shared_blocks - 1)
        for m in members:
            tables[m, :shared_blocks] = tables[p * beams, :shared_blocks]
        prefix.append(shared_blocks * b)
    wl.block_tables = tables
    dw = DeviceWorkload(wl)
    out = _shared(dw, np.array(prefix), beams, partition_size=32)
    ref, st = oracle.paged_decode(wl.query, kc, vc, tables, wl.context_lens, wl.scale, wl.dtype)
    assert dw.status() == 0
    assert_close(to_f64(out), ref, f"G{group} x {beams} members")


def test_no_prefix_equals_plain_decode():
    wl = oracle_pins.small_llama(seqs=4)
    kc, vc = oracle_pins.pool_after_step(wl)
    wl.k_cache, wl.v_cache = kc, vc
    dw = DeviceWorkload(wl)
    out = _shared(dw, np.zeros(2, np.int32), 2, partition_size=64)
    ref, _ = oracle.paged_decode(wl.query, kc, vc, wl.block_tables, wl.context_lens, wl.scale,
                                 wl.dtype)
    assert dw.status() == 0
    assert_close(to_f64(out), ref, "prefix 0")


def test_bad_prefix_is_flagged():
    wl = gen.beam_search(prompts=2, beams=4, prompt_len=40, max_new=24, num_heads=4,
                         num_blocks=96)
    dw = DeviceWorkload(wl)
    dw.step(cache_ops=True)
    dw.d_status.zero_()
    bad = wl.extra["prefix_lens"].copy()
    bad[1] = 24                                            # not a whole number of blocks
    out = _shared(dw, bad, 4, max_prefix_len=32)
    assert dw.status() & 4
    got = to_f64(out)
    assert not got[4:8].any()                              # group 1: zero rows
    _, _, ref, _ = oracle_step(wl)
    assert_close(got[:4], ref[:4], "group 0 unaffected")
    # members that do not share the blocks they claim to
    dw.d_status.zero_()
    tables = wl.block_tables.copy()
    tables[1, 0] = tables[2, 1]
    _shared(dw, wl.extra["prefix_lens"], 4, tables=torch.from_numpy(tables).cuda())
    assert dw.status() & 1


@pytest.mark.slow
def test_beam_search_full():
    """The full beam workload: every output row of the shared-prefix decode
    against the full fp64 oracle."""
    wl = gen.beam_search()
    dw = DeviceWorkload(wl)
    dw.step(cache_ops=True)
    dw.d_status.zero_()
    out = _shared(dw, wl.extra["prefix_lens"], wl.extra["group_size"])
    assert dw.status() == 0
    _, _, ref, st = oracle_step(wl)
    assert st == 0
    assert_close(to_f64(out), ref, "beam_search full, shared prefix, every row")
