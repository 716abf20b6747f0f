"""pa_paged_decode_append: the step's cache write fused into the decode
launch.  The pools must equal the oracle's cache write bit for bit, and the
output the oracle's attention (new tokens included)."""

import numpy as np
import pytest
import torch

from tests import oracle_pins
from tests.gpu_utils import DeviceWorkload, assert_close, oracle_step, to_bits, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _append(dw, partition_size=0, tables=None):
    from paged_kv_cache_415_b200 import binding as B
    wl = dw.wl
    ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                wl.head_dim, wl.block_size, wl.max_context_len,
                                                partition_size)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    out = torch.full_like(dw.query, float("nan"))
    B.pa_paged_decode_append(out, dw.query, dw.new_key, dw.new_value, dw.k_cache, dw.v_cache,
                             dw.block_tables if tables is None else tables, dw.context_lens,
                             wl.max_context_len, wl.scale, partition_size, ws, dw.d_status)
    torch.cuda.synchronize()
    return out


def _check(wl, partition_size=0):
    assert wl.num_new_tokens == wl.num_seqs          # one token per sequence, at ctx - 1
    dw = DeviceWorkload(wl)
    out = _append(dw, partition_size)
    kc, vc, ref, st = oracle_step(wl)
    assert np.array_equal(to_bits(dw.k_cache), kc) and np.array_equal(to_bits(dw.v_cache), vc)
    assert dw.status() == 0 and st == 0
    assert_close(to_f64(out), ref, f"{wl.name} append, partition {partition_size}")


@pytest.mark.parametrize("partition", [0, 32, 128])
def test_append_mha(partition):
    _check(oracle_pins.small_llama(seqs=6), partition)


@pytest.mark.parametrize("partition", [0, 16, 48, 256])
def test_append_gqa_tensor_core_path(partition):
    """16-token partitions split every context into many; the appended row
    is written by a warp of the last one."""
    _check(oracle_pins.small_gqa(), partition)


@pytest.mark.parametrize("block_size,dtype,head_dim", [(8, "f16", 64), (32, "bf16", 128)])
def test_append_other_shapes(block_size, dtype, head_dim):
    _check(oracle_pins.small_gqa(block_size=block_size, dtype=dtype, head_dim=head_dim), 64)


def test_append_long_context_small():
    _check(gen.long_context(seqs=2, ctx=3000, num_blocks=400), 512)


def test_append_bad_slot_is_flagged():
    wl = oracle_pins.small_llama(seqs=3)
    dw = DeviceWorkload(wl)
    tables = wl.block_tables.copy()
    s = 1
    tables[s, (int(wl.context_lens[s]) - 1) // wl.block_size] = wl.num_blocks + 3
    _append(dw, 64, torch.from_numpy(tables).cuda())
    assert dw.status() & 2
    # nothing was written for that sequence's token
    kc = to_bits(dw.k_cache)
    slot = int(wl.slot_mapping[s])
    assert np.all(kc[slot // wl.block_size, slot % wl.block_size] == gen.NAN_BITS[wl.dtype])


@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama7b", "mistral7b", "long_context"])
def test_append_full_size(name):
    """The entry point the benchmark times, on the full workload in its
    launch configuration: both whole pools bit for bit against the oracle's
    cache write, and every output row against the full fp64 oracle."""
    wl = gen.CONFIGS[name]()
    dw = DeviceWorkload(wl)
    out = _append(dw, wl.partition_size)
    assert dw.status() == 0
    kc, vc, ref, st = oracle_step(wl)
    assert st == 0
    assert np.array_equal(to_bits(dw.k_cache), kc), f"{name}: K pool differs"
    assert np.array_equal(to_bits(dw.v_cache), vc), f"{name}: V pool differs"
    assert_close(to_f64(out), ref, f"{name} fused append, every row")
