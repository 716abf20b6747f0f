"""Paged decode attention on the GPU against the fp64 oracle.

Tolerance: |gpu - oracle| <= 2e-3 + 1e-2 |oracle| elementwise (fp16/bf16
inputs, fp32 accumulation, output rounded to the input type).  Beyond the
tolerance the GPU result must be deterministic and independent of where the
blocks sit in the pool (bit-identical checks)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins
from tests.gpu_utils import DeviceWorkload, assert_close, oracle_step, to_bits, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _parity(wl, partition_size=None, what=""):
    dw = DeviceWorkload(wl)
    out = dw.step(partition_size=partition_size)
    torch.cuda.synchronize()
    _, _, ref, st = oracle_step(wl)
    assert_close(to_f64(out), ref, what or wl.name)
    assert dw.status() == st == 0
    return dw, out


def test_tiny_step_and_remapped_tables():
    """The tiny workload end to end (2 block copies, 4 new tokens, decode);
    then decode again through tables remapped onto the copies: identical."""
    wl = gen.tiny()
    dw, out = _parity(wl)
    remapped = torch.from_numpy(wl.extra["remapped_block_tables"]).cuda()
    out2 = dw.decode(block_tables=remapped)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("block_size", [8, 16, 32])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_every_kernel_instance(head_dim, block_size, group, dtype):
    """Each (head_dim, block_size, group, dtype) instance on ragged contexts
    that span several blocks, warps and partitions (partition of 4 blocks)."""
    rng = np.random.Generator(np.random.PCG64(head_dim * 1000 + block_size * 10 + group))
    ctx = rng.integers(1, 300, size=3, endpoint=True)
    ctx[0] = 1
    nb = int(sum(-(-int(c) // block_size) for c in ctx)) + 8
    wl = gen.make_decode("instance", seed=77, dtype=dtype, context_lens=ctx,
                         num_q_heads=2 * group, num_kv_heads=2, head_dim=head_dim,
                         block_size=block_size, num_blocks=nb, scale=1 / math.sqrt(head_dim),
                         partition_size=4 * block_size)
    _parity(wl, what=f"D{head_dim} B{block_size} G{group} {dtype}")


@pytest.mark.parametrize("make", [oracle_pins.small_beams, lambda: oracle_pins.small_llama(seqs=6),
                                  oracle_pins.small_gqa],
                         ids=["beams", "llama-small", "gqa-small"])
def test_small_workloads(make):
    _parity(make())


def _mistral_small():
    return gen.mistral7b(seqs=24, num_blocks=4096)


def _long_small():
    return gen.long_context(seqs=2, ctx=4000, num_blocks=600)


@pytest.mark.parametrize("partition", [16, 512, 0, 8192])
@pytest.mark.parametrize("make", [_mistral_small, _long_small], ids=["mistral-24", "long-2x4000"])
def test_partition_sweep(make, partition):
    """One block per partition, 512-token partitions, the library's choice and
    a single partition all match the oracle."""
    _parity(make(), partition_size=partition, what=f"partition {partition}")


def test_deterministic_and_placement_independent():
    """Two runs are bit-identical; moving every block to pi(b) and mapping the
    tables through pi is bit-identical too."""
    wl = oracle_pins.small_gqa()
    kc, vc = oracle_pins.pool_after_step(wl)
    wl.k_cache, wl.v_cache = kc, vc
    wl.slot_mapping = wl.slot_mapping[:0]
    wl.new_key, wl.new_value = wl.new_key[:0], wl.new_value[:0]
    dw = DeviceWorkload(wl)
    a = dw.decode(partition_size=64)
    b = dw.decode(partition_size=64)
    pi = np.random.Generator(np.random.PCG64(3)).permutation(wl.num_blocks)
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[pi], vc2[pi] = kc, vc
    t2 = np.where(wl.block_tables >= 0, pi[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    wl2 = oracle_pins.small_gqa()
    wl2.k_cache, wl2.v_cache, wl2.block_tables = kc2, vc2, t2
    dw2 = DeviceWorkload(wl2)
    c = dw2.decode(partition_size=64)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_single_token_context_returns_v0_exactly():
    wl = oracle_pins.small_llama()
    kc, vc = oracle_pins.pool_after_step(wl)
    wl.k_cache, wl.v_cache = kc, vc
    dw = DeviceWorkload(wl)
    ones = torch.ones(wl.num_seqs, dtype=torch.int32, device="cuda")
    out = dw.decode(context_lens=ones, max_context_len=1)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for s in range(wl.num_seqs):
        v0 = vc[wl.block_tables[s, 0], 0]                         # [Hkv][D]
        assert np.array_equal(got[s], v0)


def test_empty_and_invalid_contexts():
    """ctx 0 -> zero row, no status; negative / too long -> zero row and
    PA_STATUS_BAD_CONTEXT; the other rows are unaffected."""
    wl = oracle_pins.small_llama(seqs=4)
    kc, vc = oracle_pins.pool_after_step(wl)
    wl.k_cache, wl.v_cache = kc, vc
    dw = DeviceWorkload(wl)
    ctx = wl.context_lens.copy()
    ctx[0] = 0
    out = dw.decode(context_lens=torch.from_numpy(ctx).cuda(), partition_size=64)
    ref, st = oracle.paged_decode(wl.query, kc, vc, wl.block_tables, ctx, wl.scale, wl.dtype)
    assert_close(to_f64(out), ref)
    assert dw.status() == 0 and st == 0
    for bad in (-3, wl.max_blocks_per_seq * wl.block_size + 1):
        ctx[0] = bad
        dw.d_status.zero_()
        mcl = int(max(ctx.max(), wl.context_lens.max()))
        out = dw.decode(context_lens=torch.from_numpy(ctx).cuda(), partition_size=64,
                        max_context_len=mcl)
        ref, st = oracle.paged_decode(wl.query, kc, vc, wl.block_tables, ctx, wl.scale, wl.dtype)
        assert_close(to_f64(out), ref)
        assert dw.status() == st == 4
    # a context longer than the max_context_len the caller promised
    ctx = wl.context_lens.copy()
    dw.d_status.zero_()
    out = dw.decode(max_context_len=int(ctx.max()) - 1, partition_size=64)
    assert dw.status() & 4
    s_long = int(np.argmax(ctx))
    assert not to_f64(out)[s_long].any()


@pytest.mark.parametrize("partition", [16, 0], ids=["many-partitions", "auto"])
def test_gqa_empty_invalid_contexts_and_bad_block(partition):
    """The tensor-core path, with contexts split into many 16-token
    partitions and with the library's partition:
    ctx 0 -> zero row; negative ctx -> zero row + bit 4; an out-of-pool block
    id -> skipped + bit 1; every other row as the oracle."""
    wl = oracle_pins.small_gqa(seqs=6)
    kc, vc = oracle_pins.pool_after_step(wl)
    wl.k_cache, wl.v_cache = kc, vc
    dw = DeviceWorkload(wl)
    ctx = wl.context_lens.copy()
    ctx[0], ctx[2] = 0, -3
    tables = wl.block_tables.copy()
    s_long = int(np.argmax(ctx))
    tables[s_long, 1] = wl.num_blocks + 5
    out = dw.decode(context_lens=torch.from_numpy(ctx).cuda(),
                    block_tables=torch.from_numpy(tables).cuda(), partition_size=partition)
    ref, st = oracle.paged_decode(wl.query, kc, vc, tables, ctx, wl.scale, wl.dtype)
    assert st == 5 and dw.status() == 5
    assert_close(to_f64(out), ref)


def test_bad_block_id_is_skipped_and_flagged():
    wl = oracle_pins.small_llama(seqs=4)
    kc, vc = oracle_pins.pool_after_step(wl)
    wl.k_cache, wl.v_cache = kc, vc
    dw = DeviceWorkload(wl)
    s = int(np.argmax(wl.context_lens))
    tables = wl.block_tables.copy()
    tables[s, 0] = wl.num_blocks + 7
    out = dw.decode(block_tables=torch.from_numpy(tables).cuda(), partition_size=64)
    ref, st = oracle.paged_decode(wl.query, kc, vc, tables, wl.context_lens, wl.scale, wl.dtype)
    assert st == 1 and dw.status() == 1
    assert_close(to_f64(out), ref)


def test_large_scores_stay_finite():
    wl = oracle_pins.small_llama(seqs=3)
    q = (wl.query.view(np.float16).astype(np.float32) * 1000).astype(np.float16).view(np.uint16)
    wl.query = q
    _parity(wl, partition_size=64, what="q x 1000")


# ---------------------------------------------------------------------------
# Full-size workloads, in the launch configuration the benchmark times:
# the pools after the step's cache operations bit for bit, and every output
# row against the full fp64 oracle.
# ---------------------------------------------------------------------------

@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama7b", "mistral7b", "beam_search", "long_context"])
def test_full_size(name):
    wl = gen.CONFIGS[name]()
    dw = DeviceWorkload(wl)
    out = dw.step()
    torch.cuda.synchronize()
    assert dw.status() == 0
    kc, vc, ref, st = oracle_step(wl)
    assert st == 0
    assert np.array_equal(to_bits(dw.k_cache), kc), f"{name}: K pool differs"
    assert np.array_equal(to_bits(dw.v_cache), vc), f"{name}: V pool differs"
    assert_close(to_f64(out), ref, f"{name}, every row")
