"""reshape_and_cache and copy_blocks on the GPU: bit-exact against the
oracle over the whole pool (every untouched element included, so a stray
write anywhere fails), plus the device status bits."""
import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins
from tests.gpu_utils import DeviceWorkload, to_bits, to_dev
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _oracle_cache_ops(wl):
    kc, vc = wl.k_cache.copy(), wl.v_cache.copy()
    st = 0
    if wl.block_mapping.shape[0]:
        st |= oracle.copy_blocks(kc, vc, wl.block_mapping)
    if wl.num_new_tokens:
        st |= oracle.reshape_and_cache(wl.new_key, wl.new_value, kc, vc, wl.slot_mapping,
                                       wl.block_size)
    return kc, vc, st


def _check_cache_ops(wl):
    from paged_kv_cache_415_b200 import binding as B
    dw = DeviceWorkload(wl)
    if wl.block_mapping.shape[0]:
        B.pa_copy_blocks(dw.k_cache, dw.v_cache, dw.block_mapping, dw.d_status)
    if wl.num_new_tokens:
        B.pa_reshape_and_cache(dw.new_key, dw.new_value, dw.k_cache, dw.v_cache,
                               dw.slot_mapping, dw.d_status)
    torch.cuda.synchronize()
    ek, ev, est = _oracle_cache_ops(wl)
    assert np.array_equal(to_bits(dw.k_cache), ek)
    assert np.array_equal(to_bits(dw.v_cache), ev)
    assert dw.status() == est == 0


@pytest.mark.parametrize("make", [gen.tiny, oracle_pins.small_beams,
                                  lambda: oracle_pins.small_gqa(block_size=8, dtype="f16"),
                                  lambda: oracle_pins.small_gqa(block_size=32, head_dim=64)],
                         ids=["tiny", "beams-small", "bs8-f16", "bs32-d64"])
def test_cache_ops_small(make):
    _check_cache_ops(make())


@pytest.mark.slow
def test_cache_ops_llama7b_full():
    """64 new tokens into the 16384-block fp16 pool."""
    _check_cache_ops(gen.llama7b())


@pytest.mark.slow
def test_cache_ops_beam_search_full():
    """Copy-on-write of the shared partial prompt blocks, then every beam's
    divergent tokens, into the 8192-block pool of 40 heads."""
    wl = gen.beam_search()
    assert 0 < wl.block_mapping.shape[0] <= 96
    _check_cache_ops(wl)


def _pool(rng, nb=12, b=16, h=2, d=64):
    return rng.integers(0, 65535, size=(nb, b, h, d), dtype=np.uint16)


def test_padding_and_bad_slots():
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(1))
    kc, vc = _pool(rng), _pool(rng)
    key = rng.integers(0, 65535, size=(4, 2, 64), dtype=np.uint16)
    val = rng.integers(0, 65535, size=(4, 2, 64), dtype=np.uint16)
    slots = np.array([-1, 5, 12 * 16, 17], dtype=np.int64)      # pad, ok, out of pool, ok
    dk, dv = to_dev(kc, "f16"), to_dev(vc, "f16")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.pa_reshape_and_cache(to_dev(key, "f16"), to_dev(val, "f16"), dk, dv,
                           torch.from_numpy(slots).cuda(), status)
    ek, ev = kc.copy(), vc.copy()
    st = oracle.reshape_and_cache(key, val, ek, ev, slots, 16)
    assert np.array_equal(to_bits(dk), ek) and np.array_equal(to_bits(dv), ev)
    assert int(status.item()) == st == 2


def test_copy_conflicts_and_bad_ids():
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(2))
    kc, vc = _pool(rng), _pool(rng)
    for mapping, bit in (([[1, 4], [2, 4]], 8), ([[1, 4], [4, 2]], 8), ([[1, 40]], 1),
                         ([[-1, 3]], 1), ([[3, 3], [0, 5]], 0)):
        m = np.array(mapping, dtype=np.int64)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        dk, dv = to_dev(kc, "f16"), to_dev(vc, "f16")
        B.pa_copy_blocks(dk, dv, torch.from_numpy(m).cuda(), status)
        got = int(status.item())
        ref = oracle.copy_blocks(kc.copy(), vc.copy(), m)
        assert got == ref, (mapping, got, ref)
        assert (got & bit) == bit
        if bit == 0:
            ek, ev = kc.copy(), vc.copy()
            oracle.copy_blocks(ek, ev, m)
            assert np.array_equal(to_bits(dk), ek) and np.array_equal(to_bits(dv), ev)
