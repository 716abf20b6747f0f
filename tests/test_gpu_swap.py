"""pa_swap_blocks on the GPU: whole blocks between a device pool and a pool
in pinned host memory, bit-exact against the oracle over both pools (every
untouched byte included), plus the device status bits."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

SHAPE = (16, 8, 128)          # block_size, kv heads, head_dim


_CODES = {"fp8": np.uint8, "int8": np.int8}       # one-byte pools: e4m3 or int8 codes


def _pool(rng, nb, dtype):
    if dtype in _CODES:
        return rng.integers(0, 256, size=(nb,) + SHAPE, dtype=np.uint8)
    return rng.integers(0, 65536, size=(nb,) + SHAPE, dtype=np.uint16)


def _tensor(a, dtype):
    if dtype in _CODES:
        return torch.from_numpy(a.view(_CODES[dtype]))
    t = torch.from_numpy(a.view(np.int16))
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16)


def _dev(a, dtype):
    return _tensor(a, dtype).cuda()


def _host(a, dtype):
    return _tensor(a, dtype).pin_memory()


def _bits(t):
    t = t.cpu() if t.is_cuda else t
    if t.element_size() == 1:
        return t.view(torch.uint8).numpy().copy()
    return t.view(torch.int16).numpy().view(np.uint16).copy()


@pytest.mark.parametrize("dtype", ["f16", "bf16", "fp8", "int8"])
def test_swap_out_then_in(dtype):
    """Evict 24 scattered device blocks into a pinned host pool, then bring
    them back into other device blocks; both directions bit-exact."""
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(21))
    dk, dv = _pool(rng, 96, dtype), _pool(rng, 96, dtype)
    hk, hv = _pool(rng, 40, dtype), _pool(rng, 40, dtype)
    out_map = np.stack([rng.permutation(96)[:24], rng.permutation(40)[:24]], 1).astype(np.int64)
    d_k, d_v, h_k, h_v = _dev(dk, dtype), _dev(dv, dtype), _host(hk, dtype), _host(hv, dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.pa_swap_blocks(d_k, d_v, h_k, h_v, torch.from_numpy(out_map).cuda(), status)
    torch.cuda.synchronize()
    ek, ev = hk.copy(), hv.copy()
    assert oracle.swap_blocks(dk, dv, ek, ev, out_map) == 0
    assert np.array_equal(_bits(h_k), ek) and np.array_equal(_bits(h_v), ev)
    # swap in: host blocks -> fresh device blocks (mapping in pinned host memory)
    in_map = np.stack([out_map[:, 1], rng.permutation(96)[:24]], 1).astype(np.int64)
    dk2, dv2 = _pool(rng, 96, dtype), _pool(rng, 96, dtype)
    d_k2, d_v2 = _dev(dk2, dtype), _dev(dv2, dtype)
    B.pa_swap_blocks(h_k, h_v, d_k2, d_v2, torch.from_numpy(in_map).pin_memory(), status)
    torch.cuda.synchronize()
    fk, fv = dk2.copy(), dv2.copy()
    assert oracle.swap_blocks(ek, ev, fk, fv, in_map) == 0
    assert np.array_equal(_bits(d_k2), fk) and np.array_equal(_bits(d_v2), fv)
    for (src, mid), (_, dst) in zip(out_map, in_map):
        assert np.array_equal(fk[dst], dk[src])
    assert int(status.item()) == 0


def test_swap_status_bits():
    """Ids outside either pool are skipped and flagged (bit 1); a repeated
    destination is flagged (bit 8); statuses and bytes match the oracle."""
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(22))
    dk, dv = _pool(rng, 12, "f16"), _pool(rng, 12, "f16")
    hk, hv = _pool(rng, 6, "f16"), _pool(rng, 6, "f16")
    for pairs, bit in (([[0, 6]], 1), ([[12, 0]], 1), ([[-1, 2]], 1), ([[3, 1], [4, 1]], 8),
                       ([[3, 1], [3, 2]], 0)):
        m = np.array(pairs, dtype=np.int64)
        h_k, h_v = _host(hk.copy(), "f16"), _host(hv.copy(), "f16")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        B.pa_swap_blocks(_dev(dk, "f16"), _dev(dv, "f16"), h_k, h_v, torch.from_numpy(m).cuda(),
                         status)
        torch.cuda.synchronize()
        ek, ev = hk.copy(), hv.copy()
        st = oracle.swap_blocks(dk, dv, ek, ev, m)
        assert int(status.item()) == st and (st & bit) == bit, (pairs, int(status.item()), st)
        if bit != 8:
            assert np.array_equal(_bits(h_k), ek) and np.array_equal(_bits(h_v), ev)


def test_swap_within_one_pool_is_copy_blocks():
    """Source and destination the same pool: pa_copy_blocks semantics,
    including its conflict rule (a destination that another pair reads)."""
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(23))
    k, v = _pool(rng, 10, "bf16"), _pool(rng, 10, "bf16")
    for pairs in ([[1, 4], [7, 2], [3, 3]], [[1, 4], [4, 2]]):
        m = np.array(pairs, dtype=np.int64)
        d_k, d_v = _dev(k, "bf16"), _dev(v, "bf16")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        B.pa_swap_blocks(d_k, d_v, d_k, d_v, torch.from_numpy(m).cuda(), status)
        torch.cuda.synchronize()
        ek, ev = k.copy(), v.copy()
        st = oracle.copy_blocks(ek, ev, m)
        assert int(status.item()) == st
        if st == 0:
            assert np.array_equal(_bits(d_k), ek) and np.array_equal(_bits(d_v), ev)


def test_swap_rejects_unpinned_host_and_bad_args():
    from paged_kv_cache_415_b200 import binding as B
    k = torch.zeros((4,) + SHAPE, dtype=torch.float16, device="cuda")
    host = torch.zeros((4,) + SHAPE, dtype=torch.float16)           # pageable
    m = torch.zeros((1, 2), dtype=torch.int64, device="cuda")
    with pytest.raises(ValueError):
        B.pa_swap_blocks(k, k, host, host, m)
    # the library itself refuses a pageable host pool before launching anything
    code = B.LIB.pa_swap_blocks(k.data_ptr(), k.data_ptr(), host.data_ptr(), host.data_ptr(),
                                m.data_ptr(), 1, SHAPE[1], SHAPE[2], SHAPE[0], 4, 4,
                                B.PA_DTYPE_F16, None, B._stream(None))
    assert code == B.PA_ERR_INVALID_ARG
    assert not host.any()
    bad = torch.zeros((4, 16, 8, 96), dtype=torch.float16, device="cuda")   # head_dim 96
    with pytest.raises(B.PAError):
        B.pa_swap_blocks(bad, bad, bad.clone(), bad.clone(), m)


@pytest.mark.slow
def test_swap_llama7b_blocks_round_trip():
    """512 LLaMA-7B-shaped blocks (32 heads x 128, fp16: 128 KB per K block)
    out to a pinned pool and back, checked against the oracle on a sample
    of pairs and in full by the round trip."""
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(24))
    shape = (16, 32, 128)
    dev_k = torch.randint(-32768, 32767, (2048,) + shape, dtype=torch.int16, device="cuda")
    dev_v = torch.randint(-32768, 32767, (2048,) + shape, dtype=torch.int16, device="cuda")
    host_k = torch.zeros((1024,) + shape, dtype=torch.int16).pin_memory()
    host_v = torch.zeros((1024,) + shape, dtype=torch.int16).pin_memory()
    m = np.stack([rng.permutation(2048)[:512], rng.permutation(1024)[:512]], 1).astype(np.int64)
    f16 = lambda t: t.view(torch.float16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.pa_swap_blocks(f16(dev_k), f16(dev_v), f16(host_k), f16(host_v), torch.from_numpy(m).cuda(),
                     status)
    back_k, back_v = torch.zeros_like(dev_k), torch.zeros_like(dev_v)
    B.pa_swap_blocks(f16(host_k), f16(host_v), f16(back_k), f16(back_v),
                     torch.from_numpy(m[:, ::-1].copy()).cuda(), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    idx = torch.from_numpy(m[:, 0]).cuda()
    assert torch.equal(back_k[idx], dev_k[idx]) and torch.equal(back_v[idx], dev_v[idx])
    sample = m[rng.permutation(512)[:16]]
    ref_k = np.zeros((1024,) + shape, dtype=np.uint16)
    ref_v = np.zeros_like(ref_k)
    src_k = dev_k[torch.from_numpy(sample[:, 0]).cuda()].cpu().numpy().view(np.uint16)
    src_v = dev_v[torch.from_numpy(sample[:, 0]).cuda()].cpu().numpy().view(np.uint16)
    local = np.stack([np.arange(16), sample[:, 1]], 1)
    assert oracle.swap_blocks(np.ascontiguousarray(src_k), np.ascontiguousarray(src_v), ref_k,
                              ref_v, local) == 0
    got_k = host_k.numpy().view(np.uint16)
    for _, dst in sample:
        assert np.array_equal(got_k[dst], ref_k[dst])
