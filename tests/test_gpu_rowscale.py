"""Row-scaled one-byte K/V pools (one fp32 scale per (token, kv head) row)
on the GPU against the oracle, for e4m3 and int8 codes.

  * the quantising write: codes and scales bit for bit over the whole pools
    (untouched bytes included), on rows whose kv heads differ in magnitude by
    10^4, with an all-zero row, padding tokens and a slot past the pool;
  * the decode: within the tolerance of the 16-bit path with its absolute
    part scaled by each output row's magnitude (assert_close_rows:
    |gpu - oracle| <= 2e-3 max_d |oracle row| + 1e-2 |oracle|), on pools
    whose row scales span four orders of magnitude across kv heads, with
    NaN scales and codes in every slot the kernel must not read;
  * the decode with the fused write: pools bit for bit and every output row;
  * full-size Mistral-7B and long-context workloads in the benchmark's launch
    configuration: pools bit for bit and every output row;
  * block copies of scale pools (pa_copy_blocks with PA_DTYPE_F32).
"""
import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins
from tests.gpu_utils import assert_close_rows, to_dev, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu

CODES = ["fp8", "int8"]
_NP = {"fp8": np.uint8, "int8": np.int8}


def _pool(a, fmt):
    return torch.from_numpy(np.ascontiguousarray(a).view(_NP[fmt])).cuda()


class RowDevice:
    """A with_rowscale_pools workload on the device."""

    def __init__(self, wl):
        self.wl, self.fmt = wl, wl.extra["kv_dtype"]
        self.query = to_dev(wl.query, wl.dtype)
        self.k_cache, self.v_cache = _pool(wl.k_cache, self.fmt), _pool(wl.v_cache, self.fmt)
        self.k_scales = torch.from_numpy(wl.extra["k_scales"]).cuda()
        self.v_scales = torch.from_numpy(wl.extra["v_scales"]).cuda()
        self.block_tables = torch.from_numpy(wl.block_tables).cuda()
        self.context_lens = torch.from_numpy(wl.context_lens).cuda()
        self.new_key, self.new_value = to_dev(wl.new_key, wl.dtype), to_dev(wl.new_value, wl.dtype)
        self.slot_mapping = torch.from_numpy(wl.slot_mapping).cuda()
        self.d_status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def workspace(self, partition_size):
        from paged_kv_cache_415_b200 import binding as B
        wl = self.wl
        n = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                             wl.head_dim, wl.block_size, wl.max_context_len,
                                             partition_size)
        return torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")

    def write(self):
        from paged_kv_cache_415_b200 import binding as B
        getattr(B, f"pa_reshape_and_cache_{self.fmt}_rowscale")(
            self.new_key, self.new_value, self.k_cache, self.v_cache, self.k_scales,
            self.v_scales, self.slot_mapping, self.d_status)

    def decode(self, partition_size=0):
        from paged_kv_cache_415_b200 import binding as B
        wl = self.wl
        out = torch.full_like(self.query, float("nan"))
        getattr(B, f"pa_paged_decode_{self.fmt}_rowscale")(
            out, self.query, self.k_cache, self.v_cache, self.k_scales, self.v_scales,
            self.block_tables, self.context_lens, wl.max_context_len, wl.scale, partition_size,
            self.workspace(partition_size), self.d_status)
        torch.cuda.synchronize()
        return out

    def decode_append(self, partition_size=0):
        from paged_kv_cache_415_b200 import binding as B
        wl = self.wl
        out = torch.full_like(self.query, float("nan"))
        getattr(B, f"pa_paged_decode_{self.fmt}_rowscale_append")(
            out, self.query, self.new_key, self.new_value, self.k_cache, self.v_cache,
            self.k_scales, self.v_scales, self.block_tables, self.context_lens,
            wl.max_context_len, wl.scale, partition_size, self.workspace(partition_size),
            self.d_status)
        torch.cuda.synchronize()
        return out

    def status(self):
        return int(self.d_status.item())


def _oracle_after_write(wl):
    """Pools and scales after the oracle's row-scaled write of the step's tokens."""
    fmt = wl.extra["kv_dtype"]
    kc, vc = wl.k_cache.copy(), wl.v_cache.copy()
    ks, vs = wl.extra["k_scales"].copy(), wl.extra["v_scales"].copy()
    st = getattr(oracle, f"reshape_and_cache_{fmt}_rowscale")(
        wl.new_key, wl.new_value, kc, vc, ks, vs, wl.slot_mapping, wl.block_size, wl.dtype)
    return kc, vc, ks, vs, st


def _oracle_decode(wl, kc, vc, ks, vs):
    fmt = wl.extra["kv_dtype"]
    return getattr(oracle, f"paged_decode_{fmt}_rowscale")(
        wl.query, kc, vc, ks, vs, wl.block_tables, wl.context_lens, wl.scale, wl.dtype)


def _same_pools(dev, kc, vc, ks, vs, what):
    assert np.array_equal(dev.k_cache.cpu().numpy().view(np.uint8), kc.view(np.uint8)), what
    assert np.array_equal(dev.v_cache.cpu().numpy().view(np.uint8), vc.view(np.uint8)), what
    # scales compared bit for bit (NaN poison included)
    assert np.array_equal(dev.k_scales.cpu().numpy().view(np.uint32), ks.view(np.uint32)), what
    assert np.array_equal(dev.v_scales.cpu().numpy().view(np.uint32), vs.view(np.uint32)), what


@pytest.mark.parametrize("fmt", CODES)
@pytest.mark.parametrize("dtype,head_dim,block_size", [("f16", 128, 16), ("bf16", 64, 8),
                                                       ("bf16", 128, 32)])
def test_rowscale_write_bit_exact(fmt, dtype, head_dim, block_size):
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(41))
    nb, h, t = 24, 4, 40
    np_t = _NP[fmt]
    kc0 = rng.integers(0, 256, size=(nb, block_size, h, head_dim), dtype=np.uint8).view(np_t)
    vc0 = rng.integers(0, 256, size=(nb, block_size, h, head_dim), dtype=np.uint8).view(np_t)
    ks0 = rng.standard_normal((nb, h, block_size)).astype(np.float32)
    vs0 = rng.standard_normal((nb, h, block_size)).astype(np.float32)
    key = oracle_pins._rows_of_mixed_magnitude(rng, t, h, head_dim, dtype)
    val = oracle_pins._rows_of_mixed_magnitude(rng, t, h, head_dim, dtype)
    slots = rng.permutation(nb * block_size)[:t].astype(np.int64)
    slots[3], slots[7] = -1, nb * block_size + 5              # padding, past the pool
    kc, vc, ks, vs = kc0.copy(), vc0.copy(), ks0.copy(), vs0.copy()
    st = getattr(oracle, f"reshape_and_cache_{fmt}_rowscale")(key, val, kc, vc, ks, vs, slots,
                                                               block_size, dtype)
    assert st == 2
    dk, dv = _pool(kc0, fmt), _pool(vc0, fmt)
    dks, dvs = torch.from_numpy(ks0).cuda(), torch.from_numpy(vs0).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    getattr(B, f"pa_reshape_and_cache_{fmt}_rowscale")(
        to_dev(key, dtype), to_dev(val, dtype), dk, dv, dks, dvs, torch.from_numpy(slots).cuda(),
        status)
    torch.cuda.synchronize()
    assert int(status.item()) == 2
    assert np.array_equal(dk.cpu().numpy().view(np.uint8), kc.view(np.uint8))
    assert np.array_equal(dv.cpu().numpy().view(np.uint8), vc.view(np.uint8))
    assert np.array_equal(dks.cpu().numpy().view(np.uint32), ks.view(np.uint32))
    assert np.array_equal(dvs.cpu().numpy().view(np.uint32), vs.view(np.uint32))


def _gqa(group, head_dim, block_size, dtype="bf16", seqs=5, hkv=4):
    return gen.make_decode("rows", seed=4150 + 70 + group, dtype=dtype,
                           context_lens=np.array([1, 17, 200, 33, 511][:seqs], np.int32),
                           num_q_heads=hkv * group, num_kv_heads=hkv, head_dim=head_dim,
                           block_size=block_size, num_blocks=160, scale=head_dim ** -0.5)


@pytest.mark.parametrize("fmt", CODES)
@pytest.mark.parametrize("group,head_dim,block_size,dtype", [
    (1, 128, 16, "f16"), (2, 64, 16, "bf16"), (4, 128, 16, "bf16"), (8, 128, 32, "f16"),
    (4, 64, 32, "f16")])
@pytest.mark.parametrize("partition", [0, 32, 2048])
def test_rowscale_decode(fmt, group, head_dim, block_size, dtype, partition):
    wl = gen.with_rowscale_pools(_gqa(group, head_dim, block_size, dtype), fmt, seed=7)
    dev = RowDevice(wl)
    dev.write()
    out = dev.decode(partition)
    kc, vc, ks, vs, st = _oracle_after_write(wl)
    ref, st2 = _oracle_decode(wl, kc, vc, ks, vs)
    assert dev.status() == 0 and st == 0 and st2 == 0
    _same_pools(dev, kc, vc, ks, vs, "pools after the write")
    assert_close_rows(to_f64(out), ref, f"{fmt} rows G={group} D={head_dim} B={block_size} P={partition}")


@pytest.mark.parametrize("fmt", CODES)
@pytest.mark.parametrize("group,hkv,partition", [(4, 2, 2048), (1, 4, 2048), (4, 3, 4096), (4, 2, 8192)])
def test_rowscale_long_partitions(fmt, group, hkv, partition):
    """One warp accumulating many blocks: partitions of 2048-8192 tokens (up
    to 128 blocks per warp), contexts of up to 8000.  int8 codes widen to 1152 + c, so
    the output accumulator carries the bias of every token it has summed;
    the kernel must keep that from costing precision over a long partition.
    Every output row against the fp64 oracle at the row-scaled tolerance."""
    ctx = np.array([2000, 1999, 8000, 33], np.int32)
    nb = int(sum(-(-int(c) // 16) for c in ctx)) + 8
    wl = gen.make_decode("rows-long", seed=4150 + 80 + group, dtype="bf16", context_lens=ctx,
                         num_q_heads=hkv * group, num_kv_heads=hkv, head_dim=128, block_size=16,
                         num_blocks=nb, scale=128 ** -0.5)
    wl = gen.with_rowscale_pools(wl, fmt, seed=11)
    dev = RowDevice(wl)
    dev.write()
    out = dev.decode(partition)
    kc, vc, ks, vs, st = _oracle_after_write(wl)
    ref, st2 = _oracle_decode(wl, kc, vc, ks, vs)
    assert dev.status() == 0 and st == 0 and st2 == 0
    assert_close_rows(to_f64(out), ref, f"{fmt} rows long partition G={group} Hkv={hkv} P={partition}")


@pytest.mark.parametrize("fmt", CODES)
@pytest.mark.parametrize("group,hkv", [(4, 3), (1, 5)])
@pytest.mark.parametrize("partition", [0, 32])
def test_rowscale_odd_kv_heads(fmt, group, hkv, partition):
    """An odd number of kv heads takes the kernel with a CTA per kv head
    (an even number a CTA per pair of kv heads)."""
    wl = gen.with_rowscale_pools(_gqa(group, 128, 16, "bf16", hkv=hkv), fmt, seed=10)
    dev = RowDevice(wl)
    dev.write()
    out = dev.decode(partition)
    kc, vc, ks, vs, st = _oracle_after_write(wl)
    ref, st2 = _oracle_decode(wl, kc, vc, ks, vs)
    assert dev.status() == 0 and st == 0 and st2 == 0
    assert_close_rows(to_f64(out), ref, f"{fmt} rows Hkv={hkv} G={group} P={partition}")


@pytest.mark.parametrize("fmt", CODES)
@pytest.mark.parametrize("partition", [0, 16, 64])
def test_rowscale_fused_append(fmt, partition):
    wl = gen.with_rowscale_pools(oracle_pins.small_gqa(keep_logical=False), fmt, seed=8)
    dev = RowDevice(wl)
    out = dev.decode_append(partition)
    kc, vc, ks, vs, st = _oracle_after_write(wl)
    ref, _ = _oracle_decode(wl, kc, vc, ks, vs)
    assert dev.status() == 0 and st == 0
    _same_pools(dev, kc, vc, ks, vs, "pools after the fused write")
    assert_close_rows(to_f64(out), ref, f"{fmt} rows fused append P={partition}")


@pytest.mark.parametrize("fmt", CODES)
def test_rowscale_heads_of_very_different_magnitude(fmt):
    """The case row scales exist for: one pool-wide scale would leave the
    small heads a handful of code steps.  Here every head keeps its
    resolution: the decode of the written rows stays within tolerance of the
    fp64 attention over the unquantised 16-bit K/V scaled per head."""
    base = _gqa(4, 128, 16, "f16")
    mags = np.array([1e-2, 1.0, 1e2, 3e-1], np.float32)
    for name in ("new_key", "new_value"):
        x = getattr(base, name).view(np.float16).astype(np.float32)
        setattr(base, name, gen.f32_to_bits(x * mags[None, :, None], "f16"))
    wl = gen.with_rowscale_pools(base, fmt, seed=9)
    dev = RowDevice(wl)
    dev.write()
    out = dev.decode(0)
    kc, vc, ks, vs, _ = _oracle_after_write(wl)
    ref, _ = _oracle_decode(wl, kc, vc, ks, vs)
    assert_close_rows(to_f64(out), ref, f"{fmt} rows, heads 10^4 apart")
    # the written rows of the smallest head use the whole code range
    b = wl.block_size
    for sl in wl.slot_mapping[:3]:
        codes = dev.k_cache[sl // b, sl % b, 0].cpu().numpy()
        dec = oracle.decode_e4m3(codes.view(np.uint8)) if fmt == "fp8" else codes.astype(float)
        assert np.max(np.abs(dec)) == (448.0 if fmt == "fp8" else 127.0)


def test_scale_pools_copy_as_blocks():
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(44))
    ks = rng.standard_normal((12, 8, 16)).astype(np.float32)
    vs = rng.standard_normal((12, 8, 16)).astype(np.float32)
    pairs = np.array([[1, 7], [3, 9], [5, 5]], np.int64)
    dks, dvs = torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.pa_copy_block_scales(dks, dvs, torch.from_numpy(pairs).cuda(), status)
    torch.cuda.synchronize()
    assert oracle.copy_blocks(ks, vs, pairs) == 0
    assert int(status.item()) == 0
    assert np.array_equal(dks.cpu().numpy(), ks) and np.array_equal(dvs.cpu().numpy(), vs)


@pytest.mark.slow
@pytest.mark.parametrize("fmt", CODES)
@pytest.mark.parametrize("name", ["mistral7b", "long_context"])
def test_rowscale_full_size(fmt, name):
    """The full workloads with row-scaled pools, in the benchmark's launch
    configuration (fused write, the workload's partitions): codes and scales
    bit for bit, every output row against the fp64 oracle."""
    wl = gen.with_rowscale_pools(gen.CONFIGS[name](), fmt, seed=4150 + 51)
    dev = RowDevice(wl)
    out = dev.decode_append(wl.partition_size)
    assert dev.status() == 0
    kc, vc, ks, vs, st = _oracle_after_write(wl)
    assert st == 0
    _same_pools(dev, kc, vc, ks, vs, f"{name} {fmt} rows")
    ref, _ = _oracle_decode(wl, kc, vc, ks, vs)
    assert_close_rows(to_f64(out), ref, f"{name} {fmt} rows, every row")


def test_scale_pools_swap_to_host_and_back():
    """Eviction of row-scaled blocks moves their scales too: pa_swap_blocks
    with PA_DTYPE_F32 pools, device -> pinned host -> device, bit for bit
    against the oracle's swap."""
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(45))
    ks = rng.standard_normal((10, 8, 16)).astype(np.float32)
    vs = rng.standard_normal((10, 8, 16)).astype(np.float32)
    dks, dvs = torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda()
    hk = torch.zeros((4, 8, 16), dtype=torch.float32).pin_memory()
    hv = torch.zeros((4, 8, 16), dtype=torch.float32).pin_memory()
    out_pairs = np.array([[2, 0], [7, 3]], np.int64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.pa_swap_blocks(dks, dvs, hk, hv, torch.from_numpy(out_pairs).cuda(), status)
    torch.cuda.synchronize()
    ok_k, ok_v = np.zeros((4, 8, 16), np.float32), np.zeros((4, 8, 16), np.float32)
    assert oracle.swap_blocks(ks, vs, ok_k, ok_v, out_pairs) == 0
    assert np.array_equal(hk.numpy(), ok_k) and np.array_equal(hv.numpy(), ok_v)
    back = np.array([[0, 5], [3, 9]], np.int64)
    B.pa_swap_blocks(hk, hv, dks, dvs, torch.from_numpy(back).cuda(), status)
    torch.cuda.synchronize()
    assert oracle.swap_blocks(ok_k, ok_v, ks, vs, back) == 0
    assert int(status.item()) == 0
    assert np.array_equal(dks.cpu().numpy(), ks) and np.array_equal(dvs.cpu().numpy(), vs)
