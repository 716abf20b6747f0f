"""Quantised K/V pools (e4m3 and int8 codes) on the GPU against the oracle.

Every test runs for both code formats.  The quantising cache write is
compared bit for bit with the oracle over the whole pool (every untouched
byte included).  Decode over the codes is compared with the fp64 oracle of
the dequantised pools at the tolerance of the 16-bit path,
|gpu - oracle| <= 2e-3 + 1e-2 |oracle|: the codes of both formats widen to
fp16 exactly, so the only extra rounding is the query's to fp16 (exact for
fp16 queries; for bf16 ones it only touches values below 2^-14) next to the
probabilities' rounding that the 16-bit tensor-core path has already."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins
from tests.gpu_utils import assert_close, assert_close_rows, to_dev, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu

CODES = ["fp8", "int8"]
_NP = {"fp8": np.uint8, "int8": np.int8}


def _pool(a: np.ndarray, codes: str) -> torch.Tensor:
    """Raw code bytes on the device: uint8 for e4m3, int8 for int8 pools."""
    return torch.from_numpy(np.ascontiguousarray(a).view(_NP[codes])).cuda()


def _random_pool(rng, shape, codes):
    return rng.integers(0, 256, size=shape, dtype=np.uint8).view(_NP[codes])


def _calls(codes):
    """(cache write, decode, decode with fused write) of the binding."""
    from paged_kv_cache_415_b200 import binding as B
    return (getattr(B, f"pa_reshape_and_cache_{codes}"), getattr(B, f"pa_paged_decode_{codes}"),
            getattr(B, f"pa_paged_decode_{codes}_append"))


def _oracle_calls(codes):
    return (getattr(oracle, f"reshape_and_cache_{codes}"), getattr(oracle, f"paged_decode_{codes}"))


class Q8Device:
    """A with_code_pools workload on the device; step = write, then decode."""

    def __init__(self, wl):
        self.wl = wl
        self.codes = wl.extra["kv_dtype"]
        self.query = to_dev(wl.query, wl.dtype)
        self.k_cache, self.v_cache = _pool(wl.k_cache, self.codes), _pool(wl.v_cache, self.codes)
        self.block_tables = torch.from_numpy(wl.block_tables).cuda()
        self.context_lens = torch.from_numpy(wl.context_lens).cuda()
        self.new_key = to_dev(wl.new_key, wl.dtype)
        self.new_value = to_dev(wl.new_value, wl.dtype)
        self.slot_mapping = torch.from_numpy(wl.slot_mapping).cuda()
        self.d_status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.ks, self.vs = wl.extra["k_scale"], wl.extra["v_scale"]

    def write(self):
        _calls(self.codes)[0](self.new_key, self.new_value, self.k_cache, self.v_cache,
                              self.slot_mapping, self.ks, self.vs, self.d_status)

    def decode(self, partition_size=None, block_tables=None, context_lens=None,
               max_context_len=None):
        from paged_kv_cache_415_b200 import binding as B
        wl = self.wl
        p = wl.partition_size if partition_size is None else partition_size
        bt = self.block_tables if block_tables is None else block_tables
        cl = self.context_lens if context_lens is None else context_lens
        mcl = wl.max_context_len if max_context_len is None else max_context_len
        ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                    wl.head_dim, wl.block_size, mcl, p)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
        out = torch.full_like(self.query, float("nan"))
        _calls(self.codes)[1](out, self.query, self.k_cache, self.v_cache, bt, cl, mcl, wl.scale,
                              self.ks, self.vs, p, ws, self.d_status)
        return out

    def status(self) -> int:
        return int(self.d_status.item())


def _oracle_pools(wl):
    kc, vc = wl.k_cache.copy(), wl.v_cache.copy()
    st = _oracle_calls(wl.extra["kv_dtype"])[0](wl.new_key, wl.new_value, kc, vc,
                                                wl.slot_mapping, wl.block_size, wl.dtype,
                                                wl.extra["k_scale"], wl.extra["v_scale"])
    return kc, vc, st


def _oracle_decode(wl, kc, vc, tables=None, ctx=None):
    tables = wl.block_tables if tables is None else tables
    ctx = wl.context_lens if ctx is None else ctx
    return _oracle_calls(wl.extra["kv_dtype"])[1](wl.query, kc, vc, tables, ctx, wl.scale,
                                                  wl.dtype, wl.extra["k_scale"],
                                                  wl.extra["v_scale"])


def _parity(wl, partition_size=None, what="", row_scaled_tolerance=False):
    dev = Q8Device(wl)
    dev.write()
    out = dev.decode(partition_size)
    torch.cuda.synchronize()
    kc, vc, st = _oracle_pools(wl)
    assert st == 0
    assert np.array_equal(dev.k_cache.cpu().numpy(), kc), f"{what}: K pool"
    assert np.array_equal(dev.v_cache.cpu().numpy(), vc), f"{what}: V pool"
    ref, st = _oracle_decode(wl, kc, vc)
    assert st == 0
    (assert_close_rows if row_scaled_tolerance else assert_close)(to_f64(out), ref, what or wl.name)
    assert dev.status() == 0
    return dev, out


# ---- the quantising cache write -------------------------------------------------

@pytest.mark.parametrize("codes", CODES)
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("scales", [(1 / 64, 1 / 64), (0.0371, 0.2113)], ids=["pow2", "odd"])
def test_cache_write_bit_exact(codes, dtype, scales):
    """Random codes in the pools (a stray write anywhere shows), a mix of
    ordinary, saturating and special values (inf, NaN, -0) in the rows,
    padding slots (-1) and one slot past the pool (status 2)."""
    rng = np.random.Generator(np.random.PCG64(31 if dtype == "f16" else 32))
    nb, b, h, d = 24, 16, 4, 128
    kc = _random_pool(rng, (nb, b, h, d), codes)
    vc = _random_pool(rng, (nb, b, h, d), codes)
    t = 40
    x = rng.standard_normal((2, t, h, d)).astype(np.float32)
    x[:, ::3] *= 40.0                                       # saturates for small scales
    x[0, 1, 0, :4] = [np.inf, -np.inf, np.nan, -0.0]
    key = gen.f32_to_bits(x[0], dtype)
    val = gen.f32_to_bits(x[1], dtype)
    slots = rng.permutation(nb * b)[:t].astype(np.int64)
    slots[5] = -1
    slots[9] = nb * b + 3
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dk, dv = _pool(kc, codes), _pool(vc, codes)
    _calls(codes)[0](to_dev(key, dtype), to_dev(val, dtype), dk, dv,
                     torch.from_numpy(slots).cuda(), scales[0], scales[1], status)
    torch.cuda.synchronize()
    ek, ev = kc.copy(), vc.copy()
    st = _oracle_calls(codes)[0](key, val, ek, ev, slots, b, dtype, scales[0], scales[1])
    assert np.array_equal(dk.cpu().numpy(), ek)
    assert np.array_equal(dv.cpu().numpy(), ev)
    assert int(status.item()) == st == 2


@pytest.mark.parametrize("codes", CODES)
def test_cache_write_rejects_bad_scales(codes):
    from paged_kv_cache_415_b200 import binding as B
    kc = torch.zeros((4, 16, 2, 64), dtype=torch.from_numpy(np.zeros(1, _NP[codes])).dtype,
                     device="cuda")
    key = torch.zeros((1, 2, 64), dtype=torch.float16, device="cuda")
    slots = torch.zeros(1, dtype=torch.int64, device="cuda")
    for ks in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(B.PAError):
            _calls(codes)[0](key, key, kc, kc.clone(), slots, ks, 1.0)
    assert not kc.any()


@pytest.mark.parametrize("codes", CODES)
def test_copy_blocks_on_code_pools(codes):
    """pa_copy_blocks with the one-byte element type moves whole blocks of
    codes (checked against the oracle's copy on the same bytes)."""
    from paged_kv_cache_415_b200 import binding as B
    rng = np.random.Generator(np.random.PCG64(33))
    kc = _random_pool(rng, (12, 16, 2, 64), codes)
    vc = _random_pool(rng, (12, 16, 2, 64), codes)
    m = np.array([[1, 4], [7, 2], [3, 11]], dtype=np.int64)
    dk, dv = _pool(kc, codes), _pool(vc, codes)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.pa_copy_blocks(dk, dv, torch.from_numpy(m).cuda(), status)
    torch.cuda.synchronize()
    # the oracle copies 16-bit elements: the same bytes seen as pairs
    ek, ev = kc.copy().view(np.uint16), vc.copy().view(np.uint16)
    assert oracle.copy_blocks(ek, ev, m) == 0
    assert np.array_equal(dk.cpu().numpy(), ek.view(_NP[codes]))
    assert np.array_equal(dv.cpu().numpy(), ev.view(_NP[codes]))
    assert int(status.item()) == 0


# ---- decode over the codes --------------------------------------------------------

def _instance(codes, head_dim, block_size, group, dtype, partition_blocks=4, hkv=2):
    rng = np.random.Generator(np.random.PCG64(head_dim * 1000 + block_size * 10 + group + 5))
    ctx = rng.integers(1, 300, size=3, endpoint=True)
    ctx[0] = 1
    nb = int(sum(-(-int(c) // block_size) for c in ctx)) + 8
    wl = gen.make_decode("q8-instance", seed=78, dtype=dtype, context_lens=ctx,
                         num_q_heads=hkv * group, num_kv_heads=hkv, head_dim=head_dim,
                         block_size=block_size, num_blocks=nb, scale=1 / math.sqrt(head_dim),
                         partition_size=partition_blocks * block_size)
    return gen.with_code_pools(wl, codes, seed=head_dim + block_size + group)


@pytest.mark.parametrize("codes", CODES)
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("block_size", [16, 32])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_every_code_instance(head_dim, block_size, group, dtype, codes):
    """Each (head_dim, block_size, group, query dtype) instance on ragged
    contexts spanning several blocks, warps and partitions of 4 blocks."""
    _parity(_instance(codes, head_dim, block_size, group, dtype),
            what=f"{codes} D{head_dim} B{block_size} G{group} {dtype}")


@pytest.mark.parametrize("codes", CODES)
@pytest.mark.parametrize("partition", [16, 512, 0, 1024])
def test_code_partition_sweep(partition, codes):
    """Partitions below 16 blocks per warp take the kernel with a CTA per
    pair of kv heads, 1024 tokens (64 blocks) the one with a CTA per kv head."""
    wl = gen.with_code_pools(oracle_pins.small_gqa(seqs=6), codes, seed=40)
    _parity(wl, partition_size=partition, what=f"{codes} gqa P{partition}")


@pytest.mark.parametrize("codes", CODES)
def test_code_odd_scales_and_single_token(codes):
    """Scales that are not powers of two; a one-token context returns
    v_scale * v0 (to output rounding)."""
    wl = oracle_pins.small_llama(seqs=5)
    ctx = wl.context_lens.copy()
    ctx[0] = 1
    wl = gen.make_decode("q8-odd", seed=79, dtype="bf16", context_lens=ctx, num_q_heads=8,
                         num_kv_heads=8, head_dim=128, block_size=16, num_blocks=160,
                         scale=1 / math.sqrt(128))
    pools = {"fp8": gen.with_fp8_pools, "int8": gen.with_int8_pools}[codes]
    wl = pools(wl, seed=41, k_scale=0.0371, v_scale=0.2113)
    _parity(wl, partition_size=64, what=f"{codes} odd scales")


@pytest.mark.parametrize("codes", CODES)
def test_code_unsupported_and_invalid(codes):
    """Block size 8 has no one-byte tile path (UNSUPPORTED); non-positive or
    non-finite scales are INVALID_ARG; nothing is written."""
    from paged_kv_cache_415_b200 import binding as B
    wl8 = gen.make_decode("q8-b8", seed=80, dtype="f16", context_lens=[20, 5], num_q_heads=2,
                          num_kv_heads=2, head_dim=64, block_size=8, num_blocks=8, scale=0.125)
    wl8 = gen.with_code_pools(wl8, codes, seed=42)
    dev = Q8Device(wl8)
    with pytest.raises(B.PAError, match="UNSUPPORTED|unsupported"):
        dev.decode()
    dev = Q8Device(_instance(codes, 64, 16, 1, "f16"))
    for ks in (0.0, float("nan")):
        dev.ks = ks
        with pytest.raises(B.PAError):
            dev.decode()


@pytest.mark.parametrize("codes", CODES)
def test_code_empty_context_and_bad_block(codes):
    """ctx 0 -> zero row; an out-of-pool block id is skipped and flagged
    (status 1) exactly as the oracle does."""
    wl = gen.with_code_pools(oracle_pins.small_llama(seqs=4), codes, seed=43)
    kc, vc, _ = _oracle_pools(wl)
    wl.k_cache, wl.v_cache = kc, vc
    dev = Q8Device(wl)
    ctx = wl.context_lens.copy()
    ctx[0] = 0
    out = dev.decode(context_lens=torch.from_numpy(ctx).cuda(), partition_size=64)
    ref, st = _oracle_decode(wl, kc, vc, ctx=ctx)
    assert_close(to_f64(out), ref)
    assert dev.status() == st == 0
    tables = wl.block_tables.copy()
    s = int(np.argmax(wl.context_lens))
    tables[s, 0] = wl.num_blocks + 7
    out = dev.decode(block_tables=torch.from_numpy(tables).cuda(), partition_size=64)
    ref, st = _oracle_decode(wl, kc, vc, tables=tables)
    assert st == 1 and dev.status() == 1
    assert_close(to_f64(out), ref)


@pytest.mark.parametrize("codes", CODES)
def test_code_bad_context(codes):
    """A negative context gives a zero row and PA_STATUS_BAD_CONTEXT, the other
    rows are unaffected, for a small batch and for one of 300 sequences."""
    for seqs in (5, 300):
        ctx = np.random.Generator(np.random.PCG64(seqs)).integers(1, 70, size=seqs, endpoint=True)
        nb = int(sum(-(-int(c) // 16) for c in ctx)) + 8
        wl = gen.make_decode("q8-many", seed=81, dtype="bf16", context_lens=ctx, num_q_heads=4,
                             num_kv_heads=2, head_dim=64, block_size=16, num_blocks=nb,
                             scale=0.125, partition_size=32)
        wl = gen.with_code_pools(wl, codes, seed=45)
        kc, vc, _ = _oracle_pools(wl)
        wl.k_cache, wl.v_cache = kc, vc
        dev = Q8Device(wl)
        bad = wl.context_lens.copy()
        bad[1] = -3
        out = dev.decode(context_lens=torch.from_numpy(bad).cuda())
        ref, st = _oracle_decode(wl, kc, vc, ctx=bad)
        assert st == 4 and dev.status() == 4, (seqs, st, dev.status())
        assert_close(to_f64(out), ref, f"{seqs} seqs")


@pytest.mark.parametrize("codes", CODES)
def test_code_deterministic(codes):
    wl = _instance(codes, 128, 16, 4, "bf16")
    dev = Q8Device(wl)
    dev.write()
    a = dev.decode()
    b = dev.decode()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.slow
@pytest.mark.parametrize("codes", CODES)
@pytest.mark.parametrize("name", ["llama7b", "mistral7b", "long_context"])
def test_code_full_size(name, codes):
    """The full-size workload with quantised pools (long_context: the
    kernel with a CTA per pair of kv heads): write + decode against the
    whole oracle."""
    wl = gen.with_code_pools(gen.CONFIGS[name](), codes, seed=44)
    _parity(wl, what=f"{name}-{codes}")


# ---- the quantising write fused into the decode launch ----------------------------

def _fused(wl, partition_size=None, tables=None):
    from paged_kv_cache_415_b200 import binding as B
    dev = Q8Device(wl)
    p = wl.partition_size if partition_size is None else partition_size
    ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                wl.head_dim, wl.block_size, wl.max_context_len, p)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    out = torch.full_like(dev.query, float("nan"))
    bt = dev.block_tables if tables is None else torch.from_numpy(tables).cuda()
    _calls(dev.codes)[2](out, dev.query, dev.new_key, dev.new_value, dev.k_cache, dev.v_cache,
                         bt, dev.context_lens, wl.max_context_len, wl.scale, dev.ks, dev.vs, p,
                         ws, dev.d_status)
    torch.cuda.synchronize()
    return dev, out


@pytest.mark.slow
@pytest.mark.parametrize("codes", CODES)
@pytest.mark.parametrize("name", ["mistral7b", "long_context"])
def test_code_fused_append_full_size(name, codes):
    """The entry point the benchmark times on one-byte pools (quantising
    write fused into the decode, the workload's partitions), at full size:
    both pools bit for bit and every output row against the oracle."""
    wl = gen.with_code_pools(gen.CONFIGS[name](), codes, seed=45)
    assert wl.extra["one_token_per_seq"]
    dev, out = _fused(wl)
    kc, vc, st = _oracle_pools(wl)
    assert st == 0
    assert np.array_equal(dev.k_cache.cpu().numpy(), kc), f"{name}-{codes}: K pool"
    assert np.array_equal(dev.v_cache.cpu().numpy(), vc), f"{name}-{codes}: V pool"
    ref, st = _oracle_decode(wl, kc, vc)
    assert st == 0 and dev.status() == 0
    assert_close(to_f64(out), ref, f"{name}-{codes} fused, every row")


@pytest.mark.parametrize("codes", CODES)
@pytest.mark.parametrize("head_dim,block_size,group,dtype,partition",
                         [(128, 16, 1, "f16", 0), (128, 16, 4, "bf16", 64), (64, 32, 2, "f16", 0),
                          (128, 32, 8, "bf16", 96)])
def test_code_fused_append(head_dim, block_size, group, dtype, partition, codes):
    """The fused decode (pa_paged_decode_fp8_append / _int8_append) leaves
    the pools exactly as the quantising cache write does and returns the
    decode of the written pools."""
    wl = _instance(codes, head_dim, block_size, group, dtype)
    assert wl.extra["one_token_per_seq"]
    dev, out = _fused(wl, partition)
    kc, vc, st = _oracle_pools(wl)
    assert st == 0
    assert np.array_equal(dev.k_cache.cpu().numpy(), kc)
    assert np.array_equal(dev.v_cache.cpu().numpy(), vc)
    ref, st = _oracle_decode(wl, kc, vc)
    assert st == 0 and dev.status() == 0
    assert_close(to_f64(out), ref, f"{codes} fused append")


@pytest.mark.parametrize("codes", CODES)
@pytest.mark.parametrize("hkv,group,head_dim,block_size,dtype", [
    (1, 4, 128, 16, "bf16"), (3, 2, 128, 16, "f16"), (5, 1, 64, 32, "bf16"), (3, 8, 128, 32, "f16")])
def test_code_odd_kv_heads(hkv, group, head_dim, block_size, dtype, codes):
    """An odd number of kv heads takes the kernel with a CTA per kv head (an
    even number takes a CTA per pair of adjacent kv heads): decode over
    partitions of 4 blocks, then the fused append, against the oracle."""
    wl = _instance(codes, head_dim, block_size, group, dtype, hkv=hkv)
    _parity(wl, what=f"{codes} Hkv{hkv} G{group} D{head_dim} B{block_size} {dtype}")
    dev, out = _fused(wl)
    kc, vc, st = _oracle_pools(wl)
    assert st == 0
    assert np.array_equal(dev.k_cache.cpu().numpy(), kc)
    assert np.array_equal(dev.v_cache.cpu().numpy(), vc)
    ref, st = _oracle_decode(wl, kc, vc)
    assert st == 0 and dev.status() == 0
    assert_close(to_f64(out), ref, f"{codes} Hkv{hkv} fused append")


@pytest.mark.parametrize("codes", CODES)
def test_code_fused_append_bad_slot_is_flagged(codes):
    """A new token whose block id lies outside the pool is not written
    (PA_STATUS_BAD_SLOT, plus PA_STATUS_BAD_BLOCK for the skipped block)."""
    wl = _instance(codes, 128, 16, 4, "bf16")
    s = int(np.argmax(wl.context_lens))
    c = int(wl.context_lens[s])
    tables = wl.block_tables.copy()
    tables[s, (c - 1) // 16] = wl.num_blocks + 3
    dev, _ = _fused(wl, 0, tables)
    assert dev.status() & 2 and dev.status() & 1
    # every other new token is written as the quantising write would
    keep = np.ones(wl.num_seqs, bool)
    keep[s] = False
    kc, vc = wl.k_cache.copy(), wl.v_cache.copy()
    _oracle_calls(codes)[0](wl.new_key[keep], wl.new_value[keep], kc, vc, wl.slot_mapping[keep],
                            wl.block_size, wl.dtype, wl.extra["k_scale"], wl.extra["v_scale"])
    assert np.array_equal(dev.k_cache.cpu().numpy(), kc)
    assert np.array_equal(dev.v_cache.cpu().numpy(), vc)


# ---- int8 pools: the widening leaves a bias of 1152 that the kernel removes ------

@pytest.mark.parametrize("group", [1, 4])
@pytest.mark.parametrize("partition", [0, 8192])
def test_int8_bias_removal_under_stress(group, partition):
    """int8 codes widen to 1152 + c; the kernel subtracts 1152 * sum(q) from
    every score and 1152 * sum(p) from the output.  Stress both: scales of 1
    (codes are the values, up to +-127), a query that is positive in every
    dim (sum(q) as large as it gets), contexts up to 8192 tokens and, with an
    8192-token partition, one warp accumulating 128 blocks.  With scales of
    1 the outputs are up to ~127 (the fp16 rounding of P alone moves them by
    ~0.03), so the absolute part of the tolerance scales with each output
    row's magnitude (assert_close_rows)."""
    hkv = 2
    wl = gen.make_decode("int8-bias", seed=4150 + 90 + group, dtype="f16",
                         context_lens=np.array([8192, 3000, 1], np.int32),
                         num_q_heads=hkv * group, num_kv_heads=hkv, head_dim=128, block_size=16,
                         num_blocks=800, scale=1.0 / 128.0)
    q = np.abs(wl.query.view(np.float16).astype(np.float32)) * 2.0 + 0.5
    wl.query = gen.f32_to_bits(q, "f16")
    wl = gen.with_code_pools(wl, "int8", seed=4150 + 91)
    wl.extra["k_scale"] = 1.0
    wl.extra["v_scale"] = 1.0
    _parity(wl, partition, f"int8 bias stress G={group} P={partition}", row_scaled_tolerance=True)
