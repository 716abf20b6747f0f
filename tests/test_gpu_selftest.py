"""The bounded waits, made to run out on purpose (include/pa_selftest.h).

Every wait of the decode kernels for a block's tiles gives up after a
bounded time, sets PA_STATUS_TIMEOUT and lets the kernel finish.  These
tests make waits run out without any fault -- on an mbarrier that nothing
arrives on, with a limit of a millisecond -- and check that:
  * the standalone wait gives up after its limit, not before, and sets the
    status bit in every CTA;
  * in the decode kernels (fp32 path, tensor-core GQA path, one-byte-code
    path, shared-prefix path; one partition and split contexts) the abort
    path runs: the copies already started are drained, every output row is
    written as zeros and the status word is exactly PA_STATUS_TIMEOUT;
  * the context is healthy afterwards: the same decode without the probe
    matches the fp64 oracle in the same process.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins
from tests.gpu_utils import DeviceWorkload, assert_close, oracle_step, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu

LIMIT_US = 1000


def test_standalone_wait_gives_up_after_its_limit():
    from paged_kv_cache_415_b200 import binding as B
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(8, dtype=torch.int64, device="cuda")
    t0 = time.perf_counter()
    B.pa_selftest_bounded_wait(status, LIMIT_US, num_ctas=8, d_wait_ns=waited)
    torch.cuda.synchronize()
    host_s = time.perf_counter() - t0
    assert int(status.item()) == B.PA_STATUS_TIMEOUT
    w = waited.cpu().numpy()
    assert np.all(w >= LIMIT_US * 1000), w                 # not before the limit
    assert np.all(w < LIMIT_US * 1000 + 50_000_000), w     # and soon after it
    assert host_s < 10.0
    # the context still runs kernels: an ordinary decode against the oracle
    _healthy(oracle_pins.small_llama(seqs=3))


def _healthy(wl, partition_size=0):
    dw = DeviceWorkload(wl)
    out = dw.step(partition_size=partition_size)
    torch.cuda.synchronize()
    _, _, ref, st = oracle_step(wl)
    assert dw.status() == 0 and st == 0
    assert_close(to_f64(out), ref, f"{wl.name} after the timeout")


def _probe(dw, partition_size, k_cache=None, v_cache=None):
    from paged_kv_cache_415_b200 import binding as B
    wl = dw.wl
    kc = dw.k_cache if k_cache is None else k_cache
    vc = dw.v_cache if v_cache is None else v_cache
    ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                wl.head_dim, wl.block_size, wl.max_context_len,
                                                partition_size)
    ws = torch.full((max(ws_bytes, 16) // 4,), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.full_like(dw.query, float("nan"))
    dw.d_status.zero_()
    B.pa_selftest_decode_abort(out, dw.query, kc, vc, dw.block_tables, dw.context_lens,
                               wl.max_context_len, wl.scale, LIMIT_US, partition_size,
                               ws.view(torch.uint8), dw.d_status)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("case,partition", [
    ("mha", 0),            # fp32 path, each context one partition: zero rows written directly
    ("mha", 32),           # fp32 path, split contexts: empty partials, then the reduction
    ("gqa", 0),            # tensor-core path
    ("gqa", 16),
    ("long", 512),         # tensor-core path, many partitions of long contexts
])
def test_decode_abort_path(case, partition):
    from paged_kv_cache_415_b200 import binding as B
    wl = {"mha": lambda: oracle_pins.small_llama(seqs=5),
          "gqa": lambda: oracle_pins.small_gqa(),
          "long": lambda: gen.long_context(seqs=2, ctx=3000, num_blocks=400)}[case]()
    dw = DeviceWorkload(wl)
    dw.step(partition_size=partition)             # the step's cache write first
    out = _probe(dw, partition)
    assert dw.status() == B.PA_STATUS_TIMEOUT
    assert not to_f64(out).any(), "every row of a timed-out decode is zero"
    # the same decode without the probe, in the same process
    dw.d_status.zero_()
    got = dw.decode(partition_size=partition)
    torch.cuda.synchronize()
    kc, vc, ref, _ = oracle_step(wl)
    assert dw.status() == 0
    assert_close(to_f64(got), ref, f"{case} after the abort")


@pytest.mark.parametrize("codes", ["fp8", "int8"])
@pytest.mark.parametrize("partition", [0, 32])
@pytest.mark.parametrize("kv_heads", [2, 3])
def test_decode_abort_path_code_pools(codes, partition, kv_heads):
    """Both one-byte kernels: a CTA per pair of kv heads (2) and a CTA per
    kv head (3)."""
    from paged_kv_cache_415_b200 import binding as B
    wl = gen.with_code_pools(oracle_pins.small_gqa(keep_logical=False, kv_heads=kv_heads), codes,
                             seed=77)
    np_t = {"fp8": np.uint8, "int8": np.int8}[codes]
    dw = DeviceWorkload.__new__(DeviceWorkload)
    dw.wl = wl
    dw.query = torch.from_numpy(wl.query.view(np.int16)).cuda().view(torch.bfloat16)
    dw.block_tables = torch.from_numpy(wl.block_tables).cuda()
    dw.context_lens = torch.from_numpy(wl.context_lens).cuda()
    dw.d_status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc = torch.from_numpy(wl.k_cache.view(np_t)).cuda()
    vc = torch.from_numpy(wl.v_cache.view(np_t)).cuda()
    # the history only: the slots of this step's tokens still hold the poison code
    hist = wl.context_lens - 1
    dw.context_lens = torch.from_numpy(hist.astype(np.int32)).cuda()
    wl_hist = gen.DecodeWorkload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    wl_hist.context_lens = hist.astype(np.int32)
    dw.wl = wl_hist
    out = _probe(dw, partition, kc, vc)
    assert dw.status() == B.PA_STATUS_TIMEOUT
    assert not to_f64(out).any()
    # healthy afterwards: the real decode over the same pools against the oracle
    decode = getattr(B, f"pa_paged_decode_{codes}")
    ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                wl.head_dim, wl.block_size, int(hist.max()),
                                                partition)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    got = torch.full_like(dw.query, float("nan"))
    dw.d_status.zero_()
    ks, vs = wl.extra["k_scale"], wl.extra["v_scale"]
    decode(got, dw.query, kc, vc, dw.block_tables, dw.context_lens, int(hist.max()), wl.scale,
           ks, vs, partition, ws, dw.d_status)
    torch.cuda.synchronize()
    ref, st = getattr(oracle, f"paged_decode_{codes}")(wl.query, wl.k_cache, wl.v_cache,
                                                       wl.block_tables, hist.astype(np.int32),
                                                       wl.scale, wl.dtype, ks, vs)
    assert dw.status() == 0 and st == 0
    assert_close(to_f64(got), ref, f"{codes} after the abort")


@pytest.mark.parametrize("partition", [0, 32])
def test_shared_prefix_abort_path(partition):
    from paged_kv_cache_415_b200 import binding as B
    wl = gen.beam_search(prompts=3, beams=4, prompt_len=40, max_new=24, num_heads=4,
                         num_blocks=96)
    dw = DeviceWorkload(wl)
    dw.step(cache_ops=True)
    prefix = torch.from_numpy(wl.extra["prefix_lens"]).cuda()
    mpl = int(wl.extra["prefix_lens"].max())
    ws_bytes = B.pa_paged_decode_shared_prefix_workspace_size(
        wl.num_seqs, 4, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        wl.max_context_len, mpl, partition)
    ws = torch.full((max(ws_bytes, 16) // 4,), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.full_like(dw.query, float("nan"))
    dw.d_status.zero_()
    B.pa_selftest_shared_prefix_abort(out, dw.query, dw.k_cache, dw.v_cache, dw.block_tables,
                                      dw.context_lens, prefix, 4, wl.max_context_len, mpl,
                                      wl.scale, ws.view(torch.uint8), LIMIT_US, partition,
                                      dw.d_status)
    torch.cuda.synchronize()
    assert dw.status() == B.PA_STATUS_TIMEOUT
    assert not to_f64(out).any()
    dw.d_status.zero_()
    got = torch.full_like(dw.query, float("nan"))
    B.pa_paged_decode_shared_prefix(got, dw.query, dw.k_cache, dw.v_cache, dw.block_tables,
                                    dw.context_lens, prefix, 4, wl.max_context_len, mpl, wl.scale,
                                    ws.view(torch.uint8), partition, dw.d_status)
    torch.cuda.synchronize()
    _, _, ref, _ = oracle_step(wl)
    assert dw.status() == 0
    assert_close(to_f64(got), ref, "shared prefix after the abort")
