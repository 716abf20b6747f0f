"""pa_paged_decode_no_alloc: the decode entry point for callers that cannot
allocate device memory (a plugin inside a framework that owns every device
allocation, or a latency-critical path that must not call cudaMalloc).  Its
split-context scratch is the library's own fixed device array.

Checked through the C ABI on two calls in a row: each output must be bit
for bit the output of pa_paged_decode with a caller workspace on the same
partition (the same kernels run in the same order, so any difference would
be a scratch-aliasing error), and within the tolerance of the other GPU
tests of the fp64 oracle.  The first call leaves the larger footprint in
the shared array, so the second runs over its leftovers.  A shape that
needs more scratch than the array holds is refused before any work is
enqueued.  Self-contained: it passes alone in a fresh process and after the
other tests.
"""
import numpy as np
import pytest
import torch

from tests.gpu_utils import DeviceWorkload, assert_close, oracle_step, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _scratch_bytes(wl, partition_size):
    from paged_kv_cache_415_b200 import binding as B
    return B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                            wl.head_dim, wl.block_size, wl.max_context_len,
                                            partition_size)


def _both(wl, partition_size):
    """(no_alloc output, caller-workspace output, oracle output)."""
    from paged_kv_cache_415_b200 import binding as B
    dw = DeviceWorkload(wl)
    ref = dw.step(partition_size=partition_size)         # caller-owned workspace
    need = _scratch_bytes(wl, partition_size)
    assert 0 < need <= B.PA_NO_ALLOC_WORKSPACE_BYTES
    out = torch.full_like(dw.query, float("nan"))
    B.pa_paged_decode_no_alloc(out, dw.query, dw.k_cache, dw.v_cache, dw.block_tables,
                               dw.context_lens, wl.max_context_len, wl.scale, partition_size,
                               dw.d_status)
    torch.cuda.synchronize()
    assert dw.status() == 0
    _, _, oracle_out, st = oracle_step(wl)
    assert st == 0
    return out, ref, oracle_out


def test_no_alloc_matches_caller_workspace_twice_in_a_row():
    # call 1: 4 x 6000-token bf16 GQA contexts in 256-token partitions (1.6 MB of scratch)
    wl1 = gen.long_context(seqs=4, ctx=6000, num_blocks=1600)
    # call 2: a different fp16 MHA shape and partition, a smaller footprint (0.33 MB)
    wl2 = gen.make_decode("second", seed=99, dtype="f16",
                          context_lens=np.array([1, 70, 333, 1024, 17], np.int32),
                          num_q_heads=8, num_kv_heads=8, head_dim=128, block_size=16,
                          num_blocks=128, scale=1 / np.sqrt(128.0))
    assert _scratch_bytes(wl1, 256) > _scratch_bytes(wl2, 64)
    for i, (wl, part) in enumerate([(wl1, 256), (wl2, 64)], start=1):
        got, ref, oracle_out = _both(wl, part)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), \
            f"no_alloc call {i}: not bit-identical to pa_paged_decode"
        assert_close(to_f64(got), oracle_out, f"no_alloc call {i} against the oracle")


def test_no_alloc_refuses_oversized_scratch():
    from paged_kv_cache_415_b200 import binding as B
    s, hq, d = 64, 32, 128
    q = torch.zeros(s, hq, d, dtype=torch.float16, device="cuda")
    out = torch.zeros_like(q)
    kc = torch.zeros(4, 16, hq, d, dtype=torch.float16, device="cuda")
    tables = torch.zeros(s, 512, dtype=torch.int32, device="cuda")
    lens = torch.full((s,), 8192, dtype=torch.int32, device="cuda")
    need = B.pa_paged_decode_workspace_size(s, hq, hq, d, 16, 8192, 16)
    assert need > B.PA_NO_ALLOC_WORKSPACE_BYTES
    with pytest.raises(B.PAError) as e:
        B.pa_paged_decode_no_alloc(out, q, kc, kc, tables, lens, 8192, 0.1, 16)
    assert e.value.code == B.PA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert not out.any()                                  # nothing ran
