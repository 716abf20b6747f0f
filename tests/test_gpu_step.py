"""The step API from pinned host buffers: DecodeStep.run_from_host (one
stream, blocking order) and HostPipeline (uploads, kernels and downloads on
three streams, double-buffered).  Both must give, step by step, exactly the
output of the device-resident step, and that output must match the oracle."""
import numpy as np
import pytest
import torch

from tests import oracle_pins
from tests.gpu_utils import DeviceWorkload, assert_close, oracle_step, to_f64
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _host_inputs(wl, query_bits, fused):
    host = {"query": torch.from_numpy(query_bits.view(np.int16)).view(torch.float16).pin_memory(),
            "block_tables": torch.from_numpy(wl.block_tables).pin_memory(),
            "context_lens": torch.from_numpy(wl.context_lens).pin_memory(),
            "new_key": torch.from_numpy(wl.new_key.view(np.int16)).view(torch.float16).pin_memory(),
            "new_value": torch.from_numpy(wl.new_value.view(np.int16)).view(torch.float16).pin_memory()}
    if not fused:
        host["slot_mapping"] = torch.from_numpy(wl.slot_mapping).pin_memory()
    return host


@pytest.mark.parametrize("fused", [True, False], ids=["fused-append", "separate"])
def test_pipelined_steps_match_device_steps(fused):
    """Six steps, each with its own query, through HostPipeline (eager, then
    with graph replays): every step's host output equals the device-resident
    step on the same query (bit for bit), and the first one matches the
    oracle."""
    from paged_kv_cache_415_b200.step import DecodeStep, HostPipeline
    wl = oracle_pins.small_llama(seqs=6)
    assert wl.extra["one_token_per_seq"]
    rng = np.random.Generator(np.random.PCG64(31))
    queries = [wl.query] + [rng.integers(0, 1 << 15, size=wl.query.shape, dtype=np.uint16) & 0xBBFF
                            for _ in range(5)]             # finite fp16 patterns
    dw = DeviceWorkload(wl)
    stepper = DecodeStep(dw.k_cache, dw.v_cache, wl.num_seqs, wl.num_q_heads,
                         wl.max_context_len, 64)
    like = {"query": dw.query, "block_tables": dw.block_tables, "context_lens": dw.context_lens,
            "new_key": dw.new_key, "new_value": dw.new_value, "out": dw.query}
    if not fused:
        like["slot_mapping"] = dw.slot_mapping
    outs = [torch.empty(wl.query.shape, dtype=torch.float16).pin_memory() for _ in queries]
    for graphs in (False, True):
        pipe = HostPipeline(stepper, like, use_graphs=graphs)
        packed = []
        for q in queries:
            buf, views = pipe.host_buffer()
            for name, t in _host_inputs(wl, q, fused).items():
                views[name].copy_(t)
            packed.append(buf)
        for buf, o in zip(packed, outs):
            pipe.submit(buf, wl.scale, o, fused_append=fused)
        pipe.synchronize()
        if not graphs:
            first = [o.clone() for o in outs]
    for a, o in zip(first, outs):           # graph replays == eager steps
        assert torch.equal(a.view(torch.int16), o.view(torch.int16))
    assert int(stepper.d_status.item()) == 0
    # reference: the same steps on device-resident inputs, one stream
    for q, o in zip(queries, outs):
        dq = torch.from_numpy(q.view(np.int16)).cuda().view(torch.float16)
        ref = stepper(dq, dw.block_tables, dw.context_lens, wl.scale, new_key=dw.new_key,
                      new_value=dw.new_value, slot_mapping=dw.slot_mapping,
                      fused_append=fused)
        torch.cuda.synchronize()
        assert torch.equal(ref.cpu().view(torch.int16), o.view(torch.int16))
    _, _, want, _ = oracle_step(wl)
    assert_close(to_f64(outs[0]), want, "pipelined step 0")


def test_run_from_host_blocking_order():
    from paged_kv_cache_415_b200.step import DecodeStep
    wl = oracle_pins.small_llama(seqs=4)
    dw = DeviceWorkload(wl)
    stepper = DecodeStep(dw.k_cache, dw.v_cache, wl.num_seqs, wl.num_q_heads,
                         wl.max_context_len, 0)
    host = _host_inputs(wl, wl.query, fused=False)
    host["out"] = torch.empty(wl.query.shape, dtype=torch.float16).pin_memory()
    dev = {k: torch.empty_like(v, device="cuda") for k, v in host.items()}
    out = stepper.run_from_host(host, dev, wl.scale)
    torch.cuda.synchronize()
    _, _, want, _ = oracle_step(wl)
    assert_close(to_f64(out), want, "run_from_host")


@pytest.mark.parametrize("make", [gen.tiny, lambda: oracle_pins.small_gqa(seqs=6)],
                         ids=["tiny-copies", "gqa-split"])
def test_graph_replay_matches_eager(make):
    """A step captured into a CUDA graph (block copies, cache write, decode
    and, for split contexts, the merge) replays to exactly the eager step's
    output, also after the captured query buffer is refilled."""
    from paged_kv_cache_415_b200.step import DecodeStep
    wl = make()
    dw = DeviceWorkload(wl)
    part = 64 if wl.max_context_len > 64 else 0
    stepper = DecodeStep(dw.k_cache, dw.v_cache, wl.num_seqs, wl.num_q_heads,
                         wl.max_context_len, part)
    kw = dict(new_key=dw.new_key, new_value=dw.new_value, slot_mapping=dw.slot_mapping,
              block_mapping=dw.block_mapping if wl.block_mapping.shape[0] else None)
    eager = stepper(dw.query, dw.block_tables, dw.context_lens, wl.scale, **kw).clone()
    out = torch.empty_like(dw.query)
    g = stepper.graph(dw.query, dw.block_tables, dw.context_lens, wl.scale, out, **kw)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    _, _, want, _ = oracle_step(wl)
    assert_close(to_f64(out), want, "graph replay")
    q2 = torch.flip(dw.query, dims=[0]).contiguous()
    ref2 = stepper(q2, dw.block_tables, dw.context_lens, wl.scale, **kw).clone()
    dw.query.copy_(q2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))
    assert int(stepper.d_status.item()) == 0


@pytest.mark.parametrize("codes", ["fp8", "int8"])
@pytest.mark.parametrize("fused", [True, False], ids=["fused-append", "separate"])
def test_decode_step_on_code_pools(codes, fused):
    """DecodeStep over one-byte pools picks that format's write and decode
    (fused into one launch, or separate): the pools equal the oracle's
    quantising write bit for bit and the output matches the oracle."""
    from paged_kv_cache_415_b200.step import DecodeStep
    from tests.test_gpu_quantised import Q8Device, _instance, _oracle_decode, _oracle_pools
    wl = _instance(codes, 128, 16, 4, "bf16")
    assert wl.extra["one_token_per_seq"]
    dev = Q8Device(wl)
    stepper = DecodeStep(dev.k_cache, dev.v_cache, wl.num_seqs, wl.num_q_heads,
                         wl.max_context_len, 0, k_scale=dev.ks, v_scale=dev.vs)
    out = stepper(dev.query, dev.block_tables, dev.context_lens, wl.scale,
                  new_key=dev.new_key, new_value=dev.new_value, slot_mapping=dev.slot_mapping,
                  fused_append=fused)
    torch.cuda.synchronize()
    kc, vc, st = _oracle_pools(wl)
    assert st == 0
    assert np.array_equal(dev.k_cache.cpu().numpy(), kc)
    assert np.array_equal(dev.v_cache.cpu().numpy(), vc)
    ref, st = _oracle_decode(wl, kc, vc)
    assert st == 0 and int(stepper.d_status.item()) == 0
    assert_close(to_f64(out), ref, f"{codes} step")
