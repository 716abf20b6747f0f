"""One decode step of one attention layer over a paged KV cache.

    copy_blocks(block_mapping)         copy-on-write copies, if any
    reshape_and_cache(new K/V, slots)  append this step's tokens
    paged_decode(query, ...)           attend over each context, the new
                                       tokens included

``DecodeStep`` owns the scratch the step needs (the split-context workspace
and a device status word), allocated once with torch, and issues the three
C-ABI calls on one stream.  ``HostPipeline`` feeds a ``DecodeStep`` from
pinned host buffers step after step with the host-device copies of one step
overlapping the kernels of the previous one.  Pools of dtype uint8 hold e4m3 codes: the step
then uses the quantising write and the e4m3 decode with the pools' scales.  ``run_from_host`` is the same step fed from
pinned host buffers: it copies the step's inputs to the device, runs the
step and copies the output back, all on the same stream.
"""
from __future__ import annotations

import torch

from . import binding as B


class DecodeStep:
    def __init__(self, k_cache: torch.Tensor, v_cache: torch.Tensor, num_seqs: int,
                 num_q_heads: int, max_context_len: int, partition_size: int = 0,
                 k_scale: float = 1.0, v_scale: float = 1.0):
        self.k_cache, self.v_cache = k_cache, v_cache
        self.fp8 = k_cache.dtype == torch.uint8
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)
        num_blocks, self.block_size, self.num_kv_heads, self.head_dim = k_cache.shape
        self.num_blocks = num_blocks
        self.num_seqs, self.num_q_heads = num_seqs, num_q_heads
        self.max_context_len = max_context_len
        self.partition_size = B.pa_paged_decode_partition_size(
            num_seqs, num_q_heads, self.num_kv_heads, self.head_dim, self.block_size,
            max_context_len, partition_size)
        if self.partition_size <= 0:
            raise B.PAError("pa_paged_decode_partition_size", B.PA_ERR_INVALID_ARG)
        ws = B.pa_paged_decode_workspace_size(num_seqs, num_q_heads, self.num_kv_heads,
                                              self.head_dim, self.block_size, max_context_len,
                                              self.partition_size)
        dev = k_cache.device
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev) if ws else None
        self.d_status = torch.zeros(1, dtype=torch.int32, device=dev)

    def __call__(self, query, block_tables, context_lens, scale, out=None, new_key=None,
                 new_value=None, slot_mapping=None, block_mapping=None, stream=None,
                 max_context_len=None, fused_append=False):
        """fused_append: every sequence appends exactly one token (new_key /
        new_value hold one row per sequence, at position context_lens - 1);
        the cache write then runs inside the decode launch
        (pa_paged_decode_append) and slot_mapping is not used."""
        if block_mapping is not None and block_mapping.shape[0] > 0:
            B.pa_copy_blocks(self.k_cache, self.v_cache, block_mapping, self.d_status, stream)
        if out is None:
            out = torch.empty_like(query)
        mcl = self.max_context_len if max_context_len is None else max_context_len
        if self.fp8:
            if fused_append:
                B.pa_paged_decode_fp8_append(out, query, new_key, new_value, self.k_cache,
                                             self.v_cache, block_tables, context_lens, mcl, scale,
                                             self.k_scale, self.v_scale, self.partition_size,
                                             self.workspace, self.d_status, stream)
                return out
            if slot_mapping is not None and slot_mapping.shape[0] > 0:
                B.pa_reshape_and_cache_fp8(new_key, new_value, self.k_cache, self.v_cache,
                                           slot_mapping, self.k_scale, self.v_scale,
                                           self.d_status, stream)
            B.pa_paged_decode_fp8(out, query, self.k_cache, self.v_cache, block_tables,
                                  context_lens, mcl, scale, self.k_scale, self.v_scale,
                                  self.partition_size, self.workspace, self.d_status, stream)
            return out
        if fused_append:
            B.pa_paged_decode_append(out, query, new_key, new_value, self.k_cache, self.v_cache,
                                     block_tables, context_lens, mcl, scale, self.partition_size,
                                     self.workspace, self.d_status, stream)
            return out
        if slot_mapping is not None and slot_mapping.shape[0] > 0:
            B.pa_reshape_and_cache(new_key, new_value, self.k_cache, self.v_cache, slot_mapping,
                                   self.d_status, stream)
        B.pa_paged_decode(out, query, self.k_cache, self.v_cache, block_tables, context_lens, mcl,
                          scale, self.partition_size, self.workspace, self.d_status, stream)
        return out

    def graph(self, query, block_tables, context_lens, scale, out, new_key=None, new_value=None,
              slot_mapping=None, block_mapping=None, fused_append=False):
        """Capture one step on these device buffers into a CUDA graph and
        return it (``torch.cuda.CUDAGraph``); ``replay()`` re-runs the step's
        launches with no host work per launch.  The step runs once eagerly on
        a side stream first, so every per-kernel setting is in place before
        capture.  Refill the captured buffers in place between replays."""
        args = dict(out=out, new_key=new_key, new_value=new_value, slot_mapping=slot_mapping,
                    block_mapping=block_mapping, fused_append=fused_append)
        side = torch.cuda.Stream(device=query.device)
        side.wait_stream(torch.cuda.current_stream(query.device))
        with torch.cuda.stream(side):
            self(query, block_tables, context_lens, scale, stream=side, **args)
        torch.cuda.current_stream(query.device).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self(query, block_tables, context_lens, scale,
                 stream=torch.cuda.current_stream(query.device), **args)
        return g

    def run_from_host(self, host: dict, dev: dict, scale, stream=None, fused_append=False):
        """host / dev: dicts of same-shaped tensors (pinned host / device) for
        'query', 'block_tables', 'context_lens', 'new_key', 'new_value',
        'slot_mapping', 'block_mapping' (the last four optional) and 'out'.
        Copies host -> device, runs the step, copies out -> host, all on
        ``stream`` (default: the current stream)."""
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            for name, h in host.items():
                if name != "out":
                    dev[name].copy_(h, non_blocking=True)
            self(dev["query"], dev["block_tables"], dev["context_lens"], scale, out=dev["out"],
                 new_key=dev.get("new_key"), new_value=dev.get("new_value"),
                 slot_mapping=dev.get("slot_mapping"), block_mapping=dev.get("block_mapping"),
                 stream=s, fused_append=fused_append)
            host["out"].copy_(dev["out"], non_blocking=True)
        return host["out"]


class HostPipeline:
    """Runs a DecodeStep once per call of ``submit`` from pinned host inputs,
    with the copies of consecutive steps overlapping the kernels.

    Three streams: uploads (host -> device), the step's kernels, downloads
    (device -> host).  Device inputs and outputs are double-buffered, so the
    upload of step i+1 runs while step i computes, and the download of step
    i's output runs while step i+1 computes.  Events order each buffer's
    reuse: an upload into set b waits until the step that last read set b
    has finished, a download waits for its step, and the step waits for its
    upload.  Every step still copies all of its own inputs in and its output
    out; only the waiting is overlapped.  Kernels of consecutive steps stay
    in order on the compute stream (the cache writes of one step precede the
    next step's reads).
    """

    def __init__(self, stepper: DecodeStep, dev_like: dict, device=None):
        """dev_like: name -> device tensor giving the shape and dtype of each
        input ('query', 'block_tables', 'context_lens' and the optional
        'new_key', 'new_value', 'slot_mapping', 'block_mapping') and 'out'."""
        self.stepper = stepper
        dev = device if device is not None else stepper.k_cache.device
        self.sets = [{k: torch.empty_like(t, device=dev) for k, t in dev_like.items()}
                     for _ in range(2)]
        self.up = torch.cuda.Stream(dev)
        self.compute = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.uploaded = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.downloaded = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]
        self.i = 0

    def submit(self, host: dict, scale, host_out: torch.Tensor, fused_append=False):
        """Enqueue one step: host holds pinned inputs by name, host_out the
        pinned tensor that receives the output.  Returns without waiting;
        host_out is valid after ``synchronize`` (or the download stream's
        work up to this step) completes.  The host input tensors must not be
        modified until the upload of this step has run."""
        b = self.i % 2
        dev = self.sets[b]
        if self.used[b]:
            self.up.wait_event(self.computed[b])        # the step that last read set b
            self.compute.wait_event(self.downloaded[b])  # its output has left set b's 'out'
        with torch.cuda.stream(self.up):
            for name, h in host.items():
                dev[name].copy_(h, non_blocking=True)
            self.uploaded[b].record(self.up)
        self.compute.wait_event(self.uploaded[b])
        self.stepper(dev["query"], dev["block_tables"], dev["context_lens"], scale, out=dev["out"],
                     new_key=dev.get("new_key"), new_value=dev.get("new_value"),
                     slot_mapping=dev.get("slot_mapping"), block_mapping=dev.get("block_mapping"),
                     stream=self.compute, fused_append=fused_append)
        self.computed[b].record(self.compute)
        self.down.wait_event(self.computed[b])
        with torch.cuda.stream(self.down):
            host_out.copy_(dev["out"], non_blocking=True)
            self.downloaded[b].record(self.down)
        self.used[b] = True
        self.i += 1
        return host_out

    def synchronize(self):
        for st in (self.up, self.compute, self.down):
            st.synchronize()
