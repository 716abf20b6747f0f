"""One decode step of one attention layer over a paged KV cache.

    copy_blocks(block_mapping)         copy-on-write copies, if any
    reshape_and_cache(new K/V, slots)  append this step's tokens
    paged_decode(query, ...)           attend over each context, the new
                                       tokens included

``DecodeStep`` owns the scratch the step needs (the split-context workspace
and a device status word), allocated once with torch, and issues the three
C-ABI calls on one stream.  ``HostPipeline`` feeds a ``DecodeStep`` from
pinned host buffers step after step with the host-device copies of one step
overlapping the kernels of the previous one.  Pools of dtype uint8 (or
float8_e4m3fn) hold e4m3 codes and pools of dtype int8 hold int8 codes: the
step then uses that format's quantising write and decode with the pools'
scales.  ``run_from_host`` is the same step fed from pinned host buffers: it
copies the step's inputs to the device, runs the step and copies the output
back, all on the same stream.

Tracing: every step and each of its calls is an NVTX range on the host
thread that issues it ("pa.step", "pa.copy_blocks", "pa.cache_write",
"pa.decode"; in ``HostPipeline`` also "pa.upload" and "pa.download"), so a
timeline profiler shows which launches belong to which step.  Without a
profiler attached the ranges cost a few hundred nanoseconds of host time.
"""
from __future__ import annotations

import torch

from . import binding as B

_range = torch.cuda.nvtx.range        # NVTX range on the issuing host thread


# Pool dtype -> (cache write, decode, decode with fused write) of that code format.
_QUANTISED_CALLS = {
    torch.uint8: ("pa_reshape_and_cache_fp8", "pa_paged_decode_fp8", "pa_paged_decode_fp8_append"),
    torch.float8_e4m3fn: ("pa_reshape_and_cache_fp8", "pa_paged_decode_fp8",
                          "pa_paged_decode_fp8_append"),
    torch.int8: ("pa_reshape_and_cache_int8", "pa_paged_decode_int8",
                 "pa_paged_decode_int8_append"),
}


class DecodeStep:
    def __init__(self, k_cache: torch.Tensor, v_cache: torch.Tensor, num_seqs: int,
                 num_q_heads: int, max_context_len: int, partition_size: int = 0,
                 k_scale: float = 1.0, v_scale: float = 1.0, k_scales: torch.Tensor = None,
                 v_scales: torch.Tensor = None):
        """k_scales / v_scales: fp32 row-scale pools [num_blocks][Hkv][B] of
        one-byte code pools (one scale per (token, kv head) row; the
        _rowscale calls), or None for one scale per pool (k_scale, v_scale)."""
        self.k_cache, self.v_cache = k_cache, v_cache
        self.k_scales, self.v_scales = k_scales, v_scales
        names = _QUANTISED_CALLS.get(k_cache.dtype)
        if names is not None and k_scales is not None:
            names = tuple(n.replace("_append", "_rowscale_append") if n.endswith("_append")
                          else n + "_rowscale" for n in names)
        self.quantised = None if names is None else tuple(getattr(B, n) for n in names)
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
        with _range("pa.step"):
            return self._step(query, block_tables, context_lens, scale, out, new_key, new_value,
                              slot_mapping, block_mapping, stream, max_context_len, fused_append)

    def _step(self, query, block_tables, context_lens, scale, out, new_key, new_value,
              slot_mapping, block_mapping, stream, max_context_len, fused_append):
        if block_mapping is not None and block_mapping.shape[0] > 0:
            with _range("pa.copy_blocks"):
                B.pa_copy_blocks(self.k_cache, self.v_cache, block_mapping, self.d_status, stream)
        if out is None:
            out = torch.empty_like(query)
        mcl = self.max_context_len if max_context_len is None else max_context_len
        write_needed = slot_mapping is not None and slot_mapping.shape[0] > 0
        if self.quantised is not None and self.k_scales is not None:
            write, decode, decode_append = self.quantised
            ks, vs = self.k_scales, self.v_scales
            if block_mapping is not None and block_mapping.shape[0] > 0:
                with _range("pa.copy_blocks"):
                    B.pa_copy_block_scales(ks, vs, block_mapping, self.d_status, stream)
            if fused_append:
                with _range("pa.decode"):
                    decode_append(out, query, new_key, new_value, self.k_cache, self.v_cache, ks,
                                  vs, block_tables, context_lens, mcl, scale, self.partition_size,
                                  self.workspace, self.d_status, stream)
                return out
            if write_needed:
                with _range("pa.cache_write"):
                    write(new_key, new_value, self.k_cache, self.v_cache, ks, vs, slot_mapping,
                          self.d_status, stream)
            with _range("pa.decode"):
                decode(out, query, self.k_cache, self.v_cache, ks, vs, block_tables, context_lens,
                       mcl, scale, self.partition_size, self.workspace, self.d_status, stream)
            return out
        if self.quantised is not None:
            write, decode, decode_append = self.quantised
            if fused_append:
                with _range("pa.decode"):
                    decode_append(out, query, new_key, new_value, self.k_cache, self.v_cache,
                                  block_tables, context_lens, mcl, scale, self.k_scale,
                                  self.v_scale, self.partition_size, self.workspace,
                                  self.d_status, stream)
                return out
            if write_needed:
                with _range("pa.cache_write"):
                    write(new_key, new_value, self.k_cache, self.v_cache, slot_mapping,
                          self.k_scale, self.v_scale, self.d_status, stream)
            with _range("pa.decode"):
                decode(out, query, self.k_cache, self.v_cache, block_tables, context_lens, mcl,
                       scale, self.k_scale, self.v_scale, self.partition_size, self.workspace,
                       self.d_status, stream)
            return out
        if fused_append:
            with _range("pa.decode"):
                B.pa_paged_decode_append(out, query, new_key, new_value, self.k_cache,
                                         self.v_cache, block_tables, context_lens, mcl, scale,
                                         self.partition_size, self.workspace, self.d_status,
                                         stream)
            return out
        if write_needed:
            with _range("pa.cache_write"):
                B.pa_reshape_and_cache(new_key, new_value, self.k_cache, self.v_cache,
                                       slot_mapping, self.d_status, stream)
        with _range("pa.decode"):
            B.pa_paged_decode(out, query, self.k_cache, self.v_cache, block_tables, context_lens,
                              mcl, scale, self.partition_size, self.workspace, self.d_status,
                              stream)
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

    A step's inputs travel packed: ``host_buffer()`` hands out a pinned byte
    buffer with named views ('query', 'block_tables', ... at 256-byte aligned
    offsets) that the caller fills, and each step uploads it with one copy.
    Three streams: uploads (host -> device), the step's kernels, downloads
    (device -> host).  Device inputs and outputs are double-buffered, so the
    upload of step i+1 runs while step i computes, and the download of step
    i's output runs while step i+1 computes.  Events order each buffer's
    reuse: an upload into set b waits until the step that last read set b has
    finished, the step waits for its upload (and for the download of the
    output it overwrites), a download waits for its step.  Every step still
    copies all of its own inputs in and its output out; only the waiting is
    overlapped.  Kernels of consecutive steps stay in order on the compute
    stream (the cache writes of one step precede the next step's reads).
    With ``use_graphs`` the step's kernels are captured into a CUDA graph per
    buffer set on that set's first use and replayed afterwards.
    """

    def __init__(self, stepper: DecodeStep, dev_like: dict, device=None, use_graphs=False):
        """dev_like: name -> device tensor giving the shape and dtype of each
        input ('query', 'block_tables', 'context_lens' and the optional
        'new_key', 'new_value', 'slot_mapping', 'block_mapping') and 'out'."""
        self.stepper = stepper
        dev = device if device is not None else stepper.k_cache.device
        self.layout = {}
        off = 0
        for name, t in dev_like.items():
            if name == "out":
                continue
            nbytes = t.numel() * t.element_size()
            self.layout[name] = (off, tuple(t.shape), t.dtype, nbytes)
            off = (off + nbytes + 255) // 256 * 256
        self.packed_bytes = max(off, 256)
        self.sets = []
        for _ in range(2):
            buf = torch.empty(self.packed_bytes, dtype=torch.uint8, device=dev)
            views = self._views(buf)
            views["out"] = torch.empty_like(dev_like["out"], device=dev)
            self.sets.append((buf, views))
        self.up = torch.cuda.Stream(dev)
        self.compute = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.uploaded = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.downloaded = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]
        self.i = 0
        self.use_graphs = use_graphs
        self.graphs = {}

    def _views(self, buf: torch.Tensor) -> dict:
        return {name: buf[off:off + nbytes].view(dtype).view(shape)
                for name, (off, shape, dtype, nbytes) in self.layout.items()}

    def host_buffer(self):
        """(pinned byte buffer, {name: view}) in the packed input layout."""
        buf = torch.empty(self.packed_bytes, dtype=torch.uint8).pin_memory()
        return buf, self._views(buf)

    def submit(self, host_packed: torch.Tensor, scale, host_out: torch.Tensor,
               fused_append=False):
        """Enqueue one step: host_packed is a buffer from ``host_buffer()``
        holding this step's inputs, host_out the pinned tensor that receives
        the output.  Returns without waiting; host_out is valid once
        ``synchronize`` returns.  host_packed must not be modified until the
        upload of this step has run."""
        b = self.i % 2
        dev_buf, dev = self.sets[b]
        if self.used[b]:
            self.up.wait_event(self.computed[b])        # the step that last read set b
            self.compute.wait_event(self.downloaded[b])  # its output has left set b's 'out'
        with torch.cuda.stream(self.up), _range("pa.upload"):
            dev_buf.copy_(host_packed, non_blocking=True)
            self.uploaded[b].record(self.up)
        self.compute.wait_event(self.uploaded[b])
        key = (b, float(scale), bool(fused_append))
        graph = self.graphs.get(key)
        step_args = dict(new_key=dev.get("new_key"), new_value=dev.get("new_value"),
                         slot_mapping=dev.get("slot_mapping"),
                         block_mapping=dev.get("block_mapping"), fused_append=fused_append)
        if graph is not None:
            with torch.cuda.stream(self.compute), _range("pa.step"):
                graph.replay()
        else:
            self.stepper(dev["query"], dev["block_tables"], dev["context_lens"], scale,
                         out=dev["out"], stream=self.compute, **step_args)
            if self.use_graphs:
                # capture once the set holds a real step's inputs (the capture
                # re-runs the step eagerly first; a step is idempotent on the
                # same inputs: the same tokens into the same slots)
                self.compute.synchronize()
                self.graphs[key] = self.stepper.graph(dev["query"], dev["block_tables"],
                                                      dev["context_lens"], scale, dev["out"],
                                                      **step_args)
        self.computed[b].record(self.compute)
        self.down.wait_event(self.computed[b])
        with torch.cuda.stream(self.down), _range("pa.download"):
            host_out.copy_(dev["out"], non_blocking=True)
            self.downloaded[b].record(self.down)
        self.used[b] = True
        self.i += 1
        return host_out

    def synchronize(self):
        for st in (self.up, self.compute, self.down):
            st.synchronize()
