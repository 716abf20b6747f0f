"""Helpers of the GPU tests: move seeded workloads to the device, run the
decode step through the C-ABI binding, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from tests.oracle_pins import pool_after_step

TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}
ATOL, RTOL = 2e-3, 1e-2


def to_dev(bits: np.ndarray, dtype: str) -> torch.Tensor:
    """uint16 bit patterns -> device tensor of the element type (no rounding)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(TORCH_DTYPE[dtype])


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class DeviceWorkload:
    def __init__(self, wl):
        self.wl = wl
        d = wl.dtype
        self.query = to_dev(wl.query, d)
        self.k_cache = to_dev(wl.k_cache, d)
        self.v_cache = to_dev(wl.v_cache, d)
        self.block_tables = torch.from_numpy(wl.block_tables).cuda()
        self.context_lens = torch.from_numpy(wl.context_lens).cuda()
        self.new_key = to_dev(wl.new_key, d)
        self.new_value = to_dev(wl.new_value, d)
        self.slot_mapping = torch.from_numpy(wl.slot_mapping).cuda()
        self.block_mapping = torch.from_numpy(np.ascontiguousarray(wl.block_mapping)).cuda()
        self.d_status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(self, partition_size=None, block_tables=None, context_lens=None,
             max_context_len=None, cache_ops=True):
        """K2 -> K1 -> K3 (+K4).  Returns the output tensor."""
        from paged_kv_cache_415_b200 import binding as B
        wl = self.wl
        if cache_ops:
            if wl.block_mapping.shape[0]:
                B.pa_copy_blocks(self.k_cache, self.v_cache, self.block_mapping, self.d_status)
            if wl.num_new_tokens:
                B.pa_reshape_and_cache(self.new_key, self.new_value, self.k_cache, self.v_cache,
                                       self.slot_mapping, self.d_status)
        return self.decode(partition_size, block_tables, context_lens, max_context_len)

    def decode(self, partition_size=None, block_tables=None, context_lens=None,
               max_context_len=None, query=None):
        from paged_kv_cache_415_b200 import binding as B
        wl = self.wl
        p = wl.partition_size if partition_size is None else partition_size
        bt = self.block_tables if block_tables is None else block_tables
        cl = self.context_lens if context_lens is None else context_lens
        mcl = wl.max_context_len if max_context_len is None else max_context_len
        q = self.query if query is None else query
        ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                    wl.head_dim, wl.block_size, mcl, p)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
        out = torch.full_like(q, float("nan"))
        B.pa_paged_decode(out, q, self.k_cache, self.v_cache, bt, cl, mcl, wl.scale, p, ws,
                          self.d_status)
        return out

    def status(self) -> int:
        return int(self.d_status.item())


def oracle_step(wl, num_threads=0):
    """Pools after the step (numpy) and the fp64 oracle output."""
    kc, vc = pool_after_step(wl)
    out, st = oracle.paged_decode(wl.query, kc, vc, wl.block_tables, wl.context_lens, wl.scale,
                                  wl.dtype, num_threads=num_threads)
    return kc, vc, out, st


def assert_close(gpu: np.ndarray, ref: np.ndarray, what=""):
    """|gpu - ref| <= 2e-3 + 1e-2 |ref| elementwise (fp16/bf16 output with fp32
    accumulation against the fp64 oracle)."""
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    err = np.abs(gpu - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; worst at {i}: "
                             f"gpu {gpu[i]!r} ref {ref[i]!r} (max abs err {err.max():.3g})")


def assert_close_rows(gpu: np.ndarray, ref: np.ndarray, what=""):
    """The tolerance of assert_close with its absolute part scaled by each
    output row's magnitude: |gpu - ref| <= 2e-3 * max_d |ref row| + 1e-2 |ref|.

    For data whose kv heads differ in magnitude (row-scaled pools): attention
    is linear in V, so a head whose values are M times unit scale has outputs
    and rounding errors M times larger -- the bf16 output rounding alone is up
    to 2^-8 of a value.  The fixed 2e-3 would be out of reach near the zero
    crossings of a head of magnitude 1e2 and vacuous for a head of magnitude
    1e-2; scaled by the row, every head is held to the same relative
    precision.  A row of zeros (empty context) must come out exactly zero."""
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    scale = np.max(np.abs(ref), axis=-1, keepdims=True)
    err = np.abs(gpu - ref)
    bound = ATOL * scale + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; worst at {i}: "
                             f"gpu {gpu[i]!r} ref {ref[i]!r} row max {scale[i[:-1]][0]!r} "
                             f"(max abs err {err.max():.3g})")
