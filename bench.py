"""Benchmark of one decode step (one layer) over a paged KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is the whole hot path over one batch of synthetic input:
copy_blocks (when the workload has copy-on-write pairs), reshape_and_cache
of the step's new tokens (fused into the decode launch when every sequence
appends one token), paged_decode (plus its split-context reduction).
The default workload is the long-context decode: 16 sequences of 32768
tokens, 32 query / 8 kv heads, head_dim 128, block_size 16, bf16, a fully
shuffled 40000-block pool, 512-token partitions merged by the reduction
kernel, one new token per sequence -- the largest single-GPU workload
(2.15 GB of K/V per step).  In a one-rank run the other workloads
(LLaMA-7B MHA, Mistral-7B GQA, the beam search with shared prompts, and the
one-byte-code pools) are measured after it the same way and reported under
"per_config".

Metric: algorithmic HBM bytes of the step / device time (GB/s), with the
time per step.  The K/V a step reads (1.1 to 2.2 GB) is far larger than the
126 MB L2, so no flush is needed between steps.  For workloads whose
sequences share stored blocks the roofline fraction counts those blocks
once (unique bytes).

--impl reference times the fp64 CPU oracle on the host cores instead (the
only other code path here that runs it), on a bounded sample of the same
workload.

Multi-GPU (torchrun): every rank runs an independent replica of the
workload on its own GPU; nothing is exchanged (the path has no collective).
The time is the max over ranks and the value sums all ranks' bytes.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged-decode attention HBM GB/s (% of B200 peak) and µs per layer-step"
UNIT = "GB/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
PROFILE_GLOB_DIR = os.path.join(ROOT, "profiles")
# The device sources of each decode kernel family: a traffic line taken on a
# family's hash stays valid while those files' code is unchanged.
_CSRC = "paged_kv_cache_415_b200/csrc/"
# Blocks per warp below which the library decodes one-byte pools with a CTA
# per pair of kv heads (kPairBelowBlocks in csrc/paged_decode.cu).
PAIR_BELOW_BLOCKS = 16

KERNEL_FAMILIES = {
    "fp32": ["pa_common.cuh", "decode_common.cuh", "paged_decode_fp32.cuh"],
    "mma": ["pa_common.cuh", "decode_common.cuh", "paged_decode_mma.cuh"],
    "q8": ["pa_common.cuh", "decode_common.cuh", "pa_codes.cuh", "paged_decode_q8.cuh",
           "paged_decode_q8_pair.cuh"],
    "shared": ["pa_common.cuh", "decode_common.cuh", "paged_decode_mma.cuh",
               "paged_decode_shared.cuh"],
}
NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                0x100: "display_clock_setting"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="long_context",
                    choices=["tiny", "llama7b", "mistral7b", "beam_search", "long_context"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads measured after the headline in a one-rank run")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--partition", type=int, default=-1,
                    help="context partition in tokens (-1 = the workload's, 0 = library's choice)")
    ap.add_argument("--separate", action="store_true",
                    help="run the cache write and the decode as separate calls even when every "
                         "sequence appends one token (default: pa_paged_decode_append)")
    ap.add_argument("--shared-prefix", action="store_true",
                    help="beam_search: decode with pa_paged_decode_shared_prefix (shared "
                         "prompt blocks read once per group)")
    ap.add_argument("--kv-dtype", default="auto",
                    choices=["auto", "fp8", "int8", "fp8-rows", "int8-rows"],
                    help="fp8 / int8: the same workload with e4m3 / int8 K/V pools (per-pool "
                         "scales), quantising cache write + decode over the codes; -rows: one "
                         "fp32 scale per (token, kv head) row instead")
    ap.add_argument("--swap", choices=["out", "in"], default=None,
                    help="measure pa_swap_blocks instead of the decode step: 512 LLaMA-7B-shaped "
                         "blocks (K and V, 256 KB a pair) device -> pinned host (out) or back (in)")
    ap.add_argument("--eager", action="store_true",
                    help="issue every launch from the host in the timed region (default: the "
                         "step's cache operations and its decode are captured into two CUDA "
                         "graphs once and replayed)")
    ap.add_argument("--seqs", type=int, default=0,
                    help="shrink the batch (and the pool) for profiling; 0 = the full workload")
    return ap.parse_args()


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def strip_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines (string and
    character literals kept), so that an edit of comments alone leaves
    kernel_source_hash unchanged."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":                               # a literal: copy through its end
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            end = src.find("*/", i + 2)
            i = n if end < 0 else end + 2
        else:
            out.append(c)
            i += 1
    lines = ("".join(out)).split("\n")
    return "\n".join(line.rstrip() for line in lines if line.strip())


def kernel_source_hash(family: str) -> str:
    """sha256[:16] of a decode kernel family's device sources, comments and
    blank lines removed: a profile taken on a hash still describes the
    current code of that family."""
    h = hashlib.sha256()
    for name in KERNEL_FAMILIES[family]:
        with open(os.path.join(ROOT, _CSRC + name), encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, family: str):
    """DRAM bytes per launch of the decode kernels from a committed ncu
    summary, if it was taken on the current sources of their family."""
    want = kernel_source_hash(family)
    if not os.path.isdir(PROFILE_GLOB_DIR):
        return None
    for name in sorted(os.listdir(PROFILE_GLOB_DIR)):
        if not name.endswith((".md", ".txt")):
            continue
        with open(os.path.join(PROFILE_GLOB_DIR, name)) as f:
            for line in f:
                m = re.search(r"bench-traffic:\s*workload=(\S+)\s+bytes_per_launch=(\d+)\s+"
                              r"source_sha256=(\w+)", line)
                if m and m.group(1) == workload and m.group(3) == want:
                    return int(m.group(2))
    return None


class ClockSampler:
    """Polls NVML (SM clock, clock-event reasons) in a thread while the
    timed region runs."""

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            handle = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                handle = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:   # noqa: BLE001
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h, self.nv = handle, pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:       # noqa: BLE001
            self.ok = False

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while True:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception:   # noqa: BLE001
                pass
            if self._stop.wait(0.001):
                break

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml unavailable"}
        names = [n for bit, n in NVML_REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "source": "nvml"}


def max_over_ranks(values, device=None):
    """Elementwise max of per-rank floats over the process group (identity
    without one).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_gbs(bytes_per_step: int, steps: int, world: int, max_elapsed_ms: float) -> float:
    """Every rank runs its own replica: total bytes over the slowest rank's time."""
    return world * bytes_per_step * steps / (max_elapsed_ms * 1e-3) / 1e9


_BASE = {}            # the last 16-bit workload made, reused by its code-pool variants


def make_workload(config: str, seqs: int = 0, kv_dtype: str = "auto"):
    """The named workload; with seqs > 0 a smaller batch of the same shape
    and a pool sized to it (profiling captures stay a few GB); kv_dtype fp8
    or int8 redraws its pools as e4m3 or int8 codes (one scale per pool),
    fp8-rows / int8-rows as codes with one scale per (token, kv head) row."""
    from workloads import generators as gen
    key = (config, seqs)
    if key not in _BASE:
        _BASE.clear()
        _BASE[key] = _make_workload(config, seqs)
    wl = _BASE[key]
    if kv_dtype in ("fp8", "int8"):
        wl = gen.with_code_pools(wl, kv_dtype, seed=gen.SEED_BASE + 50)
    elif kv_dtype in ("fp8-rows", "int8-rows"):
        wl = gen.with_rowscale_pools(wl, kv_dtype[:-5], seed=gen.SEED_BASE + 50)
    return wl


def _make_workload(config: str, seqs: int = 0):
    from workloads import generators as gen
    if seqs <= 0:
        return gen.CONFIGS[config]()
    if config == "llama7b":
        return gen.llama7b(seqs=seqs, num_blocks=seqs * 130 + 64)
    if config == "mistral7b":
        return gen.mistral7b(seqs=seqs, num_blocks=seqs * 520 + 64)
    if config == "long_context":
        return gen.long_context(seqs=seqs, num_blocks=seqs * 2048 + 64)
    if config == "beam_search":
        return gen.beam_search(prompts=max(1, seqs // 4))
    return gen.CONFIGS[config]()


def workload_config(wl, partition_size, l2_note):
    kv = {"fp8": ", e4m3 K/V pools", "int8": ", int8 K/V pools"}.get(wl.extra.get("kv_dtype"), "")
    if kv and wl.extra.get("rowscale"):
        kv += " with one scale per (token, kv head) row"
    return {"workload": f"{wl.name}: {wl.num_seqs} seqs, {wl.num_q_heads}/{wl.num_kv_heads} heads, "
                        f"head_dim {wl.head_dim}, block {wl.block_size}, {wl.dtype}{kv}, "
                        f"contexts {int(wl.context_lens.min())}..{int(wl.context_lens.max())} "
                        f"(sum {int(wl.context_lens.sum())}), pool {wl.num_blocks} blocks, "
                        f"{wl.num_new_tokens} new tokens, {int(wl.block_mapping.shape[0])} block copies",
            "num_seqs": wl.num_seqs, "num_q_heads": wl.num_q_heads,
            "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
            "block_size": wl.block_size, "partition_size": partition_size,
            "layers": 1, "l2": l2_note}


# ---------------------------------------------------------------------------
# CPU oracle timing (the cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

class OracleStep:
    """The oracle's whole step (block copies, cache write, fp64 decode of the
    first ``max_seqs`` sequences) on host copies of the workload."""

    def __init__(self, wl, max_seqs=None):
        import oracle
        from workloads import byte_model as bm
        self.oracle, self.wl = oracle, wl
        n = wl.num_seqs if max_seqs is None else max(1, min(max_seqs, wl.num_seqs))
        self.n = n
        self.ctx = np.ascontiguousarray(wl.context_lens[:n])
        self.tables = np.ascontiguousarray(wl.block_tables[:n])
        self.q = np.ascontiguousarray(wl.query[:n])
        self.kc, self.vc = wl.k_cache.copy(), wl.v_cache.copy()
        att = bm.decode_bytes(self.ctx, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                              wl.block_size, 2, bm.kv_elem_bytes(wl), bm.row_scale_bytes(wl))
        self.codes = wl.extra.get("kv_dtype")          # None, "fp8" or "int8"
        self.rows = bool(wl.extra.get("rowscale"))
        if self.rows:
            self.ks, self.vs = wl.extra["k_scales"].copy(), wl.extra["v_scales"].copy()
        full = bm.step_bytes(wl)
        self.bytes = att["total"] + full["append"] + full["copy"]
        self.threads = oracle.max_threads()

    def run(self) -> float:
        o, wl = self.oracle, self.wl
        t0 = time.perf_counter()
        if wl.block_mapping.shape[0]:
            o.copy_blocks(self.kc, self.vc, wl.block_mapping)
            if self.rows:
                o.copy_blocks(self.ks, self.vs, wl.block_mapping)
        if self.rows:
            write = getattr(o, f"reshape_and_cache_{self.codes}_rowscale")
            decode = getattr(o, f"paged_decode_{self.codes}_rowscale")
            if wl.num_new_tokens:
                write(wl.new_key, wl.new_value, self.kc, self.vc, self.ks, self.vs,
                      wl.slot_mapping, wl.block_size, wl.dtype)
            decode(self.q, self.kc, self.vc, self.ks, self.vs, self.tables, self.ctx, wl.scale,
                   wl.dtype)
            return time.perf_counter() - t0
        if self.codes is not None:
            ks, vs = wl.extra["k_scale"], wl.extra["v_scale"]
            write = getattr(o, f"reshape_and_cache_{self.codes}")
            decode = getattr(o, f"paged_decode_{self.codes}")
            if wl.num_new_tokens:
                write(wl.new_key, wl.new_value, self.kc, self.vc, wl.slot_mapping, wl.block_size,
                      wl.dtype, ks, vs)
            decode(self.q, self.kc, self.vc, self.tables, self.ctx, wl.scale, wl.dtype, ks, vs)
            return time.perf_counter() - t0
        if wl.num_new_tokens:
            o.reshape_and_cache(wl.new_key, wl.new_value, self.kc, self.vc, wl.slot_mapping,
                                wl.block_size)
        o.paged_decode(self.q, self.kc, self.vc, self.tables, self.ctx, wl.scale, wl.dtype)
        return time.perf_counter() - t0

    def describe(self) -> str:
        wl = self.wl
        return (f"{wl.name}: one full step (block copies, all {wl.num_new_tokens} new tokens, "
                f"fp64 decode of {self.n} of {wl.num_seqs} sequences)")


def oracle_sample_time(wl, seconds: float):
    """Repeat the oracle's full step until ``seconds`` have passed (at least
    once).  Returns (GB/s, seconds per step, sample description, threads)."""
    st = OracleStep(wl)
    reps, total = 0, 0.0
    while reps == 0 or total < seconds:
        total += st.run()
        reps += 1
    per = total / reps
    return st.bytes / per / 1e9, per, f"{st.describe()}, repeated {reps}x in {total:.1f}s", st.threads


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = make_workload(args.config, args.seqs, args.kv_dtype)
    # size the per-step sample so warm-up + timed steps end within ~2 minutes
    probe = OracleStep(wl, max_seqs=max(1, wl.num_seqs // 8))
    per_seq = probe.run() / probe.n
    del probe
    budget = 120.0 / max(1, args.steps + args.warmup)
    st = OracleStep(wl, max_seqs=int(max(1, min(wl.num_seqs, budget / max(per_seq, 1e-9)))))
    for _ in range(args.warmup):
        st.run()
    times = [st.run() for _ in range(args.steps)]
    per_step = statistics.mean(times)
    value = st.bytes / per_step / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(per_step * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, None, "host memory"),
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": st.threads,
                             "kind": "oracle", "sample": st.describe() + " per step"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

# Workloads measured in the same run as the headline, each on its own
# (name, K/V code format, shared-prefix decode), when the run has one rank.
# Variants of one base workload follow each other, so it is drawn once.
PER_CONFIG = [("long_context", "fp8", False), ("long_context", "int8", False),
              ("long_context", "fp8-rows", False), ("long_context", "int8-rows", False),
              ("llama7b", "auto", False), ("mistral7b", "auto", False),
              ("mistral7b", "fp8", False), ("mistral7b", "int8", False),
              ("beam_search", "auto", True)]


class GpuStep:
    """One workload resident on the device and its step: the copy-on-write
    copies, the cache write (fused into the decode launch when every
    sequence appends one token), the decode and its split-context
    reduction, all through the C-ABI binding; captured into two CUDA graphs
    (cache operations, decode) unless eager."""

    def __init__(self, wl, dev, partition=-1, separate=False, shared_prefix=False):
        import torch
        from paged_kv_cache_415_b200 import binding as B
        self.B, self.torch, self.wl, self.dev = B, torch, wl, dev
        self.tdt = {"f16": torch.float16, "bf16": torch.bfloat16}[wl.dtype]
        self.codes = wl.extra.get("kv_dtype")                  # None, "fp8" or "int8"
        self.quant = self.codes is not None
        self.rows = bool(wl.extra.get("rowscale"))             # one scale per row
        self.k_scale = wl.extra.get("k_scale", 1.0)
        self.v_scale = wl.extra.get("v_scale", 1.0)
        if self.quant:
            self.k_cache = torch.from_numpy(wl.k_cache).to(dev)
            self.v_cache = torch.from_numpy(wl.v_cache).to(dev)
        else:
            self.k_cache, self.v_cache = self.up(wl.k_cache), self.up(wl.v_cache)
        if self.rows:
            self.k_scales = torch.from_numpy(wl.extra["k_scales"]).to(dev)
            self.v_scales = torch.from_numpy(wl.extra["v_scales"]).to(dev)
        self.query = self.up(wl.query)
        self.new_key, self.new_value = self.up(wl.new_key), self.up(wl.new_value)
        self.slot_mapping = torch.from_numpy(wl.slot_mapping).to(dev)
        self.block_tables = torch.from_numpy(wl.block_tables).to(dev)
        self.context_lens = torch.from_numpy(wl.context_lens).to(dev)
        self.block_mapping = torch.from_numpy(np.ascontiguousarray(wl.block_mapping)).to(dev)
        self.out = torch.empty_like(self.query)
        self.d_status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.mcl = wl.max_context_len
        want = wl.partition_size if partition < 0 else partition
        self.part = B.pa_paged_decode_partition_size(wl.num_seqs, wl.num_q_heads,
                                                     wl.num_kv_heads, wl.head_dim,
                                                     wl.block_size, self.mcl, want)
        ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                    wl.head_dim, wl.block_size, self.mcl,
                                                    self.part)
        self.max_parts = -(-self.mcl // self.part) if self.mcl > 0 else 1
        self.n_pairs = int(wl.block_mapping.shape[0])
        self.fused = (not separate and not shared_prefix
                      and wl.extra.get("one_token_per_seq", False)
                      and wl.num_new_tokens == wl.num_seqs)
        self.shared = shared_prefix and "prefix_lens" in wl.extra and not self.quant
        self.shared_reduce = False
        if self.shared:
            self.group_size = int(wl.extra["group_size"])
            self.prefix_lens = torch.from_numpy(wl.extra["prefix_lens"]).to(dev)
            self.mpl = int(wl.extra["prefix_lens"].max())
            ws_bytes = B.pa_paged_decode_shared_prefix_workspace_size(
                wl.num_seqs, self.group_size, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                wl.block_size, self.mcl, self.mpl, 0)
            self.shared_reduce = ws_bytes > 0
        self.workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.has_cache = bool(self.n_pairs or (wl.num_new_tokens and not self.fused))
        self.run_cache, self.run_decode = self.cache_ops, self.decode

    def up(self, bits):
        return self.torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(self.dev).view(
            self.tdt)

    def cache_ops(self):
        B, wl = self.B, self.wl
        if self.n_pairs:
            B.pa_copy_blocks(self.k_cache, self.v_cache, self.block_mapping, self.d_status,
                             self.stream)
            if self.rows:
                B.pa_copy_block_scales(self.k_scales, self.v_scales, self.block_mapping,
                                       self.d_status, self.stream)
        if wl.num_new_tokens and not self.fused:
            if self.rows:
                getattr(B, f"pa_reshape_and_cache_{self.codes}_rowscale")(
                    self.new_key, self.new_value, self.k_cache, self.v_cache, self.k_scales,
                    self.v_scales, self.slot_mapping, self.d_status, self.stream)
            elif self.quant:
                getattr(B, f"pa_reshape_and_cache_{self.codes}")(
                    self.new_key, self.new_value, self.k_cache, self.v_cache, self.slot_mapping,
                    self.k_scale, self.v_scale, self.d_status, self.stream)
            else:
                B.pa_reshape_and_cache(self.new_key, self.new_value, self.k_cache, self.v_cache,
                                       self.slot_mapping, self.d_status, self.stream)

    def decode(self):
        B, wl = self.B, self.wl
        if self.rows and self.fused:
            getattr(B, f"pa_paged_decode_{self.codes}_rowscale_append")(
                self.out, self.query, self.new_key, self.new_value, self.k_cache, self.v_cache,
                self.k_scales, self.v_scales, self.block_tables, self.context_lens, self.mcl,
                wl.scale, self.part, self.workspace, self.d_status, self.stream)
        elif self.rows:
            getattr(B, f"pa_paged_decode_{self.codes}_rowscale")(
                self.out, self.query, self.k_cache, self.v_cache, self.k_scales, self.v_scales,
                self.block_tables, self.context_lens, self.mcl, wl.scale, self.part,
                self.workspace, self.d_status, self.stream)
        elif self.quant and self.fused:
            getattr(B, f"pa_paged_decode_{self.codes}_append")(
                self.out, self.query, self.new_key, self.new_value, self.k_cache, self.v_cache,
                self.block_tables, self.context_lens, self.mcl, wl.scale, self.k_scale,
                self.v_scale, self.part, self.workspace, self.d_status, self.stream)
        elif self.quant:
            getattr(B, f"pa_paged_decode_{self.codes}")(
                self.out, self.query, self.k_cache, self.v_cache, self.block_tables,
                self.context_lens, self.mcl, wl.scale, self.k_scale, self.v_scale, self.part,
                self.workspace, self.d_status, self.stream)
        elif self.fused:
            B.pa_paged_decode_append(self.out, self.query, self.new_key, self.new_value,
                                     self.k_cache, self.v_cache, self.block_tables,
                                     self.context_lens, self.mcl, wl.scale, self.part,
                                     self.workspace, self.d_status, self.stream)
        elif self.shared:
            B.pa_paged_decode_shared_prefix(self.out, self.query, self.k_cache, self.v_cache,
                                            self.block_tables, self.context_lens,
                                            self.prefix_lens, self.group_size, self.mcl,
                                            self.mpl, wl.scale, self.workspace, 0, self.d_status,
                                            self.stream)
        else:
            B.pa_paged_decode(self.out, self.query, self.k_cache, self.v_cache,
                              self.block_tables, self.context_lens, self.mcl, wl.scale,
                              self.part, self.workspace, self.d_status, self.stream)

    @property
    def launches_per_step(self) -> int:
        wl = self.wl
        reduce = self.shared_reduce if self.shared else self.max_parts > 1
        copies = (2 if self.rows else 1) if self.n_pairs else 0
        return (copies + (1 if (wl.num_new_tokens and not self.fused) else 0)
                + 1 + (1 if reduce else 0))

    def prepare(self, warmup: int, eager: bool, barrier):
        """Warm-up steps, then (unless eager) the step captured once into two
        graphs whose replay issues the launches with no host work; checks
        the status word and that the output is finite."""
        torch = self.torch
        for _ in range(warmup):
            self.cache_ops()
            self.decode()
        barrier()
        if not eager:
            g_cache, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            saved = self.stream
            with torch.cuda.graph(g_dec):
                self.stream = torch.cuda.current_stream(self.dev)
                self.decode()
            if self.has_cache:
                with torch.cuda.graph(g_cache):
                    self.stream = torch.cuda.current_stream(self.dev)
                    self.cache_ops()
            self.stream = saved
            self.graphs = (g_cache, g_dec)
            self.run_cache = g_cache.replay if self.has_cache else (lambda: None)
            self.run_decode = g_dec.replay
            self.run_cache()
            self.run_decode()
            barrier()
        st = int(self.d_status.item())
        if st != 0 or not bool(torch.isfinite(self.out.float()).all()):
            raise SystemExit(f"{self.wl.name}: bad step (status {st})")

    def timed(self, steps: int):
        """K steps between two events on the launching stream; events also
        bracket the decode launches of every step.  Returns (elapsed ms,
        per-step decode ms)."""
        torch = self.torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(self.stream)
        for i in range(steps):
            self.run_cache()
            ev[i][0].record(self.stream)
            self.run_decode()
            ev[i][1].record(self.stream)
        stop.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return start.elapsed_time(stop), [a.elapsed_time(b) for a, b in ev]

    def kernel_name(self) -> str:
        wl = self.wl
        group = wl.num_q_heads // wl.num_kv_heads
        if self.shared:
            return "paged_decode_shared_kernel" + (
                " + paged_decode_shared_reduce_kernel" if self.shared_reduce else "")
        # one-byte pools: a CTA per pair of kv heads when the kv-head count is
        # even and a CTA per kv head (4 warps) would give each warp fewer than
        # PAIR_BELOW_BLOCKS blocks of its partition (the library's rule)
        pair = (wl.num_kv_heads % 2 == 0 and self.part < PAIR_BELOW_BLOCKS * 4 * wl.block_size)
        name = (f"paged_decode_{self.codes}{'_pair' if pair else ''}_kernel" if self.quant else
                "paged_decode_mma_kernel" if group >= 4 and wl.block_size % 16 == 0
                else "paged_decode_kernel")
        return name + (" + paged_decode_reduce_kernel" if self.max_parts > 1 else "")

    def entry(self) -> str:
        c = self.codes
        if self.rows:
            return (f"pa_paged_decode_{c}_rowscale_append (row-scaled quantising write fused)"
                    if self.fused else
                    f"pa_reshape_and_cache_{c}_rowscale + pa_paged_decode_{c}_rowscale")
        return (f"pa_paged_decode_{c}_append (quantising cache write fused)" if self.quant and self.fused
                else f"pa_reshape_and_cache_{c} + pa_paged_decode_{c}" if self.quant
                else "pa_paged_decode_shared_prefix" if self.shared
                else "pa_paged_decode_append (cache write fused)" if self.fused
                else "pa_reshape_and_cache + pa_paged_decode")

    def roofline_bytes(self):
        """(algorithmic bytes of one decode launch, referenced bytes or None).
        A sharing workload (beams over one stored prompt) counts its K/V on
        unique bytes -- the blocks the step must read at least once -- and
        reports the bytes its block tables reference beside them."""
        from workloads import byte_model as bm
        step = bm.step_bytes(self.wl)
        referenced = step["attention"] + (step["append"] if self.fused else 0)
        if "prefix_lens" not in self.wl.extra:
            return referenced, None
        unique = referenced - step["kv"] + bm.unique_kv_bytes(self.wl)
        return unique, referenced

    def free(self):
        for name in ("k_cache", "v_cache", "k_scales", "v_scales", "query", "new_key",
                     "new_value", "out", "workspace",
                     "graphs", "block_tables", "context_lens", "slot_mapping", "block_mapping"):
            if hasattr(self, name):
                delattr(self, name)
        self.run_cache = self.run_decode = None
        self.torch.cuda.empty_cache()


def measure_per_config(name, kv_dtype, shared, args, dev, barrier, peak):
    """One more workload in the same run: its step timed as the headline's
    (graph replay, events on the launching stream), reported per layer-step
    with the decode launches' roofline fraction."""
    wl = make_workload(name, 0, kv_dtype)
    g = GpuStep(wl, dev, shared_prefix=shared)
    g.prepare(args.warmup, args.eager, barrier)
    sampler = ClockSampler(dev.index or 0)
    barrier()
    with sampler:
        elapsed_ms, decode_ms = g.timed(args.steps)
    decode_avg = statistics.mean(decode_ms)
    dbytes, referenced = g.roofline_bytes()
    achieved = dbytes / (decode_avg * 1e-3) / 1e9
    label = name + (f"-{kv_dtype}" if kv_dtype != "auto" else "")   # e.g. mistral7b-int8-rows
    entry = {"workload": workload_config(wl, g.part, "")["workload"],
             "us_per_layer_step": round(elapsed_ms / args.steps * 1e3, 2),
             "kernel": g.kernel_name(), "decode_entry": g.entry(),
             "avg_launch_us": round(decode_avg * 1e3, 2),
             "algorithmic_bytes_per_launch": dbytes, "achieved": round(achieved, 1),
             "frac": round(achieved / peak, 4),
             "traffic": profiled_traffic(label + ("-shared" if g.shared else ""),
                                         kernel_family(g)),
             "sm_mhz": sampler.summary()["sm_mhz"]}
    if referenced is not None:
        entry["frac_on"] = "unique K/V bytes (shared blocks counted once)"
        entry["referenced_bytes_per_launch"] = referenced
    g.free()
    del wl
    return label + ("-shared" if g.shared else ""), entry


def kernel_family(g) -> str:
    """The decode kernel family whose sources a traffic line depends on."""
    if g.shared:
        return "shared"
    if g.quant:
        return "q8"
    group = g.wl.num_q_heads // g.wl.num_kv_heads
    return "mma" if group >= 4 and g.wl.block_size % 16 == 0 else "fp32"


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    from workloads import byte_model as bm

    dev = torch.device("cuda", local)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    wl = make_workload(args.config, args.seqs, args.kv_dtype)
    g = GpuStep(wl, dev, args.partition, args.separate, args.shared_prefix)
    g.prepare(args.warmup, args.eager, barrier)

    # timed region: K steps
    sampler = ClockSampler(local)
    barrier()
    with sampler:
        elapsed_ms, decode_ms = g.timed(args.steps)
    barrier()

    # end to end through the public API: pinned host inputs -> device -> step -> host output
    from paged_kv_cache_415_b200.step import DecodeStep, HostPipeline
    tdt, fused = g.tdt, g.fused
    stepper = DecodeStep(g.k_cache, g.v_cache, wl.num_seqs, wl.num_q_heads, g.mcl, g.part,
                         g.k_scale, g.v_scale, getattr(g, "k_scales", None),
                         getattr(g, "v_scales", None))
    host = {"query": torch.from_numpy(wl.query.view(np.int16)).view(tdt).pin_memory(),
            "block_tables": torch.from_numpy(wl.block_tables).pin_memory(),
            "context_lens": torch.from_numpy(wl.context_lens).pin_memory(),
            "out": torch.empty(g.out.shape, dtype=tdt).pin_memory()}
    devb = {"query": torch.empty_like(g.query), "block_tables": torch.empty_like(g.block_tables),
            "context_lens": torch.empty_like(g.context_lens), "out": torch.empty_like(g.out)}
    if wl.num_new_tokens:
        host["new_key"] = torch.from_numpy(wl.new_key.view(np.int16)).view(tdt).pin_memory()
        host["new_value"] = torch.from_numpy(wl.new_value.view(np.int16)).view(tdt).pin_memory()
        names = ("new_key", "new_value")
        if not fused:
            host["slot_mapping"] = torch.from_numpy(wl.slot_mapping).pin_memory()
            names += ("slot_mapping",)
        for k in names:
            devb[k] = torch.empty_like(host[k], device=dev)
    if g.n_pairs:
        host["block_mapping"] = torch.from_numpy(np.ascontiguousarray(wl.block_mapping)).pin_memory()
        devb["block_mapping"] = torch.empty_like(host["block_mapping"], device=dev)
    h2d = sum(t.numel() * t.element_size() for k, t in host.items() if k != "out")
    d2h = host["out"].numel() * host["out"].element_size()
    host_out = host.pop("out")
    pipe = HostPipeline(stepper, devb, dev)
    packed, views = pipe.host_buffer()
    for name, t in host.items():
        views[name].copy_(t)
    for _ in range(max(3, args.warmup)):
        pipe.submit(packed, wl.scale, host_out, fused_append=fused)
    pipe.synchronize()
    barrier()
    e_sampler = ClockSampler(local)
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with e_sampler:
        e_start.record(pipe.up)
        for _ in range(args.steps):
            pipe.submit(packed, wl.scale, host_out, fused_append=fused)
        e_stop.record(pipe.down)
        pipe.synchronize()
        torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = e_start.elapsed_time(e_stop)

    elapsed_ms, e2e_ms, decode_avg = max_over_ranks(
        [elapsed_ms, e2e_ms, statistics.mean(decode_ms)], dev)

    step = bm.step_bytes(wl)
    per_step_ms = elapsed_ms / args.steps
    value = whole_job_gbs(step["total"], args.steps, world, elapsed_ms)
    e2e_value = whole_job_gbs(step["total"], args.steps, world, e2e_ms)
    peak, peak_kind = hbm_peak()
    decode_bytes, referenced = g.roofline_bytes()
    achieved = decode_bytes / (decode_avg * 1e-3) / 1e9
    label = (args.config + (f"-{g.codes}" if g.quant else "") + ("-rows" if g.rows else "")
             + ("-shared" if g.shared else ""))
    traffic = profiled_traffic(label, kernel_family(g)) if args.seqs <= 0 else None
    clocks = sampler.summary()
    clocks = merge_clocks(clocks, e_sampler.summary())
    kernel_name, entry, launches_per_step = g.kernel_name(), g.entry(), g.launches_per_step
    config_block = workload_config(wl, g.part, "")
    del stepper, pipe, devb, host, host_out, packed, views
    g.free()

    per_config = {}
    if world == 1 and not args.no_per_config and args.seqs <= 0:
        for name, kv, shared in PER_CONFIG:
            if name == args.config and kv == args.kv_dtype and shared == args.shared_prefix:
                continue
            key, entry_i = measure_per_config(name, kv, shared, args, dev, barrier, peak)
            per_config[key] = entry_i

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gb, _, desc, threads = oracle_sample_time(wl, args.cpu_seconds)
        cpu = {"value": round(gb, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    l2 = (f"no flush: {step['kv'] / 1e9:.2f} GB of K/V per step > 126 MB L2"
          if step["kv"] > 4 * 126e6 else "working set smaller than L2 (values include L2 hits)")
    config_block["l2"] = l2
    roof = {"bound": "hbm", "kernel": kernel_name,
            "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "traffic": traffic, "algorithmic_bytes_per_launch": decode_bytes,
            "avg_launch_us": round(decode_avg * 1e3, 2)}
    if referenced is not None:
        roof["frac_on"] = "unique K/V bytes (shared blocks counted once)"
        roof["referenced_bytes_per_launch"] = referenced
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ({"fp8": "f16 (e4m3 K/V)", "int8": "f16 (int8 K/V)"}[g.codes]
                  + (", row scales" if g.rows else "") if g.quant else wl.dtype),
        "data": "synthetic", "config": config_block,
        "us_per_layer_step": round(per_step_ms * 1e3, 2),
        "kv_tokens_per_s": round(world * int(wl.context_lens.sum()) * args.steps / (elapsed_ms * 1e-3)),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / args.steps, 5),
                "api": "step.HostPipeline: per step, the packed pinned inputs uploaded in one "
                       "copy on one stream, the step's kernels on another, the output "
                       "downloaded on a third; double-buffered so copies overlap the "
                       "neighbouring steps' kernels"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "bytes_per_step": step,
        "launch": "eager" if args.eager else "CUDA-graph replay (cache ops graph, decode graph)",
        "decode_entry": entry,
    }
    if per_config:
        line["per_config"] = per_config
    print(json.dumps(line))
    return 0


def merge_clocks(a: dict, b: dict) -> dict:
    """Clock records of the timed region and of the end-to-end loop as one:
    the median of both regions' samples is not kept per sample, so the
    record keeps the lower median, the union of reasons and the sample
    counts of both."""
    if not b.get("samples"):
        return a
    if not a.get("samples"):
        return dict(b, regions="e2e loop")
    return {"sm_mhz": min(a["sm_mhz"], b["sm_mhz"]), "sm_max_mhz": a["sm_max_mhz"] or b["sm_max_mhz"],
            "reasons": sorted(set(a["reasons"]) | set(b["reasons"])),
            "samples": a["samples"] + b["samples"], "source": a["source"],
            "regions": "timed region and e2e loop"}


# ---------------------------------------------------------------------------
# Swap of blocks over the host link (pa_swap_blocks)
# ---------------------------------------------------------------------------

SWAP_SHAPE = (16, 32, 128)          # LLaMA-7B block: 16 tokens x 32 heads x 128, fp16
SWAP_DEVICE_BLOCKS, SWAP_HOST_BLOCKS, SWAP_PAIRS = 4096, 1024, 512


def run_swap(args):
    """One step = one pa_swap_blocks call moving SWAP_PAIRS scattered blocks
    (K and V) between a device pool and a pinned host pool.  The roofline
    peak is the copy engine's own rate for the same byte count as one
    contiguous pinned copy in the same direction, measured here."""
    import torch
    from paged_kv_cache_415_b200 import binding as B
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rng = np.random.Generator(np.random.PCG64(4150 + 60))
    dk = torch.randint(-32768, 32767, (SWAP_DEVICE_BLOCKS,) + SWAP_SHAPE, dtype=torch.int16,
                       device=dev).view(torch.float16)
    dv = torch.randint(-32768, 32767, (SWAP_DEVICE_BLOCKS,) + SWAP_SHAPE, dtype=torch.int16,
                       device=dev).view(torch.float16)
    hk = torch.zeros((SWAP_HOST_BLOCKS,) + SWAP_SHAPE, dtype=torch.float16).pin_memory()
    hv = torch.zeros((SWAP_HOST_BLOCKS,) + SWAP_SHAPE, dtype=torch.float16).pin_memory()
    pairs = np.stack([rng.permutation(SWAP_DEVICE_BLOCKS)[:SWAP_PAIRS],
                      rng.permutation(SWAP_HOST_BLOCKS)[:SWAP_PAIRS]], 1).astype(np.int64)
    if args.swap == "in":
        pairs = pairs[:, ::-1].copy()
        src, dst = (hk, hv), (dk, dv)
    else:
        src, dst = (dk, dv), (hk, hv)
    mapping = torch.from_numpy(pairs).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    block_bytes = int(np.prod(SWAP_SHAPE)) * 2
    moved = SWAP_PAIRS * block_bytes * 2

    def step():
        B.pa_swap_blocks(src[0], src[1], dst[0], dst[1], mapping, status, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise SystemExit(f"swap status {int(status.item())}")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize(dev)
    ms = start.elapsed_time(stop) / args.steps
    # the copy engine on one contiguous buffer of the same size and direction
    hbuf = torch.empty(moved // 2, dtype=torch.int16).pin_memory()
    dbuf = torch.empty(moved // 2, dtype=torch.int16, device=dev)
    a, b = (dbuf, hbuf) if args.swap == "in" else (hbuf, dbuf)
    for _ in range(3):
        a.copy_(b, non_blocking=True)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(args.steps):
        a.copy_(b, non_blocking=True)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    dma_ms = start.elapsed_time(stop) / args.steps
    value = moved / (ms * 1e-3) / 1e9
    peak = moved / (dma_ms * 1e-3) / 1e9
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        host_src = [np.zeros((SWAP_PAIRS,) + SWAP_SHAPE, np.uint16) for _ in range(2)]
        host_dst = [np.zeros((SWAP_PAIRS,) + SWAP_SHAPE, np.uint16) for _ in range(2)]
        local_map = np.stack([np.arange(SWAP_PAIRS), rng.permutation(SWAP_PAIRS)], 1)
        t0 = time.perf_counter()
        reps = 0
        while reps == 0 or time.perf_counter() - t0 < min(args.cpu_seconds, 5.0):
            oracle.swap_blocks(host_src[0], host_src[1], host_dst[0], host_dst[1], local_map)
            reps += 1
        per = (time.perf_counter() - t0) / reps
        cpu = {"value": round(moved / per / 1e9, 3), "unit": "GB/s", "cores": 1,
               "kind": "oracle",
               "sample": f"oracle swap of the same {SWAP_PAIRS} block pairs between host arrays, "
                         f"repeated {reps}x"}
    if rank != 0:
        return 0
    line = {
        "metric": f"swap_blocks GB/s over the host link ({args.swap})", "value": round(value, 2),
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 (bit copy)", "data": "synthetic",
        "config": {"workload": f"swap {args.swap}: {SWAP_PAIRS} scattered LLaMA-7B blocks "
                               f"(16 x 32 x 128 fp16, K and V) between a {SWAP_DEVICE_BLOCKS}-block "
                               f"device pool and a {SWAP_HOST_BLOCKS}-block pinned host pool",
                   "bytes_per_step": moved, "l2": "host pool in pinned memory; no flush"},
        "roofline": {"bound": "link", "kernel": "swap_blocks_kernel", "achieved": round(value, 1),
                     "peak": round(peak, 1),
                     "peak_kind": "measured here: copy engine, one contiguous pinned copy",
                     "unit": "GB/s", "frac": round(value / peak, 4), "traffic": None},
        "e2e": {"value": round(value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": moved if args.swap == "in" else 0,
                "d2h_bytes_per_step": moved if args.swap == "out" else 0},
        "gpu_launches": args.steps, "clocks": sampler.summary(), "cpu_baseline": cpu,
        "decode_entry": "pa_swap_blocks",
    }
    print(json.dumps(line))
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.swap:
        return run_swap(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
