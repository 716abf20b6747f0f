"""Benchmark of one decode step (one layer) over a paged KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is the whole hot path over one batch of synthetic input:
copy_blocks (when the workload has copy-on-write pairs), reshape_and_cache
of the step's new tokens, paged_decode (plus its split-context reduction).
The default workload is the LLaMA-7B-shaped decode: 64 sequences, 32/32
heads, head_dim 128, block_size 16, fp16, contexts uniform in [128, 2048],
16384-block pool, one new token per sequence.

Metric: algorithmic HBM bytes of the step / device time (GB/s), with the
time per step.  The K/V a step reads (about 1.1 GB) is far larger than the
126 MB L2, so no flush is needed between steps.

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
KERNEL_SOURCES = ["paged_kv_cache_415_b200/csrc/paged_decode.cu",
                  "paged_kv_cache_415_b200/csrc/paged_decode_mma.cuh",
                  "paged_kv_cache_415_b200/csrc/paged_decode_q8.cuh",
                  "paged_kv_cache_415_b200/csrc/pa_codes.cuh",
                  "paged_kv_cache_415_b200/csrc/pa_common.cuh"]
NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                0x100: "display_clock_setting"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="llama7b",
                    choices=["tiny", "llama7b", "mistral7b", "beam_search", "long_context"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--partition", type=int, default=-1,
                    help="context partition in tokens (-1 = the workload's, 0 = library's choice)")
    ap.add_argument("--separate", action="store_true",
                    help="run the cache write and the decode as separate calls even when every "
                         "sequence appends one token (default: pa_paged_decode_append)")
    ap.add_argument("--shared-prefix", action="store_true",
                    help="beam_search: decode with pa_paged_decode_shared_prefix (shared "
                         "prompt blocks read once per group)")
    ap.add_argument("--kv-dtype", default="auto", choices=["auto", "fp8", "int8"],
                    help="fp8 / int8: the same workload with e4m3 / int8 K/V pools (per-pool "
                         "scales), quantising cache write + decode over the codes")
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


def kernel_source_hash() -> str:
    """sha256[:16] of the decode kernels' sources, comments and blank lines
    removed: a profile taken on a hash still describes the current code."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(config: str):
    """DRAM bytes per launch of the decode kernel from a committed ncu
    summary, if it was taken on the current kernel source."""
    want = kernel_source_hash()
    if not os.path.isdir(PROFILE_GLOB_DIR):
        return None
    for name in sorted(os.listdir(PROFILE_GLOB_DIR)):
        if not name.endswith((".md", ".txt")):
            continue
        with open(os.path.join(PROFILE_GLOB_DIR, name)) as f:
            for line in f:
                m = re.search(r"bench-traffic:\s*workload=(\S+)\s+bytes_per_launch=(\d+)\s+"
                              r"source_sha256=(\w+)", line)
                if m and m.group(1) == config and m.group(3) == want:
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


def make_workload(config: str, seqs: int = 0, kv_dtype: str = "auto"):
    """The named workload; with seqs > 0 a smaller batch of the same shape
    and a pool sized to it (profiling captures stay a few GB); kv_dtype fp8
    or int8 redraws its pools as e4m3 or int8 codes."""
    from workloads import generators as gen
    wl = _make_workload(config, seqs)
    if kv_dtype in ("fp8", "int8"):
        wl = gen.with_code_pools(wl, kv_dtype, seed=gen.SEED_BASE + 50)
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
                              wl.block_size, 2, bm.kv_elem_bytes(wl))
        self.codes = wl.extra.get("kv_dtype")          # None, "fp8" or "int8"
        full = bm.step_bytes(wl)
        self.bytes = att["total"] + full["append"] + full["copy"]
        self.threads = oracle.max_threads()

    def run(self) -> float:
        o, wl = self.oracle, self.wl
        t0 = time.perf_counter()
        if wl.block_mapping.shape[0]:
            o.copy_blocks(self.kc, self.vc, wl.block_mapping)
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

    from paged_kv_cache_415_b200 import binding as B
    from workloads import byte_model as bm

    wl = make_workload(args.config, args.seqs, args.kv_dtype)
    dev = torch.device("cuda", local)
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16}[wl.dtype]
    codes = wl.extra.get("kv_dtype")                  # None, "fp8" or "int8"
    quant = codes is not None
    if quant:
        q_write, q_decode, q_decode_append = (
            getattr(B, f"pa_reshape_and_cache_{codes}"), getattr(B, f"pa_paged_decode_{codes}"),
            getattr(B, f"pa_paged_decode_{codes}_append"))
    k_scale, v_scale = wl.extra.get("k_scale", 1.0), wl.extra.get("v_scale", 1.0)

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(tdt)

    if quant:
        k_cache = torch.from_numpy(wl.k_cache).to(dev)
        v_cache = torch.from_numpy(wl.v_cache).to(dev)
    else:
        k_cache, v_cache = up(wl.k_cache), up(wl.v_cache)
    query = up(wl.query)
    new_key, new_value = up(wl.new_key), up(wl.new_value)
    slot_mapping = torch.from_numpy(wl.slot_mapping).to(dev)
    block_tables = torch.from_numpy(wl.block_tables).to(dev)
    context_lens = torch.from_numpy(wl.context_lens).to(dev)
    block_mapping = torch.from_numpy(np.ascontiguousarray(wl.block_mapping)).to(dev)
    out = torch.empty_like(query)
    d_status = torch.zeros(1, dtype=torch.int32, device=dev)
    mcl = wl.max_context_len
    want = wl.partition_size if args.partition < 0 else args.partition
    part = B.pa_paged_decode_partition_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                            wl.head_dim, wl.block_size, mcl, want)
    ws_bytes = B.pa_paged_decode_workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                                wl.head_dim, wl.block_size, mcl, part)
    workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    max_parts = -(-mcl // part) if mcl > 0 else 1
    n_pairs = int(wl.block_mapping.shape[0])
    stream = torch.cuda.current_stream(dev)

    fused = (not args.separate and not args.shared_prefix
             and wl.extra.get("one_token_per_seq", False) and wl.num_new_tokens == wl.num_seqs)

    def cache_ops():
        if n_pairs:
            B.pa_copy_blocks(k_cache, v_cache, block_mapping, d_status, stream)
        if wl.num_new_tokens and quant and not fused:
            q_write(new_key, new_value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                    d_status, stream)
        elif wl.num_new_tokens and not fused:
            B.pa_reshape_and_cache(new_key, new_value, k_cache, v_cache, slot_mapping, d_status,
                                   stream)

    shared = args.shared_prefix and "prefix_lens" in wl.extra and not quant
    if shared:
        group_size = int(wl.extra["group_size"])
        prefix_lens = torch.from_numpy(wl.extra["prefix_lens"]).to(dev)
        mpl = int(wl.extra["prefix_lens"].max())
        sws = B.pa_paged_decode_shared_prefix_workspace_size(
            wl.num_seqs, group_size, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
            mcl, mpl, 0)
        workspace = torch.empty(max(sws, 16), dtype=torch.uint8, device=dev)

    def decode():
        if quant and fused:
            q_decode_append(out, query, new_key, new_value, k_cache, v_cache, block_tables,
                            context_lens, mcl, wl.scale, k_scale, v_scale, part, workspace,
                            d_status, stream)
        elif quant:
            q_decode(out, query, k_cache, v_cache, block_tables, context_lens, mcl, wl.scale,
                     k_scale, v_scale, part, workspace, d_status, stream)
        elif fused:
            B.pa_paged_decode_append(out, query, new_key, new_value, k_cache, v_cache,
                                     block_tables, context_lens, mcl, wl.scale, part, workspace,
                                     d_status, stream)
        elif shared:
            B.pa_paged_decode_shared_prefix(out, query, k_cache, v_cache, block_tables,
                                            context_lens, prefix_lens, group_size, mcl, mpl,
                                            wl.scale, workspace, 0, d_status, stream)
        else:
            B.pa_paged_decode(out, query, k_cache, v_cache, block_tables, context_lens, mcl,
                              wl.scale, part, workspace, d_status, stream)

    shared_parts_gt1 = shared and sws > 0            # a reduction runs after the shared kernel
    launches_per_step = (1 if n_pairs else 0) + (1 if (wl.num_new_tokens and not fused) else 0) + \
        1 + (1 if (max_parts > 1 and not shared) or shared_parts_gt1 else 0)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # warm-up
    for _ in range(args.warmup):
        cache_ops()
        decode()
    barrier()
    run_cache, run_decode = cache_ops, decode
    if not args.eager:
        # the step's launches captured once; replay issues them with no host work
        g_cache, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        has_cache = bool(n_pairs or (wl.num_new_tokens and not fused))
        saved = stream
        with torch.cuda.graph(g_dec):
            stream = torch.cuda.current_stream(dev)
            decode()
        if has_cache:
            with torch.cuda.graph(g_cache):
                stream = torch.cuda.current_stream(dev)
                cache_ops()
        stream = saved
        run_cache = g_cache.replay if has_cache else (lambda: None)
        run_decode = g_dec.replay
        run_cache()
        run_decode()
        barrier()
    if int(d_status.item()) != 0 or not torch.isfinite(out.float()).all():
        raise SystemExit(f"rank {rank}: bad step (status {int(d_status.item())})")

    # timed region: K steps; events bracket the decode kernels of every step
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier()
    with sampler:
        start.record(stream)
        for i in range(args.steps):
            run_cache()
            ev[i][0].record(stream)
            run_decode()
            ev[i][1].record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    elapsed_ms = start.elapsed_time(stop)
    decode_ms = [a.elapsed_time(b) for a, b in ev]

    # end to end through the public API: pinned host inputs -> device -> step -> host output
    from paged_kv_cache_415_b200.step import DecodeStep, HostPipeline
    stepper = DecodeStep(k_cache, v_cache, wl.num_seqs, wl.num_q_heads, mcl, part, k_scale,
                         v_scale)
    host = {"query": torch.from_numpy(wl.query.view(np.int16)).view(tdt).pin_memory(),
            "block_tables": torch.from_numpy(wl.block_tables).pin_memory(),
            "context_lens": torch.from_numpy(wl.context_lens).pin_memory(),
            "out": torch.empty(out.shape, dtype=tdt).pin_memory()}
    devb = {"query": torch.empty_like(query), "block_tables": torch.empty_like(block_tables),
            "context_lens": torch.empty_like(context_lens), "out": torch.empty_like(out)}
    if wl.num_new_tokens:
        host["new_key"] = torch.from_numpy(wl.new_key.view(np.int16)).view(tdt).pin_memory()
        host["new_value"] = torch.from_numpy(wl.new_value.view(np.int16)).view(tdt).pin_memory()
        names = ("new_key", "new_value")
        if not fused:
            host["slot_mapping"] = torch.from_numpy(wl.slot_mapping).pin_memory()
            names += ("slot_mapping",)
        for k in names:
            devb[k] = torch.empty_like(host[k], device=dev)
    if n_pairs:
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
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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
    # the decode launch also carries the step's cache write when it is fused
    decode_bytes = step["attention"] + (step["append"] if fused else 0)
    achieved = decode_bytes / (decode_avg * 1e-3) / 1e9
    traffic = profiled_traffic(args.config + (f"-{codes}" if quant else ""))
    clocks = sampler.summary()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        g, _, desc, threads = oracle_sample_time(wl, args.cpu_seconds)
        cpu = {"value": round(g, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    group = wl.num_q_heads // wl.num_kv_heads
    if shared:
        kernel_name = "paged_decode_shared_kernel" + (
            " + paged_decode_shared_reduce_kernel" if shared_parts_gt1 else "")
    else:
        kernel_name = (f"paged_decode_{codes}_kernel" if quant else
                       "paged_decode_mma_kernel" if group >= 4 and wl.block_size % 16 == 0
                       else "paged_decode_kernel")
        if max_parts > 1:
            kernel_name += " + paged_decode_reduce_kernel"
    l2 = (f"no flush: {step['kv'] / 1e9:.2f} GB of K/V per step > 126 MB L2"
          if step["kv"] > 4 * 126e6 else "working set smaller than L2 (values include L2 hits)")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ({"fp8": "f16 (e4m3 K/V)", "int8": "f16 (int8 K/V)"}[codes] if quant
                  else wl.dtype),
        "data": "synthetic", "config": workload_config(wl, part, l2),
        "us_per_layer_step": round(per_step_ms * 1e3, 2),
        "kv_tokens_per_s": round(world * int(wl.context_lens.sum()) * args.steps / (elapsed_ms * 1e-3)),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "roofline": {"bound": "hbm", "kernel": kernel_name,
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "algorithmic_bytes_per_launch": decode_bytes,
                     "avg_launch_us": round(decode_avg * 1e3, 2)},
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
        "decode_entry": (f"pa_paged_decode_{codes}_append (quantising cache write fused)"
                         if quant and fused else
                         f"pa_reshape_and_cache_{codes} + pa_paged_decode_{codes}" if quant else
                         "pa_paged_decode_shared_prefix" if shared else
                         "pa_paged_decode_append (cache write fused)" if fused else
                         "pa_reshape_and_cache + pa_paged_decode"),
    }
    if "prefix_lens" in wl.extra:
        uniq = bm.unique_kv_bytes(wl)
        line["unique_kv_bytes"] = uniq
        line["unique_kv_gbs_decode"] = round(uniq / (decode_avg * 1e-3) / 1e9, 1)
    print(json.dumps(line))
    return 0


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
