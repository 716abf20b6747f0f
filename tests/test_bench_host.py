"""Host-side logic of bench.py (no GPU): workload construction for every
mode, the JSON config block, the byte accounting of the CPU legs and the
committed profile lines the roofline object reads."""
import os
import re

import numpy as np
import pytest

import bench
from workloads import byte_model as bm


@pytest.mark.parametrize("config", ["tiny", "llama7b", "mistral7b", "long_context", "beam_search"])
def test_small_workloads_and_config_block(config):
    wl = bench.make_workload(config, seqs=4 if config != "tiny" else 0)
    cfg = bench.workload_config(wl, 64, "note")
    assert cfg["num_seqs"] == wl.num_seqs and cfg["partition_size"] == 64
    for key in ("workload", "num_q_heads", "num_kv_heads", "head_dim", "block_size", "layers", "l2"):
        assert key in cfg
    assert cfg["workload"].startswith(wl.name)


@pytest.mark.parametrize("kv,np_dtype,label", [("fp8", np.uint8, "e4m3"), ("int8", np.int8, "int8")])
def test_code_workload_modes(kv, np_dtype, label):
    wl = bench.make_workload("llama7b", seqs=3, kv_dtype=kv)
    assert wl.extra["kv_dtype"] == kv and wl.k_cache.dtype == np_dtype
    assert label in bench.workload_config(wl, 0, "")["workload"]
    full = bm.step_bytes(wl)
    base = bm.step_bytes(bench.make_workload("llama7b", seqs=3))
    assert full["kv"] * 2 == base["kv"]


@pytest.mark.parametrize("kv", ["fp8-rows", "int8-rows"])
def test_rowscale_workload_mode(kv):
    """--kv-dtype fp8-rows / int8-rows: code pools plus fp32 row-scale pools
    [num_blocks][Hkv][B] (NaN where no history token sits); the byte model
    adds 4 bytes per (token, kv head) row and per written row."""
    wl = bench.make_workload("mistral7b", seqs=3, kv_dtype=kv)
    assert wl.extra["rowscale"] and wl.extra["kv_dtype"] == kv[:-5]
    nb, b, h = wl.num_blocks, wl.block_size, wl.num_kv_heads
    assert wl.extra["k_scales"].shape == (nb, h, b) and wl.extra["k_scales"].dtype == np.float32
    assert "one scale per (token, kv head) row" in bench.workload_config(wl, 0, "")["workload"]
    plain = bm.step_bytes(bench.make_workload("mistral7b", seqs=3, kv_dtype=kv[:-5]))
    rows = bm.step_bytes(wl)
    assert rows["kv"] - plain["kv"] == int(wl.context_lens.sum()) * h * 4 * 2
    assert rows["append"] - plain["append"] == wl.num_new_tokens * h * 4 * 2
    st = bench.OracleStep(wl)
    assert st.bytes == rows["total"] and st.run() > 0.0


def test_oracle_step_counts_the_step_bytes():
    """The CPU leg times the oracle on the same step the GPU runs and
    counts the same algorithmic bytes (all sequences, 16-bit and both code
    formats)."""
    for config, seqs in (("llama7b", 2), ("tiny", 0)):          # tiny: block copies too
        for kv in ("auto", "fp8", "int8"):
            wl = bench.make_workload(config, seqs=seqs, kv_dtype=kv)
            st = bench.OracleStep(wl)
            assert st.bytes == bm.step_bytes(wl)["total"]
            assert st.run() > 0.0


def test_committed_traffic_lines_parse():
    """Every bench-traffic line under profiles/ has a workload, a byte count
    and a source hash, and names one of the bench's workloads."""
    names = {"tiny", "llama7b", "mistral7b", "long_context", "beam_search"}
    found = 0
    for name in os.listdir(bench.PROFILE_GLOB_DIR):
        with open(os.path.join(bench.PROFILE_GLOB_DIR, name)) as f:
            for line in f:
                if line.startswith("bench-traffic:"):
                    m = re.match(r"bench-traffic:\s*workload=(\S+)\s+bytes_per_launch=(\d+)\s+"
                                 r"source_sha256=(\w{16})\s*$", line)
                    assert m, line
                    base = re.sub(r"-((fp8|int8)(-rows)?|shared)$", "", m.group(1))
                    assert base in names, m.group(1)
                    assert int(m.group(2)) > 0
                    found += 1
    assert found >= 3


def test_source_hash_ignores_comments_only():
    """The profile hash covers code, not comments: stripping removes // and
    /* */ comments and blank lines, keeps string and character literals."""
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "a//b"; char q = \'/\';\n\n'
    assert bench.strip_comments(src) == 'int a = 1;\n const char* s = "a//b"; char q = \'/\';'
    assert bench.strip_comments(src) == bench.strip_comments(src.replace("note", "other"))
    assert bench.strip_comments(src) != bench.strip_comments(src.replace("a = 1", "a = 2"))


def _json_lines(text):
    import json
    return [json.loads(x) for x in text.splitlines() if x.startswith("{")]


def test_reference_arm_line():
    """`bench.py --impl reference` times the oracle on the host and prints
    one JSON line with the contract's keys; its value is its own e2e and
    cpu_baseline value."""
    import subprocess
    import sys
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny",
                          "--steps", "2", "--warmup", "1"], cwd=bench.ROOT, capture_output=True,
                         text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    lines = _json_lines(res.stdout)
    assert len(lines) == 1
    line = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["value"] == line["value"] and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 == line["e2e"]["d2h_bytes_per_step"]


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the multi-GPU run is (torchrun, two ranks), only rank 0
    runs the oracle and prints; the other rank exits 0 without output."""
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    res = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                          "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                          str(port), "bench.py", "--impl", "reference", "--gpus", "2",
                          "--config", "tiny", "--steps", "1", "--warmup", "1"],
                         cwd=bench.ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = _json_lines(res.stdout)
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_sharing_workload_roofline_counts_unique_bytes():
    """A workload whose sequences share stored blocks (the beams of a prompt)
    gets its roofline fraction on unique K/V bytes -- the blocks the step
    must read at least once -- and reports the referenced bytes beside
    them; other workloads have no referenced figure."""
    wl = bench.make_workload("beam_search", seqs=8)
    g = bench.GpuStep.__new__(bench.GpuStep)
    g.wl, g.fused = wl, False
    unique, referenced = g.roofline_bytes()
    step = bm.step_bytes(wl)
    assert referenced == step["attention"]
    assert unique == step["attention"] - step["kv"] + bm.unique_kv_bytes(wl)
    assert unique < referenced
    g.wl = bench.make_workload("llama7b", seqs=3)
    assert g.roofline_bytes() == (bm.step_bytes(g.wl)["attention"], None)


def test_clock_records_of_both_regions_merge():
    a = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 3, "source": "nvml"}
    b = {"sm_mhz": 1950, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 40,
         "source": "nvml"}
    m = bench.merge_clocks(a, b)
    assert m["sm_mhz"] == 1950 and m["samples"] == 43 and m["reasons"] == ["sw_power_cap"]
    assert bench.merge_clocks(a, {"samples": 0}) == a


def test_pair_rule_matches_the_library():
    """The bench names the one-byte kernel the library picks: its
    blocks-per-warp threshold is the library's kPairBelowBlocks."""
    src = os.path.join(os.path.dirname(bench.__file__), "paged_kv_cache_415_b200", "csrc",
                       "paged_decode.cu")
    with open(src, encoding="utf-8") as f:
        m = re.search(r"constexpr int kPairBelowBlocks = (\d+);", f.read())
    assert m, "kPairBelowBlocks not found"
    assert int(m.group(1)) == bench.PAIR_BELOW_BLOCKS
