"""The C-ABI library: it loads, exports every entry point include/pa.h
declares, and its host-side argument checks reject bad calls before any
device work (CPU only: no call here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


def _declared(header=HEADER):
    text = open(header).read()
    return re.findall(r"^PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text, flags=re.M)


def _all_headers():
    inc = os.path.join(ROOT, "include")
    return [os.path.join(inc, f) for f in sorted(os.listdir(inc)) if f.endswith(".h")]


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_415_b200 import build
    build.build()
    from paged_kv_cache_415_b200 import binding
    return binding


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("pa_reshape_and_cache", "pa_copy_blocks", "pa_paged_decode",
              "pa_paged_decode_workspace_size", "pa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(pa):
    lib = ctypes.CDLL(pa.LIB_PATH)
    names = [n for h in _all_headers() for n in _declared(h)]
    assert len(names) >= 20
    for name in names:
        assert hasattr(lib, name), f"libpa.so does not export {name}"
    assert set(_declared()) == set(pa.EXPORTS)
    assert set(_declared(os.path.join(ROOT, "include", "pa_selftest.h"))) == set(pa.SELFTEST_EXPORTS)


def test_no_alloc_scratch_size_matches_the_header(pa):
    """The binding's PA_NO_ALLOC_WORKSPACE_BYTES is the header's #define."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+PA_NO_ALLOC_WORKSPACE_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", text)
    assert m, "PA_NO_ALLOC_WORKSPACE_BYTES not found in pa.h"
    assert pa.PA_NO_ALLOC_WORKSPACE_BYTES == int(m.group(1)) << int(m.group(2))


def _no_alloc(pa, **kw):
    args = dict(out=FAKE, query=FAKE, k_cache=FAKE, v_cache=FAKE, block_tables=FAKE,
                context_lens=FAKE, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=128,
                block_size=16, max_blocks_per_seq=8, num_blocks=64, max_context_len=100,
                scale=0.1, partition_size=0, dtype=0, d_status=None, stream=None)
    args.update(kw)
    return pa.LIB.pa_paged_decode_no_alloc(*args.values())


def test_no_alloc_refuses_oversized_scratch_on_the_host(pa):
    """A shape whose split-context scratch is larger than the library's
    fixed array is refused (PA_ERR_INVALID_ARG) before anything is enqueued
    or any device address is looked up; one just inside the limit gets past
    that check (and fails on the null pointer instead)."""
    s, hq, d = 64, 32, 128
    need = pa.pa_paged_decode_workspace_size(s, hq, hq, d, 16, 8192, 16)
    assert need > pa.PA_NO_ALLOC_WORKSPACE_BYTES
    assert _no_alloc(pa, num_seqs=s, num_q_heads=hq, num_kv_heads=hq, max_context_len=8192,
                     max_blocks_per_seq=512, partition_size=16) == pa.PA_ERR_INVALID_ARG
    # the largest fitting context for one sequence of 8 query heads, 16-token partitions
    per_part = 8 * (d + 2) * 4
    fit = pa.PA_NO_ALLOC_WORKSPACE_BYTES // per_part * 16
    assert pa.pa_paged_decode_workspace_size(1, 8, 2, d, 16, fit, 16) <= pa.PA_NO_ALLOC_WORKSPACE_BYTES
    assert pa.pa_paged_decode_workspace_size(1, 8, 2, d, 16, fit + 16, 16) > pa.PA_NO_ALLOC_WORKSPACE_BYTES
    assert _no_alloc(pa, num_seqs=1, max_context_len=fit + 16, partition_size=16) == pa.PA_ERR_INVALID_ARG
    assert _no_alloc(pa, num_seqs=1, max_context_len=fit, partition_size=16, out=None) == pa.PA_ERR_INVALID_ARG


def test_selftest_entry_points_check_their_arguments(pa):
    """Refused on the host: a missing status word, a wait limit of 0 or
    above 1 s, a grid outside 1..1024 CTAs, a key-value type that is neither
    the query's nor a code type."""
    B = pa
    assert B.LIB.pa_selftest_bounded_wait(None, None, 1000, 1, None) == 1
    assert B.LIB.pa_selftest_bounded_wait(FAKE, None, 0, 1, None) == 1
    assert B.LIB.pa_selftest_bounded_wait(FAKE, None, 1000001, 1, None) == 1
    assert B.LIB.pa_selftest_bounded_wait(FAKE, None, 1000, 0, None) == 1
    assert B.LIB.pa_selftest_bounded_wait(FAKE, None, 1000, 1025, None) == 1
    assert B.LIB.pa_selftest_bounded_wait(FAKE, FAKE + 4, 1000, 1, None) == 1
    base = [FAKE] * 6 + [4, 8, 2, 128, 16, 8, 64, 100, 0.1, 0, None, 0, 0]
    assert B.LIB.pa_selftest_decode_abort(*base, 0, 0, None, None) == 1          # limit 0
    assert B.LIB.pa_selftest_decode_abort(*base, 0, 2000000, None, None) == 1    # limit > 1 s
    assert B.LIB.pa_selftest_decode_abort(*base, 1, 1000, None, None) == 2       # bf16 pools, f16 query


def test_status_strings(pa):
    assert pa.pa_status_string(0) == "PA_OK"
    assert pa.pa_status_string(1) == "PA_ERR_INVALID_ARG"
    assert pa.pa_status_string(2) == "PA_ERR_UNSUPPORTED"
    assert pa.pa_status_string(3) == "PA_ERR_CUDA"
    assert pa.pa_status_string(77) == "PA_ERR_UNKNOWN"
    assert re.match(r"\d+\.\d+\.\d+", pa.pa_version())


def test_partition_and_workspace_sizes(pa):
    ps, ws = pa.pa_paged_decode_partition_size, pa.pa_paged_decode_workspace_size
    # short contexts: one partition covering the whole (block-rounded) context, no workspace
    assert ps(4, 2, 2, 64, 16, 40, 0) == 48 and ws(4, 2, 2, 64, 16, 40, 0) == 0
    # many (seq, kv head) pairs and contexts up to 2048: one partition per context
    assert ps(64, 32, 32, 128, 16, 1982, 0) == 1984 and ws(64, 32, 32, 128, 16, 1982, 0) == 0
    # longer contexts: about 1/4 of the longest, a power of two in [512, 2048] ...
    assert ps(256, 32, 8, 128, 16, 8192, 0) == 2048
    assert ps(256, 32, 8, 128, 16, 3900, 0) == 1024
    assert ps(16, 32, 8, 128, 16, 32768, 0) == 2048
    # ... halved while the grid would hold fewer than 4 x 148 CTAs
    assert ps(16, 32, 8, 128, 16, 3000, 0) == 512
    assert ps(2, 32, 8, 128, 16, 32768, 0) == 512
    # workspace: (D + 2) floats per (seq, q head, partition)
    assert ws(16, 32, 8, 128, 16, 32768, 0) == 16 * 32 * 16 * (128 + 2) * 4      # P = 2048
    assert ws(16, 32, 8, 128, 16, 32768, 1024) == 16 * 32 * 32 * (128 + 2) * 4
    # the caller's partition wins; it must be a multiple of block_size
    assert ps(1, 1, 1, 128, 16, 100, 32) == 32
    assert ps(1, 1, 1, 128, 16, 100, 24) == 0
    # unsupported shapes
    assert ps(1, 3, 1, 128, 16, 100, 0) == 0          # group of 3
    assert ps(1, 2, 2, 96, 16, 100, 0) == 0           # head_dim 96
    assert ps(1, 2, 2, 128, 12, 100, 0) == 0          # block 12


FAKE = 1 << 20                       # 16-byte aligned, never dereferenced


def _decode(pa, **kw):
    args = dict(out=FAKE, query=FAKE, k_cache=FAKE, v_cache=FAKE, block_tables=FAKE,
                context_lens=FAKE, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=128,
                block_size=16, max_blocks_per_seq=8, num_blocks=64, max_context_len=100,
                scale=0.1, partition_size=0, workspace=None, workspace_bytes=0, dtype=0,
                d_status=None, stream=None)
    args.update(kw)
    return pa.LIB.pa_paged_decode(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(out=None), 1), (dict(query=None), 1), (dict(k_cache=None), 1),
    (dict(block_tables=None), 1), (dict(context_lens=None), 1),
    (dict(out=FAKE + 8), 1), (dict(k_cache=FAKE + 4), 1), (dict(block_tables=FAKE + 2), 1),
    (dict(num_q_heads=6, num_kv_heads=4), 1), (dict(num_q_heads=0), 1),
    (dict(num_seqs=-1), 1), (dict(max_context_len=-5), 1), (dict(partition_size=24), 1),
    (dict(partition_size=-16), 1), (dict(max_blocks_per_seq=0), 1), (dict(num_blocks=0), 1),
    (dict(scale=float("nan")), 1),
    (dict(max_context_len=4096, workspace=None), 1),
    (dict(max_context_len=4096, workspace=FAKE, workspace_bytes=16), 1),
    (dict(head_dim=96), 2), (dict(block_size=12), 2), (dict(num_q_heads=6, num_kv_heads=2), 2),
    (dict(num_q_heads=32, num_kv_heads=2), 2), (dict(dtype=5), 2),
])
def test_decode_rejects_bad_arguments(pa, kw, code):
    assert _decode(pa, **kw) == code


def test_decode_with_no_sequences_is_a_no_op(pa):
    assert _decode(pa, num_seqs=0) == 0


def _cache(pa, **kw):
    args = dict(key=FAKE, value=FAKE, k_cache=FAKE, v_cache=FAKE, slot_mapping=FAKE, num_tokens=4,
                num_kv_heads=2, head_dim=64, block_size=16, num_blocks=64, dtype=0, d_status=None,
                stream=None)
    args.update(kw)
    return pa.LIB.pa_reshape_and_cache(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(key=None), 1), (dict(v_cache=None), 1), (dict(slot_mapping=None), 1),
    (dict(key=FAKE + 8), 1), (dict(slot_mapping=FAKE + 4), 1), (dict(num_tokens=-1), 1),
    (dict(num_kv_heads=0), 1), (dict(num_blocks=0), 1), (dict(d_status=FAKE + 1), 1),
    (dict(head_dim=80), 2), (dict(block_size=64), 2), (dict(dtype=9), 2),
])
def test_reshape_and_cache_rejects_bad_arguments(pa, kw, code):
    assert _cache(pa, **kw) == code


def test_empty_calls_are_no_ops(pa):
    assert _cache(pa, num_tokens=0) == 0
    assert pa.LIB.pa_copy_blocks(FAKE, FAKE, FAKE, 0, 2, 64, 16, 64, 0, None, None) == 0


@pytest.mark.parametrize("args,code", [
    ((None, FAKE, FAKE, 2, 2, 64, 16, 64, 0, None, None), 1),
    ((FAKE, FAKE, None, 2, 2, 64, 16, 64, 0, None, None), 1),
    ((FAKE, FAKE, FAKE + 4, 2, 2, 64, 16, 64, 0, None, None), 1),
    ((FAKE, FAKE, FAKE, -1, 2, 64, 16, 64, 0, None, None), 1),
    ((FAKE, FAKE, FAKE, 2, 2, 48, 16, 64, 0, None, None), 2),
    ((FAKE, FAKE, FAKE, 2, 2, 64, 16, 64, 4, None, None), 2),
])
def test_copy_blocks_rejects_bad_arguments(pa, args, code):
    assert pa.LIB.pa_copy_blocks(*args) == code


def test_headers_and_library_from_plain_c(pa, tmp_path):
    """A C99 program that includes include/*.h alone (no CUDA or C++
    header) compiles without warnings, links against libpa.so and runs its
    host-only checks (tests/c/abi_from_c.c)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    exe = tmp_path / "abi_from_c"
    lib_dir = os.path.dirname(pa.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_from_c.c"),
                    "-o", str(exe), "-L", lib_dir, "-l:libpa.so", f"-Wl,-rpath,{lib_dir}"],
                   check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stderr
    assert "abi from C ok" in res.stdout


def test_decode_refuses_grids_past_the_launch_limits(pa):
    """More than 65535 sequences, or more than 65535 context partitions,
    would exceed the grid's y/z limits: refused as PA_ERR_UNSUPPORTED before
    any launch (the workspace, when one is needed, is large enough)."""
    assert _decode(pa, num_seqs=70000, max_context_len=100) == 2
    assert _decode(pa, num_seqs=65535, max_context_len=100, out=None) == 1   # checks still run
    mcl, part = 16 * 70000, 16
    need = pa.pa_paged_decode_workspace_size(1, 8, 2, 128, 16, mcl, part)
    assert need == 8 * 70000 * (128 + 2) * 4
    assert _decode(pa, num_seqs=1, max_context_len=mcl, partition_size=part, workspace=FAKE,
                   workspace_bytes=need) == 2
    assert _decode(pa, num_seqs=1, max_context_len=mcl, partition_size=part, workspace=FAKE,
                   workspace_bytes=need - 16) == 1                                # too small first


def test_no_fallback_without_the_library(tmp_path):
    """The package has no CPU path: a copy of it without libpa.so fails at
    import of the binding, naming the missing library, and an op reached
    through the package's lazy exports fails the same way."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "paged_kv_cache_415_b200")
    dst = tmp_path / "paged_kv_cache_415_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "*.o", "__pycache__", "_build"))
    for code in ("import paged_kv_cache_415_b200.binding",
                 "import paged_kv_cache_415_b200 as p; p.pa_paged_decode"):
        res = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True,
                             text=True, timeout=300)
        assert res.returncode != 0
        assert "libpa.so" in res.stderr and "ImportError" in res.stderr, res.stderr[-500:]


def test_rowscale_calls_check_their_arguments(pa):
    """The row-scaled calls refuse, before any device work: missing or
    misaligned scale pools, block size 8 in the decode (whole 16-token
    slices only), a bad query type.  pa_copy_blocks takes scale pools as
    PA_DTYPE_F32 with head_dim 1 only."""
    L = pa.LIB
    w = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 16, 64, 0, None, None]
    for fn in (L.pa_reshape_and_cache_fp8_rowscale, L.pa_reshape_and_cache_int8_rowscale):
        bad = list(w); bad[4] = None
        assert fn(*bad) == 1                                   # no K scale pool
        bad = list(w); bad[5] = FAKE + 4
        assert fn(*bad) == 1                                   # V scales not 16-byte aligned
        bad = list(w); bad[9] = 96
        assert fn(*bad) == 2                                   # head_dim 96
        bad = list(w); bad[7] = -1
        assert fn(*bad) == 1
        bad = list(w); bad[7] = 0
        assert fn(*bad) == 0                                   # nothing to write
    d = [FAKE] * 8 + [4, 8, 2, 128, 16, 8, 64, 100, 0.1, 0, None, 0, 0, None, None]
    for fn in (L.pa_paged_decode_fp8_rowscale, L.pa_paged_decode_int8_rowscale):
        bad = list(d); bad[4] = None
        assert fn(*bad) == 1
        bad = list(d); bad[5] = FAKE + 8
        assert fn(*bad) == 1
        bad = list(d); bad[12] = 8
        assert fn(*bad) == 2                                   # block size 8
        bad = list(d); bad[20] = 7
        assert fn(*bad) == 2                                   # unknown query type
    a = [FAKE] * 10 + [4, 8, 2, 128, 16, 8, 64, 100, 0.1, 0, None, 0, 0, None, None]
    for fn in (L.pa_paged_decode_fp8_rowscale_append, L.pa_paged_decode_int8_rowscale_append):
        bad = list(a); bad[2] = None
        assert fn(*bad) == 1                                   # no new keys
        bad = list(a); bad[7] = None
        assert fn(*bad) == 1                                   # no V scale pool
    cp = L.pa_copy_blocks
    assert cp(FAKE, FAKE, FAKE, 0, 8, 1, 16, 64, pa.PA_DTYPE_F32, None, None) == 0
    assert cp(FAKE, FAKE, FAKE, 2, 8, 2, 16, 64, pa.PA_DTYPE_F32, None, None) == 2   # head_dim 2
    assert cp(FAKE, FAKE, FAKE, 2, 8, 1, 12, 64, pa.PA_DTYPE_F32, None, None) == 2   # block 12
    assert cp(FAKE, FAKE, FAKE, 2, 8, 1, 16, 64, pa.PA_DTYPE_F16, None, None) == 2   # 16-bit, D 1
