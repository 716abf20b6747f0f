"""The oracle and the product path share no code: no module of the product
package imports the oracle (or the test-side workload generators), and no
module of the oracle imports the product package.  Checked on the import
statements of every Python source, and on the C sources' #include lines."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _py_files(folder):
    for dirpath, _, files in os.walk(os.path.join(ROOT, folder)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def test_product_never_imports_the_oracle():
    files = list(_py_files("paged_kv_cache_415_b200"))
    assert files
    for path in files:
        bad = _imports(path) & {"oracle", "workloads", "tests"}
        assert not bad, f"{path} imports {bad}"


def test_oracle_never_imports_the_product():
    files = list(_py_files("oracle"))
    assert files
    for path in files:
        assert "paged_kv_cache_415_b200" not in _imports(path), path


def test_c_sources_share_no_headers():
    """The oracle's C source includes only the C standard library (and
    OpenMP); the CUDA sources include nothing from oracle/."""
    oracle_c = open(os.path.join(ROOT, "oracle", "pa_oracle.c")).read()
    for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', oracle_c):
        assert inc in {"float.h", "math.h", "stdint.h", "stdlib.h", "string.h", "omp.h"}, inc
    csrc = os.path.join(ROOT, "paged_kv_cache_415_b200", "csrc")
    for f in os.listdir(csrc):
        text = open(os.path.join(csrc, f)).read()
        assert "oracle" not in " ".join(re.findall(r'#include\s*[<"]([^>"]+)[>"]', text)), f


def _tracked_code():
    import subprocess
    out = subprocess.run(["git", "ls-files", "*.py", "*.cu", "*.cuh", "*.h", "*.c", "*.cpp"],
                         cwd=ROOT, capture_output=True, text=True)
    files = out.stdout.split() if out.returncode == 0 else []
    if not files:                                    # not a git checkout: walk the sources
        for folder in ("paged_kv_cache_415_b200", "oracle", "workloads", "tests", "include"):
            for dirpath, _, names in os.walk(os.path.join(ROOT, folder)):
                files += [os.path.relpath(os.path.join(dirpath, n), ROOT) for n in names
                          if n.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp"))]
        files += ["bench.py", "__graft_entry__.py"]
    return files


def test_code_reads_no_reference_pages_and_no_working_files():
    """No committed source reaches the reference pages' location or the
    untracked working folder at run time."""
    me = os.path.relpath(os.path.abspath(__file__), ROOT)
    for rel in _tracked_code():
        if rel == me:
            continue
        text = open(os.path.join(ROOT, rel), encoding="utf-8").read()
        assert "/root/reference" not in text, rel
        assert not re.search(r"[\"'/]_work[/\"']", text), rel
