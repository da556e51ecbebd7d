"""The C-ABI library loads and exports every entry point the header declares
(no GPU needed: only host-side calls that touch no device)."""
import ctypes
import os
import re
import subprocess

import pytest

from token_level_sparse_kv_b200 import build as jbuild
from token_level_sparse_kv_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jssa.h")


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(jssa_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def libpath():
    return jbuild.build()


def test_header_declares_the_path_entry_points():
    names = declared()
    for n in ("jssa_append_lowrank", "jssa_score", "jssa_topk", "jssa_select", "jssa_indexed_decode",
              "jssa_dense_decode", "jssa_gather_then_dense", "jssa_decode_step", "jssa_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in declared() if n not in exported]
    assert not missing, "declared but not exported: %s" % missing
    extra = sorted(n for n in exported if n.startswith("jssa_") and n not in declared())
    assert not extra, "exported but not declared: %s" % extra
    assert set(ops.EXPORTS) <= set(declared())


def test_library_loads_and_host_only_calls_work(libpath):
    L = ops.lib()
    assert L.jssa_version() == 2
    assert L.jssa_status_string(0) == b"JSSA_OK"
    assert b"INVALID" in L.jssa_status_string(-1)
    n = ctypes.c_size_t(0)
    # NULL dims and bad dims are rejected on the host before any CUDA call
    assert L.jssa_workspace_size(None, 1, 0, ctypes.byref(n)) == -1
    assert b"NULL" in L.jssa_last_error()
    bad = ops.Dims(1, 6, 4, 128, 128, 32, 16, 0, 0)  # Hq not a multiple of Hkv
    assert L.jssa_workspace_size(ctypes.byref(bad), 1, 0, ctypes.byref(n)) == -1
    odd_r = ops.Dims(1, 8, 2, 128, 128, 24, 16, 0, 0)
    assert L.jssa_workspace_size(ctypes.byref(odd_r), 1, 0, ctypes.byref(n)) == -2
    wide = ops.Dims(1, 8, 2, 96, 96, 32, 16, 0, 0)
    assert L.jssa_workspace_size(ctypes.byref(wide), 1, 0, ctypes.byref(n)) == -2
    good = ops.Dims(1, 8, 2, 128, 128, 32, 16, 0, 0)
    # k outside [1, 2048] and NULL / misaligned pointers
    assert L.jssa_workspace_size(ctypes.byref(good), 0, ops.OP_SELECT, ctypes.byref(n)) == -1
    assert L.jssa_workspace_size(ctypes.byref(good), 4096, ops.OP_SELECT, ctypes.byref(n)) == -1
    assert L.jssa_append_lowrank(ctypes.byref(good), None, None, None, None, 1, None, 0, None) == -1
    assert b"K is NULL" in L.jssa_last_error()
    p = ctypes.c_void_p(0x1001)
    assert L.jssa_append_lowrank(ctypes.byref(good), p, p, p, p, 1, p, 256, None) == -1
    assert b"aligned" in L.jssa_last_error()


def test_product_package_has_no_oracle_dependency():
    pkg = os.path.join(ROOT, "token_level_sparse_kv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "jssa_oracle" not in txt, f


def test_library_reads_no_environment_variables():
    """Dispatch choices are explicit arguments (jssa_select_opts), never the
    environment: the library source holds no getenv call."""
    csrc = os.path.join(ROOT, "token_level_sparse_kv_b200", "csrc")
    for f in os.listdir(csrc):
        if f.endswith((".cu", ".cuh", ".h")):
            assert "getenv" not in open(os.path.join(csrc, f)).read(), f


def test_select_opts_layout_matches_the_header():
    src = open(HEADER).read()
    body = re.search(r"typedef struct \{([^}]*)\} jssa_select_opts;", src).group(1)
    fields = re.findall(r"int32_t\s+(\w+);", body)
    fields += re.findall(r"float \*(\w+);", body)
    assert fields == [n for n, _ in ops.SelectOpts._fields_]
