"""CPU-side checks of the C-ABI library: it builds, loads without a GPU, exports every
symbol that include/rmm.h declares, and its pure host functions behave.  No call
here launches GPU work."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "rmm.h")


@pytest.fixture(scope="module")
def lib():
    from input_adaptive_reduced_rmm_b200 import build as b

    b.build()
    from input_adaptive_reduced_rmm_b200 import rmm

    return rmm.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(rmm_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("rmm_linear", "rmm_attn_qk", "rmm_score", "rmm_select", "rmm_gemm_reduced",
                 "rmm_transpose_weight", "rmm_get_status", "rmm_k_for"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    from input_adaptive_reduced_rmm_b200 import rmm

    names = declared_functions()
    assert sorted(rmm.EXPORTED) == names
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", rmm.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}\b", out), f"{n} not exported"


def test_k_for_matches_golden(lib, golden):
    from input_adaptive_reduced_rmm_b200 import rmm

    g = golden("k_for.json")
    for H, r, k in g["cases"]:
        assert rmm.rmm_k_for(H, r) == k
    for H, r in g["rejected"]:
        assert rmm.rmm_k_for(H, r) == -1


def test_status_strings(lib):
    from input_adaptive_reduced_rmm_b200 import rmm

    assert rmm.rmm_status_string(0) == "RMM_OK"
    assert rmm.rmm_status_string(5) == "RMM_ERR_TIMEOUT"
    assert rmm.rmm_status_string(99) == "RMM_ERR_UNKNOWN"


def test_argument_errors_return_before_any_launch(lib):
    from input_adaptive_reduced_rmm_b200 import rmm

    L = rmm.lib()
    # null pointers and bad r are rejected on the host with nothing enqueued
    assert L.rmm_linear(None, None, 4, 64, 64, 0.5, None, None, None, 0, None, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_attn_qk(None, None, None, 1, 1, 1, 1, 1, 8, 128, 0.5, 1, 1.0, None, None, None, 0, None,
                         None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_select(None, 10, 3, None, None, 0, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_transpose_weight(None, None, 4, 4, None) == rmm.RMM_ERR_INVALID_ARG
    bad = rmm.options()
    bad.t_gemv = 99
    assert L.rmm_linear_workspace_bytes(4, 64, 64, ctypes.byref(bad)) == 0


def test_workspace_sizes_are_monotone(lib):
    from input_adaptive_reduced_rmm_b200 import rmm

    small = rmm.rmm_linear_workspace_bytes(16, 4096, 4096)
    big = rmm.rmm_linear_workspace_bytes(2048, 4096, 4096)
    assert 0 < small and 0 < big
    # the GEMM path holds a full X^T
    assert big >= 4096 * 2048 * 2
    assert rmm.rmm_attn_workspace_bytes(1, 32, 8, 1, 4096) > 0
    assert rmm.rmm_attn_workspace_bytes(1, 32, 8, 1, 4096, 64) == 0  # d != 128


def test_product_code_never_touches_the_oracle():
    """The product package must not import, load or run anything under oracle/ (no CPU fallback)."""
    pkg = os.path.join(ROOT, "input_adaptive_reduced_rmm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "liboracle" not in text, f
                assert "rmm_oracle" not in text, f


def test_binding_fails_loudly_without_library(tmp_path):
    code = (
        "import input_adaptive_reduced_rmm_b200.rmm as r\n"
        f"r.LIB_PATH = {str(tmp_path / 'missing.so')!r}\n"
        "try:\n    r.lib()\nexcept RuntimeError as e:\n    print('raised', e)\n"
    )
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert "raised" in out.stdout
