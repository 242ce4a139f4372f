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


def test_context_block_entry_points_validate_on_the_host(lib):
    """rmm_ctx_block_means / rmm_attn_ctx reject bad arguments before anything is enqueued
    (the fake pointers below are never dereferenced)."""
    from input_adaptive_reduced_rmm_b200 import rmm

    L = rmm.lib()
    fake = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never touched
    # block means: null pointers, a block size outside {32, 64, 128, 256}, a range past ceil(L/block)
    assert L.rmm_ctx_block_means(None, 1, 1, 128, 256, 256, 64, 0, 4, None, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_ctx_block_means(fake, 1, 1, 128, 256, 256, 48, 0, 1, fake, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_ctx_block_means(fake, 1, 1, 128, 256, 256, 64, 3, 5, fake, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_ctx_block_means(fake, 1, 1, 128, 256, 256, 64, 2, 2, fake, None) == rmm.RMM_ERR_INVALID_ARG
    # attention: no block means, a bad block, r_ctx out of (0, 1]
    args = lambda means, block, r_ctx: (fake, fake, fake, means, 1, 4, 1, 1, 256, 256, 128, 0.5, r_ctx, block, 1,
                                        1.0, fake, None, None, fake, 1 << 20, None, None)
    assert L.rmm_attn_ctx(*args(None, 64, 0.5)) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_attn_ctx(*args(fake, 48, 0.5)) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_attn_ctx(*args(fake, 64, 1.5)) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_attn_ctx(*args(fake, 64, 0.0)) == rmm.RMM_ERR_INVALID_ARG


def test_context_block_workspace_sizes(lib):
    from input_adaptive_reduced_rmm_b200 import rmm

    w1 = rmm.rmm_attn_ctx_workspace_bytes(1, 32, 8, 1, 4096, 64, 0.5)
    w2 = rmm.rmm_attn_ctx_workspace_bytes(1, 32, 8, 1, 65536, 64, 0.5)
    assert 0 < w1 <= w2
    assert rmm.rmm_attn_ctx_workspace_bytes(1, 32, 8, 1, 4096, 48, 0.5) == 0   # block size
    assert rmm.rmm_attn_ctx_workspace_bytes(1, 32, 8, 1, 4096, 64, 0.0) == 0   # r_ctx
    assert rmm.rmm_attn_ctx_workspace_bytes(1, 32, 8, 1, 4096, 64, 0.5, d=64) == 0


def test_option_fields_are_validated(lib):
    """Option values outside their ranges make every size query return 0 (and every call
    RMM_ERR_INVALID_ARG): a block score without blocks, unknown scores, paths and producers."""
    from input_adaptive_reduced_rmm_b200 import rmm

    assert rmm.rmm_linear_workspace_bytes(4, 1024, 1024, rmm.options(block_size=64, block_score=1)) > 0
    for bad in (rmm.options(block_score=1), rmm.options(block_size=64, block_score=2), rmm.options(attn_path=3),
                rmm.options(gemm_producer=3), rmm.options(block_size=-1)):
        assert rmm.rmm_linear_workspace_bytes(4, 1024, 1024, bad) == 0
