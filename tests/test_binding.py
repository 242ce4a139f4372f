"""The Python binding's own checks, on the CPU: tensors on the wrong device, of
the wrong dtype or of mismatched shapes are refused before the C ABI is called,
and the options struct carries every field the header declares, in order."""
import ctypes
import re

import pytest
import torch

from conftest import ROOT


@pytest.fixture(scope="module")
def rmm():
    from input_adaptive_reduced_rmm_b200 import build as b

    b.build()
    from input_adaptive_reduced_rmm_b200 import rmm as _rmm

    return _rmm


def test_host_tensors_are_refused(rmm):
    X = torch.zeros(4, 64, dtype=torch.bfloat16)
    Wt = torch.zeros(64, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rmm.rmm_linear(X, Wt, 0.5)
    with pytest.raises(ValueError):
        rmm.rmm_linear_group(X, [Wt], 0.5)
    Q = torch.zeros(1, 4, 1, 128, dtype=torch.bfloat16)
    Kt = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    V = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rmm.rmm_attn_qk(Q, Kt, V, 64, 0.5)
    with pytest.raises(ValueError):
        rmm.rmm_swiglu(X, X)


def test_wrong_dtype_is_refused(rmm):
    X = torch.zeros(4, 64, dtype=torch.float32)
    Wt = torch.zeros(64, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rmm.rmm_linear(X, Wt, 0.5)


def test_options_struct_matches_the_header(rmm):
    """Field names and order of rmm_options in include/rmm.h, against the ctypes mirror."""
    text = open(f"{ROOT}/include/rmm.h").read()
    body = re.search(r"typedef struct rmm_options \{(.*?)\} rmm_options;", text, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\b(\w+)\s*(?:\[\d+\])?\s*;", body)
    assert names == [f[0] for f in rmm.rmm_options._fields_]
    o = rmm.options(block_size=64, block_score=1, attn_path=2)
    assert (o.block_size, o.block_score, o.attn_path, o.t_gemv) == (64, 1, 2, 16)
    assert ctypes.sizeof(rmm.rmm_options) == 8 * 4 + 2 * ctypes.sizeof(ctypes.c_void_p)
