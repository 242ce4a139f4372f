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
    assert ctypes.sizeof(rmm.rmm_options) == 9 * 4 + 4 + 2 * ctypes.sizeof(ctypes.c_void_p)  # 4 bytes of padding
    assert rmm.options(swiglu_pair=True).swiglu_pair == 1


def test_wrong_sizes_are_refused_before_the_call(rmm):
    """A wrong-sized output or kept-list buffer would let a kernel write past its end:
    the binding names the mismatch instead of calling the library."""
    X = torch.zeros(4, 64, dtype=torch.bfloat16)
    Wt = torch.zeros(64, 32, dtype=torch.bfloat16)
    bad = [
        dict(Y=torch.zeros(4, 16, dtype=torch.bfloat16)),                  # Y not [T, N]
        dict(Y=torch.zeros(4, 32, dtype=torch.bfloat16), idx_out=torch.zeros(3, dtype=torch.int32)),  # k = 32
        dict(Y=torch.zeros(4, 32, dtype=torch.bfloat16), idx_out=torch.zeros(64, dtype=torch.int64)),
    ]
    for kw in bad:
        for fn in (rmm.rmm_linear, rmm.rmm_linear_decode_noalloc):
            with pytest.raises(ValueError):
                fn(X, Wt, 0.5, **kw)
    with pytest.raises(ValueError, match="disagree on H"):
        rmm.rmm_linear_decode_noalloc(X, torch.zeros(32, 32, dtype=torch.bfloat16), 0.5,
                                      torch.zeros(4, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="Y must be given"):
        rmm.rmm_linear_decode_noalloc(X, Wt, 0.5, None)
    with pytest.raises(ValueError, match="expected"):
        rmm.rmm_linear_group(X, [Wt, Wt], 0.5, Ys=[torch.zeros(4, 32, dtype=torch.bfloat16),
                                                 torch.zeros(4, 31, dtype=torch.bfloat16)])
    with pytest.raises(ValueError, match="at least 64"):
        rmm.rmm_score(X, s_out=torch.zeros(63, dtype=torch.int32))
    with pytest.raises(ValueError, match="at least 10"):
        rmm.rmm_select(torch.zeros(64, dtype=torch.int32), 10, idx_out=torch.zeros(9, dtype=torch.int32))
    with pytest.raises(ValueError, match="expected"):
        rmm.rmm_gemm_reduced(X, Wt, torch.zeros(8, dtype=torch.int32), Y=torch.zeros(4, 33, dtype=torch.bfloat16))
    Q = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    Kt = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    V = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="expected"):
        rmm.rmm_attn_qk(Q, Kt, V, 64, 0.5, O=torch.zeros(1, 4, 1, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="at least 128"):  # 1 batch x 2 sets x 64 kept dims
        rmm.rmm_attn_qk(Q, Kt, V, 64, 0.5, idx_out=torch.zeros(127, dtype=torch.int32))
    with pytest.raises(ValueError, match="expected"):
        rmm.rmm_attn_ctx(Q, Kt, V, torch.zeros(1, 2, 2, 128), 64, 0.5, 0.5, 16)  # needs 4 blocks of 16
    # the right sizes pass every structural check and stop at the device check
    with pytest.raises(ValueError, match="CUDA"):
        rmm.rmm_linear_decode_noalloc(X, Wt, 0.5, torch.zeros(4, 32, dtype=torch.bfloat16),
                                      idx_out=torch.zeros(32, dtype=torch.int32))
