"""The workspace-free decode entry point, for callers that cannot allocate device memory.

rmm_linear_decode_noalloc keeps its scratch in a fixed array inside the library
instead of a caller workspace.  This test calls it through the C ABI twice in a
row for each case and checks kept sets and outputs against the workspace entry
point rmm_linear, within the float bar the other parity tests use.  It lives in
its own file, collected last, and passes alone or after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import rmm_synth
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from input_adaptive_reduced_rmm_b200 import rmm as _rmm

    _rmm.lib()
    return _rmm


@pytest.mark.parametrize("T,H,N,r", [(1, 4096, 14336, 0.5), (16, 512, 1024, 0.5), (5, 1000, 264, 0.25),
                                     (16, 4096, 14336, 0.75), (1, 28672, 8192, 0.125)])
def test_noalloc_matches_workspace_entry_point(rmm, T, H, N, r):
    X = rmm_synth.activations(T, H, rmm_synth.seed_for(5, T, 0)).cuda()
    Wt = rmm.rmm_transpose_weight(rmm_synth.weights(N, H, rmm_synth.seed_for(5, T, 1), std=0.02).cuda())
    k = rmm.rmm_k_for(H, r)
    idx_ref = torch.empty(k, dtype=torch.int32, device="cuda")
    Y_ref = rmm.rmm_linear(X, Wt, r, idx_out=idx_ref)
    torch.cuda.synchronize()
    ref = Y_ref.double().cpu().numpy()
    L = rmm.lib()
    for call in range(2):
        Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        idx = torch.full((k,), -1, dtype=torch.int32, device="cuda")
        rc = L.rmm_linear_decode_noalloc(rmm._ptr(X), rmm._ptr(Wt), T, H, N, ctypes.c_double(r), rmm._ptr(Y),
                                         rmm._ptr(idx), rmm._stream(None))
        assert rc == rmm.RMM_OK, rmm.rmm_status_string(rc)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy()), f"call {call}"
        assert_close(Y.cpu(), ref, f"noalloc call {call} T={T} H={H} N={N} r={r}")


def test_noalloc_rejects_sizes_beyond_its_limits(rmm):
    X = torch.zeros(17, 64, dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(17, 64, dtype=torch.bfloat16, device="cuda")
    L = rmm.lib()
    rc = L.rmm_linear_decode_noalloc(rmm._ptr(X), rmm._ptr(Wt), 17, 64, 64, ctypes.c_double(0.5), rmm._ptr(Y),
                                     None, rmm._stream(None))
    assert rc == rmm.RMM_ERR_UNSUPPORTED
