"""The workspace-free decode entry point, for callers that cannot allocate device memory.

Some callers may not allocate GPU memory themselves: a plugin inside a host
framework that owns every allocation and lends it only input and output
buffers, or a serving loop whose memory budget is fixed once it starts.
rmm_linear_decode_noalloc serves them by keeping its scratch in a fixed array
inside the library instead of a caller workspace.

Each case calls it through the C ABI twice in a row and checks, on both calls,
the kept set and the output against the workspace entry point rmm_linear and
against the oracle, within the float bar the other parity tests use; one case
goes through the Python binding instead.  The file is collected last and passes
alone or after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import rmm_synth
from parity import assert_close, sample_indices

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from input_adaptive_reduced_rmm_b200 import rmm as _rmm

    _rmm.lib()
    return _rmm


@pytest.mark.parametrize("T,H,N,r,via", [(1, 4096, 14336, 0.5, "abi"), (16, 512, 1024, 0.5, "abi"),
                                         (5, 1000, 264, 0.25, "abi"), (16, 4096, 14336, 0.75, "abi"),
                                         (1, 28672, 8192, 0.125, "abi"), (3, 4096, 1024, 0.5, "binding")])
def test_noalloc_matches_workspace_entry_point(rmm, T, H, N, r, via):
    Xh = rmm_synth.activations(T, H, rmm_synth.seed_for(5, T, 0))
    Wh = rmm_synth.weights(N, H, rmm_synth.seed_for(5, T, 1), std=0.02)
    X = Xh.cuda()
    Wt = rmm.rmm_transpose_weight(Wh.cuda())
    k = rmm.rmm_k_for(H, r)
    idx_ref = torch.empty(k, dtype=torch.int32, device="cuda")
    Y_ref = rmm.rmm_linear(X, Wt, r, idx_out=idx_ref)
    torch.cuda.synchronize()
    ref = Y_ref.double().cpu().numpy()
    # the oracle on a sample of output columns (every row; its kept set over the whole batch)
    cols = sample_indices(N, 256, seed=N + T)
    Y_or, idx_or = oracle.linear(Xh, Wh, r, cols=cols)
    assert np.array_equal(idx_ref.cpu().numpy(), idx_or)
    L = rmm.lib()
    for call in range(2):
        Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        idx = torch.full((k,), -1, dtype=torch.int32, device="cuda")
        if via == "abi":
            rc = L.rmm_linear_decode_noalloc(rmm._ptr(X), rmm._ptr(Wt), T, H, N, ctypes.c_double(r), rmm._ptr(Y),
                                             rmm._ptr(idx), rmm._stream(None))
            assert rc == rmm.RMM_OK, rmm.rmm_status_string(rc)
        else:
            rmm.rmm_linear_decode_noalloc(X, Wt, r, Y, idx_out=idx)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy()), f"call {call}"
        assert np.array_equal(idx.cpu().numpy(), idx_or), f"call {call} (oracle)"
        assert_close(Y.cpu(), ref, f"noalloc call {call} T={T} H={H} N={N} r={r}")
        assert_close(Y.cpu()[:, cols], Y_or, f"noalloc call {call} vs oracle T={T} H={H} N={N} r={r}")


def test_noalloc_rejects_sizes_beyond_its_limits(rmm):
    X = torch.zeros(17, 64, dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(17, 64, dtype=torch.bfloat16, device="cuda")
    L = rmm.lib()
    rc = L.rmm_linear_decode_noalloc(rmm._ptr(X), rmm._ptr(Wt), 17, 64, 64, ctypes.c_double(0.5), rmm._ptr(Y),
                                     None, rmm._stream(None))
    assert rc == rmm.RMM_ERR_UNSUPPORTED
