"""GPU parity of the reduced linear map (score, select, GEMV and tcgen05 GEMM) against the oracle.

Every call goes through the C ABI (librmm.so via the ctypes binding).  Kept
index sets are compared bit for bit; outputs within the float bar of
tests/parity.py.  Sizes span several tiles and ragged tails; the full
Llama-3-8B / 70B shapes are checked on sampled outputs.
"""
import numpy as np
import pytest
import torch

import oracle
import rmm_synth
from parity import assert_close, bits_u16, sample_indices, tile_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from input_adaptive_reduced_rmm_b200 import rmm as _rmm

    _rmm.lib()
    return _rmm


def run_linear(rmm, X, W, r, opts=None):
    """GPU path through the C ABI: transpose W once, then rmm_linear."""
    Xd, Wd = X.cuda(), W.cuda()
    Wt = rmm.rmm_transpose_weight(Wd)
    T, H = X.shape
    k = rmm.rmm_k_for(H, r)
    idx = torch.full((k,), -1, dtype=torch.int32, device="cuda")
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(T, H, W.shape[0], opts))
    Y = rmm.rmm_linear(Xd, Wt, r, idx_out=idx, workspace=ws, opts=opts)
    torch.cuda.synchronize()
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK
    return Y.cpu(), idx.cpu().numpy()


# ---------------------------------------------------------------- score / select

@pytest.mark.parametrize("T,H", [(1, 1), (1, 7), (3, 65), (16, 512), (17, 129), (64, 4096),
                                 (129, 1000), (2048, 4096), (5, 14336)])
@pytest.mark.parametrize("kind", ["normal", "ties"])
def test_score_bit_exact(rmm, T, H, kind):
    seed = rmm_synth.seed_for(9, T % 97, H % 7)
    X = rmm_synth.activations(T, H, seed) if kind == "normal" else rmm_synth.tie_heavy((T, H), seed)
    s = rmm.rmm_score(X.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().astype(np.uint32), oracle.score(X).astype(np.uint32))


@pytest.mark.parametrize("H", [1, 2, 7, 12, 64, 65, 127, 128, 129, 1000, 4096, 14336, 16384, 16385, 20001, 28672,
                               40961, 65535])
def test_select_bit_exact(rmm, H):
    """One CTA up to H = 16384, a cluster of CTAs above (16385: 8 slices of 2049 keys,
    the last one short; 20001 and 40961: ragged slices)."""
    rng = np.random.default_rng(H)
    for trial in range(3):
        if trial == 0:
            s = rng.integers(0, 0x7F80, size=H)
        elif trial == 1:
            s = rng.integers(0, 3, size=H)  # heavy ties
        else:
            s = rng.integers(0, 0x10000, size=H)  # full 16-bit keys
        s = s.astype(np.uint16)
        sd = torch.from_numpy(s.astype(np.int32)).cuda()
        for k in sorted({1, max(1, H // 3), max(1, H // 2), max(1, H - 1), H}):
            got = rmm.rmm_select(sd, k)
            torch.cuda.synchronize()
            assert np.array_equal(got.cpu().numpy(), oracle.select(s, k)), (H, k, trial)


# ---------------------------------------------------------------- small full-output sweep

@pytest.mark.parametrize("T", [1, 2, 3, 16, 17, 127, 128, 129])
@pytest.mark.parametrize("H,N", [(64, 8), (65, 200), (127, 1024), (512, 264)])
@pytest.mark.parametrize("r", [0.25, 0.5, 1.0])
def test_linear_small(rmm, T, H, N, r):
    seed = rmm_synth.seed_for(8, T, H % 10)
    X = rmm_synth.activations(T, H, seed)
    W = rmm_synth.weights(N, H, seed + 1)
    Y, idx = run_linear(rmm, X, W, r)
    Yo, io = oracle.linear(X, W, r)
    assert np.array_equal(idx, io)
    assert_close(Y, Yo, f"T={T} H={H} N={N} r={r}")


@pytest.mark.parametrize("T", [1, 5, 16, 33])
def test_linear_gemm_path_for_small_T(rmm, T):
    """t_gemv = 0 forces the tcgen05 GEMM for every T (one M tile, mostly zero-filled)."""
    X = rmm_synth.activations(T, 320, 77 + T)
    W = rmm_synth.weights(520, 320, 78 + T)
    Y, idx = run_linear(rmm, X, W, 0.5, rmm.options(t_gemv=0))
    Yo, io = oracle.linear(X, W, 0.5)
    assert np.array_equal(idx, io)
    assert_close(Y, Yo, f"gemm T={T}")


@pytest.mark.parametrize("producer", [0, 1, 2])
@pytest.mark.parametrize("T,H,N", [(300, 384, 776), (129, 1000, 520), (513, 256, 264), (1, 640, 1024)])
def test_gemm_producers(rmm, producer, T, H, N):
    """CTA-pair cp.async (0, default), single-CTA TMA gather4 (1), single-CTA cp.async (2)."""
    X = rmm_synth.activations(T, H, 300 + T)
    W = rmm_synth.weights(N, H, 301 + T)
    Y, idx = run_linear(rmm, X, W, 0.4, rmm.options(t_gemv=0, gemm_producer=producer))
    Yo, io = oracle.linear(X, W, 0.4)
    assert np.array_equal(idx, io)
    assert_close(Y, Yo, f"producer {producer} T={T} H={H} N={N}")


@pytest.mark.parametrize("producer", [0, 2])
@pytest.mark.parametrize("T,H,N,r", [(1000, 1024, 5000, 0.4), (2304, 512, 4608, 0.5)])
def test_gemm_pair_many_tiles(rmm, producer, T, H, N, r):
    """Several tiles per CTA (the accumulator reused tile after tile), a ragged last M
    tile and N tile, and a split last wave."""
    X = rmm_synth.activations(T, H, 310 + T)
    W = rmm_synth.weights(N, H, 311 + T)
    Y, idx = run_linear(rmm, X, W, r, rmm.options(gemm_producer=producer))
    Yo, io = oracle.linear(X, W, r)
    assert np.array_equal(idx, io)
    assert_close(Y, Yo, f"producer {producer} T={T} H={H} N={N}")


def test_linear_tie_heavy_inputs(rmm):
    X = rmm_synth.tie_heavy((40, 256), 5)
    W = rmm_synth.weights(128, 256, 6)
    for r in (0.1, 0.5, 0.9):
        for opts in (None, rmm.options(t_gemv=0)):
            Y, idx = run_linear(rmm, X, W, r, opts)
            Yo, io = oracle.linear(X, W, r)
            assert np.array_equal(idx, io)
            assert_close(Y, Yo, f"ties r={r}")


def test_linear_all_zero_input(rmm):
    X = torch.zeros(20, 96, dtype=torch.bfloat16)
    W = rmm_synth.weights(64, 96, 9)
    Y, idx = run_linear(rmm, X, W, 0.5)
    assert idx.tolist() == list(range(48))
    assert torch.count_nonzero(Y.float()) == 0


# ---------------------------------------------------------------- single linear of 16 x 512 -> 1024

@pytest.mark.parametrize("t_gemv", [16, 0])
def test_single_linear_16x512x1024(rmm, t_gemv):
    X = rmm_synth.activations(16, 512, rmm_synth.seed_for(0, 0, 0))
    W = rmm_synth.weights(1024, 512, rmm_synth.seed_for(0, 0, 1))  # std 1/sqrt(H)
    Y, idx = run_linear(rmm, X, W, 0.5, rmm.options(t_gemv=t_gemv))
    Yo, io = oracle.linear(X, W, 0.5)
    assert len(idx) == 256
    assert np.array_equal(idx, io)
    assert_close(Y, Yo, "16x512x1024")


# ---------------------------------------------------------------- Llama-3-8B / 70B projection shapes

_cache = {}


def _inputs(cfg, T, H, N):
    key = (cfg, T, H, N)
    if key not in _cache:
        if len(_cache) > 6:
            _cache.clear()
        X = rmm_synth.activations(T, H, rmm_synth.seed_for(cfg, T % 1000, 0))
        W = rmm_synth.weights(N, H, rmm_synth.seed_for(cfg, N % 1000, 1), std=0.02)
        _cache[key] = (X, W)
    return _cache[key]


def check_projection(rmm, cfg, T, H, N, r, nrows=12, ncols=384):
    """Kept set in full; Y on a row sample with one row in every 128-row M tile (and
    `nrows` more at random) and a column sample with one column in every 512-column N
    tile of the CTA-pair GEMM (and `ncols` more at random)."""
    X, W = _inputs(cfg, T, H, N)
    Y, idx = run_linear(rmm, X, W, r)
    k = oracle.k_for(H, r)
    io = oracle.select(oracle.score(X), k)
    assert np.array_equal(idx, io), "kept set differs"
    rows = np.union1d(sample_indices(T, nrows, seed=T + N), tile_rows(T, 128, seed=T))
    cols = np.union1d(sample_indices(N, ncols, seed=H + N), tile_rows(N, 512, seed=N))
    Yo = oracle.reduced_product(X, W, io, rows=rows, cols=cols)
    assert_close(Y[rows][:, cols], Yo, f"cfg{cfg} T={T} H={H} N={N} r={r}")


@pytest.mark.parametrize("H,N", [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)])
@pytest.mark.parametrize("T", [1, 16, 128, 2048])
@pytest.mark.parametrize("r", [0.25, 0.5, 0.75, 1.0])
def test_llama3_8b_projections(rmm, H, N, T, r):
    check_projection(rmm, 1, T, H, N, r)


@pytest.mark.parametrize("H,N", [(8192, 8192), (8192, 1024), (8192, 28672), (28672, 8192)])
@pytest.mark.parametrize("T", [1, 4096])
@pytest.mark.parametrize("r", [0.125, 0.25, 0.375, 0.5, 0.625, 0.75, 0.875, 1.0])
def test_llama3_70b_projections(rmm, H, N, T, r):
    check_projection(rmm, 4, T, H, N, r, nrows=8, ncols=256)


# ---------------------------------------------------------------- projections sharing one input

@pytest.mark.parametrize("T", [1, 16, 130, 2048])
def test_linear_group_shares_one_kept_set(rmm, T):
    """q, k, v of one layer (4096 -> 4096, 1024, 1024) in one grouped call."""
    H = 4096
    X = rmm_synth.activations(T, H, rmm_synth.seed_for(1, 90 + T % 100, 0))
    Ws = [rmm_synth.weights(N, H, rmm_synth.seed_for(1, 91 + i, 1), std=0.02) for i, N in enumerate((4096, 1024, 1024))]
    Wts = [rmm.rmm_transpose_weight(W.cuda()) for W in Ws]
    k = rmm.rmm_k_for(H, 0.5)
    idx = torch.empty(k, dtype=torch.int32, device="cuda")
    Ys = rmm.rmm_linear_group(X.cuda(), Wts, 0.5, idx_out=idx)
    torch.cuda.synchronize()
    io = oracle.select(oracle.score(X), k)
    assert np.array_equal(idx.cpu().numpy(), io)
    rows = sample_indices(T, 12, seed=T)
    for W, Y in zip(Ws, Ys):
        cols = sample_indices(W.shape[0], 256, seed=W.shape[0])
        Yo = oracle.reduced_product(X, W, io, rows=rows, cols=cols)
        assert_close(Y.cpu()[rows][:, cols], Yo, f"group T={T} N={W.shape[0]}")


# ---------------------------------------------------------------- product for a given kept list

@pytest.mark.parametrize("T", [4, 300])
def test_gemm_reduced_given_sets(rmm, T):
    H, N = 384, 776
    X = rmm_synth.activations(T, H, 123)
    W = rmm_synth.weights(N, H, 124)
    Wt = rmm.rmm_transpose_weight(W.cuda())
    rng = np.random.default_rng(7)
    perm = rng.permutation(H).astype(np.int32)
    kept, dropped = perm[:150], perm[150:]  # unsorted lists
    ys = []
    for sub in (kept, dropped):
        Y = rmm.rmm_gemm_reduced(X.cuda(), Wt, torch.from_numpy(sub).cuda())
        torch.cuda.synchronize()
        Yo = oracle.reduced_product(X, W, sub)
        assert_close(Y.cpu(), Yo, f"given set T={T}")
        ys.append(Y.cpu().double())
    full = X.double() @ W.double().T
    assert_close(ys[0] + ys[1], full.numpy(), "kept + dropped vs dense")


def test_transpose_weight(rmm):
    W = rmm_synth.weights(200, 136, 3)
    Wt = rmm.rmm_transpose_weight(W.cuda())
    torch.cuda.synchronize()
    assert torch.equal(Wt.cpu(), W.t().contiguous())


def test_deterministic_repeat(rmm):
    for T, opts in ((8, None), (300, None)):
        X = rmm_synth.activations(T, 2048, 31)
        W = rmm_synth.weights(3072, 2048, 32)
        Y1, i1 = run_linear(rmm, X, W, 0.5, opts)
        Y2, i2 = run_linear(rmm, X, W, 0.5, opts)
        assert np.array_equal(i1, i2)
        assert torch.equal(Y1, Y2)


# ---------------------------------------------------------------- errors and the watchdog

def test_invalid_arguments_are_rejected(rmm):
    X = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(4, 64, dtype=torch.bfloat16, device="cuda")
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(4, 64, 64))
    L = rmm.lib()
    s = rmm._stream(None)
    p = rmm._ptr
    assert L.rmm_linear(p(X), p(Wt), 4, 64, 64, 0.0, p(Y), None, p(ws), ws.numel(), s, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_linear(p(X), p(Wt), 4, 64, 64, 1.5, p(Y), None, p(ws), ws.numel(), s, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_linear(None, p(Wt), 4, 64, 64, 0.5, p(Y), None, p(ws), ws.numel(), s, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_linear(p(X), p(Wt), 4, 64, 60, 0.5, p(Y), None, p(ws), ws.numel(), s, None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_linear(p(X), p(Wt), 4, 64, 64, 0.5, p(Y), None, p(ws), 16, s, None) == rmm.RMM_ERR_WORKSPACE
    Xm = torch.zeros(4 * 64 + 1, dtype=torch.bfloat16, device="cuda")[1:]
    assert L.rmm_linear(p(Xm), p(Wt), 4, 64, 64, 0.5, p(Y), None, p(ws), ws.numel(), s, None) == rmm.RMM_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK


def test_watchdog_reports_timeout_and_context_survives(rmm):
    """The GEMM waits (50 ms limit) on a barrier nothing signals and reports RMM_ERR_TIMEOUT."""
    X = rmm_synth.activations(200, 256, 1)
    W = rmm_synth.weights(256, 256, 2)
    Xd = X.cuda()
    Wt = rmm.rmm_transpose_weight(W.cuda())
    opts = rmm.options(debug_timeout_test=True)
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(200, 256, 256, opts))
    rmm.rmm_linear(Xd, Wt, 0.5, workspace=ws, opts=opts)
    assert rmm.rmm_get_status(ws) == rmm.RMM_ERR_TIMEOUT
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK  # read-and-clear
    Y = rmm.rmm_linear(Xd, Wt, 0.5, workspace=ws)
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK
    Yo, _ = oracle.linear(X, W, 0.5)
    assert_close(Y.cpu(), Yo, "after watchdog")


# ---------------------------------------------------------------- gated-MLP epilogue

@pytest.mark.parametrize("T,r,splits", [(1, 1.0, 0), (1, 0.5, 0), (4, 0.5, 0), (16, 0.25, 0), (1, 0.5, 1),
                                        (40, 0.5, 0), (300, 1.0, 0)])
def test_swiglu_pair_epilogue_matches_the_two_steps(rmm, T, r, splits):
    """options.swiglu_pair on a gate/up group writes the same bits as the two products followed
    by rmm_swiglu: fused into the fold of the split-K GEMV (T <= 16), run after the products
    when the GEMV has one split (nothing to fold) and on the tensor-core GEMM path."""
    H, F = 1024, 3072
    X = rmm_synth.activations(T, H, rmm_synth.seed_for(1, 170 + T, 0)).cuda()
    Wg = rmm.rmm_transpose_weight(rmm_synth.weights(F, H, 171, std=0.02).cuda())
    Wu = rmm.rmm_transpose_weight(rmm_synth.weights(F, H, 172, std=0.02).cuda())
    g, u = rmm.rmm_linear_group(X, [Wg, Wu], r, opts=rmm.options(gemv_splits=splits))
    ref = rmm.rmm_swiglu(g, u)
    h = torch.full((T, F), float("nan"), dtype=torch.bfloat16, device="cuda")
    scratch = torch.empty(T, F, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(rmm.rmm_k_for(H, r), dtype=torch.int32, device="cuda")
    rmm.rmm_linear_group(X, [Wg, Wu], r, Ys=[h, scratch], idx_out=idx,
                         opts=rmm.options(gemv_splits=splits, swiglu_pair=True))
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), ref.view(torch.int16))
    assert np.array_equal(idx.cpu().numpy(), oracle.select(oracle.score(X.cpu()), rmm.rmm_k_for(H, r)))


def test_swiglu_pair_needs_a_pair_of_equal_widths(rmm):
    X = torch.zeros(1, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros(64, 32, dtype=torch.bfloat16, device="cuda")
    o = rmm.options(swiglu_pair=True)
    for Wts in ([W], [W, W2], [W, W, W]):
        with pytest.raises(rmm.RmmError):
            rmm.rmm_linear_group(X, Wts, 0.5, opts=o)
    with pytest.raises(rmm.RmmError):
        rmm.rmm_gemm_reduced(X, W, torch.arange(8, dtype=torch.int32, device="cuda"), opts=o)
