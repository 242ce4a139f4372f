"""Block-granular kept sets on the GPU against the oracle.

Kept slices must match the oracle's blocks (expanded to their slices) bit for
bit; the outputs meet the float bar on both product paths (GEMV for T <= 16,
the CTA-pair GEMM above).
"""
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


def expand(blocks, block):
    return (np.asarray(blocks)[:, None] * block + np.arange(block)[None, :]).reshape(-1)


def run_blocks(rmm, X, W, r, block, t_gemv=16, producer=0):
    T, H = X.shape
    N = W.shape[0]
    Wt = rmm.rmm_transpose_weight(W.cuda())
    kb = oracle.k_for(H // block, r)
    opts = rmm.options(block_size=block, t_gemv=t_gemv, gemm_producer=producer)
    idx = torch.full((kb * block,), -1, dtype=torch.int32, device="cuda")
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(T, H, N, opts))
    Y = rmm.rmm_linear(X.cuda(), Wt, r, idx_out=idx, workspace=ws, opts=opts)
    torch.cuda.synchronize()
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK
    return Y.cpu(), idx.cpu().numpy(), kb


@pytest.mark.parametrize("T,H,N,r,block", [
    (1, 512, 1024, 0.5, 64),
    (5, 1024, 264, 0.25, 64),
    (16, 1024, 512, 0.3, 32),
    (17, 512, 1024, 0.5, 64),     # first T on the GEMM path
    (300, 1024, 520, 0.75, 128),
    (64, 4096, 1024, 0.5, 64),
    (1, 4096, 14336, 0.5, 256),
    (40, 768, 1024, 1.0, 16),     # r = 1: every block, the dense product
])
def test_blocks_small(rmm, T, H, N, r, block):
    X = rmm_synth.activations(T, H, rmm_synth.seed_for(9, T, 1))
    W = rmm_synth.weights(N, H, rmm_synth.seed_for(9, T, 2), std=0.02)
    Y, idx, kb = run_blocks(rmm, X, W, r, block)
    Yo, blocks = oracle.linear_blocks(X, W, r, block=block)
    assert idx.tolist() == expand(blocks, block).tolist()
    assert_close(Y, Yo, f"T={T} H={H} N={N} r={r} block={block}")


@pytest.mark.parametrize("t_gemv", [16, 0])
def test_blocks_ties(rmm, t_gemv):
    """Tie-heavy activations: many blocks share their max; the lower block index wins."""
    T, H, N, block = 4, 1024, 256, 64
    X = rmm_synth.tie_heavy((T, H), 95)
    W = rmm_synth.weights(N, H, 96)
    Y, idx, kb = run_blocks(rmm, X, W, 0.5, block, t_gemv=t_gemv)
    Yo, blocks = oracle.linear_blocks(X, W, 0.5, block=block)
    assert idx.tolist() == expand(blocks, block).tolist()
    assert_close(Y, Yo, f"ties t_gemv={t_gemv}")


def test_blocks_llama3_8b_prefill_sampled(rmm):
    """T=2048, 4096 -> 14336, r=0.5, 64-wide blocks; output rows sampled."""
    T, H, N, r, block = 2048, 4096, 14336, 0.5, 64
    X = rmm_synth.activations(T, H, rmm_synth.seed_for(9, 77, 1))
    W = rmm_synth.weights(N, H, rmm_synth.seed_for(9, 77, 2), std=0.02)
    Y, idx, kb = run_blocks(rmm, X, W, r, block)
    rows = sample_indices(T, 48, seed=5)
    Yo, blocks = oracle.linear_blocks(X, W, r, block=block, rows=rows)
    assert idx.tolist() == expand(blocks, block).tolist()
    assert_close(Y[rows], Yo, "llama3-8b prefill blocks")


@pytest.mark.parametrize("producer", [0, 2])
@pytest.mark.parametrize("T,H,N,block", [(700, 1024, 1800, 64), (300, 2048, 776, 128), (2048, 512, 3000, 256)])
def test_blocks_tma_tiles(rmm, producer, T, H, N, block):
    """Blocks of 64 slices or more: the CTA-pair GEMM (0) loads whole 64-row runs by TMA
    tile copies; the single-CTA cp.async GEMM (2) gathers them row by row.  Ragged M and N
    edges, split last wave."""
    X = rmm_synth.activations(T, H, rmm_synth.seed_for(9, T, 3))
    W = rmm_synth.weights(N, H, rmm_synth.seed_for(9, T, 4), std=0.02)
    Y, idx, kb = run_blocks(rmm, X, W, 0.5, block, producer=producer)
    Yo, blocks = oracle.linear_blocks(X, W, 0.5, block=block)
    assert idx.tolist() == expand(blocks, block).tolist()
    assert_close(Y, Yo, f"T={T} H={H} N={N} block={block} producer={producer}")


def test_blocks_group_shares_one_set(rmm):
    T, H, block = 24, 1024, 64
    X = rmm_synth.activations(T, H, 97)
    Ws = [rmm_synth.weights(n, H, 98 + i, std=0.02) for i, n in enumerate((512, 128, 128))]
    opts = rmm.options(block_size=block)
    kb = oracle.k_for(H // block, 0.5)
    idx = torch.empty(kb * block, dtype=torch.int32, device="cuda")
    Ys = rmm.rmm_linear_group(X.cuda(), [rmm.rmm_transpose_weight(W.cuda()) for W in Ws], 0.5, idx_out=idx,
                              opts=opts)
    torch.cuda.synchronize()
    for W, Y in zip(Ws, Ys):
        Yo, blocks = oracle.linear_blocks(X, W, 0.5, block=block)
        assert idx.cpu().numpy().tolist() == expand(blocks, block).tolist()
        assert_close(Y.cpu(), Yo, "group member")


def test_blocks_reject_bad_sizes(rmm):
    X = torch.zeros(2, 1000, dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros(1000, 64, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(2, 64, dtype=torch.bfloat16, device="cuda")
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(2, 1000, 64))
    L = rmm.lib()
    for bs in (64, 48):  # 1000 % 64 != 0; 48 is not an allowed block size
        opts = rmm.options(block_size=bs)
        rc = L.rmm_linear(rmm._ptr(X), rmm._ptr(Wt), 2, 1000, 64, 0.5, rmm._ptr(Y), None, rmm._ptr(ws),
                          ws.numel(), rmm._stream(None), rmm.ctypes.byref(opts))
        assert rc == rmm.RMM_ERR_UNSUPPORTED


# ---------------------------------------------------------------- mean-magnitude blocks

def run_mean_blocks(rmm, X, W, r, block, t_gemv=16):
    T, H = X.shape
    N = W.shape[0]
    Wt = rmm.rmm_transpose_weight(W.cuda())
    kb = oracle.k_for(H // block, r)
    opts = rmm.options(block_size=block, block_score=1, t_gemv=t_gemv)
    idx = torch.full((kb * block,), -1, dtype=torch.int32, device="cuda")
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(T, H, N, opts))
    Y = rmm.rmm_linear(X.cuda(), Wt, r, idx_out=idx, workspace=ws, opts=opts)
    torch.cuda.synchronize()
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK
    return Y.cpu(), idx.cpu().numpy(), ws


@pytest.mark.parametrize("T,H,N,r,block,t_gemv", [
    (1, 4096, 1024, 0.5, 64, 16),    # the FFN demo's down projection
    (1, 512, 264, 0.3, 16, 16),
    (7, 1024, 520, 0.5, 128, 16),
    (16, 2048, 1024, 0.25, 256, 16),
    (5, 1024, 1032, 0.5, 64, 0),     # the GEMM path (score pass still writes X^T)
])
def test_blocks_mean_score(rmm, T, H, N, r, block, t_gemv):
    X = rmm_synth.activations(T, H, rmm_synth.seed_for(9, T, 5))
    W = rmm_synth.weights(N, H, rmm_synth.seed_for(9, T, 6), std=0.02)
    Y, idx, _ = run_mean_blocks(rmm, X, W, r, block, t_gemv)
    Yo, blocks = oracle.linear_blocks(X, W, r, block=block, block_score="mean")
    assert idx.tolist() == expand(blocks, block).tolist()
    assert_close(Y, Yo, f"mean blocks T={T} H={H} block={block}")


def test_blocks_mean_then_max_on_one_workspace(rmm):
    """A mean-score call leaves the workspace's score vector at zero for the next call."""
    T, H, N, block = 4, 1024, 256, 64
    X = rmm_synth.activations(T, H, 131)
    W = rmm_synth.weights(N, H, 132)
    Wt = rmm.rmm_transpose_weight(W.cuda())
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(T, H, N, rmm.options(block_size=block, t_gemv=0)))
    for score, t_gemv in ((1, 0), (0, 0), (1, 16), (0, 16)):
        opts = rmm.options(block_size=block, block_score=score, t_gemv=t_gemv)
        idx = torch.empty(8 * block, dtype=torch.int32, device="cuda")
        Y = rmm.rmm_linear(X.cuda(), Wt, 0.5, idx_out=idx, workspace=ws, opts=opts)
        torch.cuda.synchronize()
        Yo, blocks = oracle.linear_blocks(X, W, 0.5, block=block, block_score="mean" if score else "max")
        assert idx.cpu().numpy().tolist() == expand(blocks, block).tolist()
        assert_close(Y.cpu(), Yo, f"score={score} t_gemv={t_gemv}")


def test_blocks_mean_rejects_long_chunks(rmm):
    X = torch.zeros(17, 512, dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros(512, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rmm.RmmError):
        rmm.rmm_linear(X, Wt, 0.5, opts=rmm.options(block_size=64, block_score=1))
    with pytest.raises(rmm.RmmError):  # a block score needs blocks
        rmm.rmm_linear(X[:1].contiguous(), Wt, 0.5, opts=rmm.options(block_score=1))
