"""GPU parity of the context-block reduction of Q K^T (keys cut into blocks, a cheap
per-block score, attention over the kept blocks only).

Every call goes through the C ABI.  Block means and kept blocks are compared bit
for bit with the oracle (both sides compute the deciding score in single precision
in the same order); kept head dimensions bit for bit; outputs within the float bar
of tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import rmm_synth
from parity import assert_close

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module")
def rmm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from input_adaptive_reduced_rmm_b200 import rmm as _rmm

    _rmm.lib()
    return _rmm


def to_device_cache(K, V, pad=8):
    B, Hkv, L, d = K.shape
    ldL = (L + pad - 1) // pad * pad
    Kt = torch.zeros(B, Hkv, d, ldL, dtype=torch.bfloat16)
    Kt[..., :L] = K.transpose(-1, -2)
    Vp = torch.zeros(B, Hkv, ldL, d, dtype=torch.bfloat16)
    Vp[:, :, :L] = V
    return Kt.cuda(), Vp.cuda()


def run_ctx(rmm, Q, K, V, r, r_ctx, block, causal=True, per_head=False):
    B, Hq, T, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    Kt, Vp = to_device_cache(K, V)
    means = rmm.rmm_ctx_block_means(Kt, L, block)
    k = rmm.rmm_k_for(d, r)
    kc = rmm.rmm_k_for(rmm.ctx_num_blocks(L, block), r_ctx)
    nsets = Hq if per_head else Hkv
    idx = torch.full((B, nsets, k), -1, dtype=torch.int32, device="cuda")
    blocks = torch.full((B, nsets, kc), -1, dtype=torch.int32, device="cuda")
    o = rmm.options(attn_per_query_head=per_head)
    ws = rmm.new_workspace(rmm.rmm_attn_ctx_workspace_bytes(B, Hq, Hkv, T, L, block, r_ctx, d, o))
    O = rmm.rmm_attn_ctx(Q.cuda(), Kt, Vp, means, L, r, r_ctx, block, causal=causal, idx_out=idx,
                         blocks_out=blocks, workspace=ws, opts=o)
    torch.cuda.synchronize()
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK
    return O.cpu(), idx.cpu().numpy(), blocks.cpu().numpy(), k, kc, means


@pytest.mark.parametrize("L,block", [(64, 64), (1000, 64), (4096, 32), (3000, 128), (5000, 256), (131, 64)])
def test_block_means_bit_exact(rmm, L, block):
    B, Hkv = 2, 3
    K = rmm_synth.normal((B, Hkv, L, D), rmm_synth.seed_for(11, L, 1))
    Kt, _ = to_device_cache(K, K)
    means = rmm.rmm_ctx_block_means(Kt, L, block)
    torch.cuda.synchronize()
    ref = oracle.ctx_block_means(K, block)
    nblk = ref.shape[2]
    assert np.array_equal(means.cpu().numpy()[:, :, :nblk], ref)


def test_block_means_refresh_of_the_last_block(rmm):
    """After keys are appended, refreshing only the blocks they landed in matches the
    oracle's means of the grown cache; the other blocks are left as they were."""
    B, Hkv, L0, L1, block, ldL = 1, 2, 700, 777, 64, 800
    K = rmm_synth.normal((B, Hkv, L1, D), 12)
    Kt = torch.zeros(B, Hkv, D, ldL, dtype=torch.bfloat16)
    Kt[..., :L0] = K[:, :, :L0].transpose(-1, -2)
    Kt = Kt.cuda()
    means = rmm.rmm_ctx_block_means(Kt, L0, block)
    Kt[..., L0:L1] = K[:, :, L0:L1].transpose(-1, -2).cuda()
    first = L0 // block
    rmm.rmm_ctx_block_means(Kt, L1, block, means=means, blk_begin=first, blk_end=rmm.ctx_num_blocks(L1, block))
    torch.cuda.synchronize()
    ref = oracle.ctx_block_means(K, block)
    assert np.array_equal(means.cpu().numpy()[:, :, :ref.shape[2]], ref)


@pytest.mark.parametrize("L", [4096, 16384, 32768])
@pytest.mark.parametrize("r,r_ctx", [(0.25, 0.25), (0.5, 0.5), (0.5, 0.25)])
def test_ctx_decode_llama_shapes(rmm, L, r, r_ctx):
    """Decode (T = 1), Hq = 32, Hkv = 8, d = 128, 64-key blocks: the long-context cases."""
    B, Hq, Hkv, T, block = 1, 32, 8, 1, 64
    seed = rmm_synth.seed_for(12, L, int(4 * r + 16 * r_ctx))
    Q = rmm_synth.normal((B, Hq, T, D), seed)
    K = rmm_synth.normal((B, Hkv, L, D), seed + 1)
    V = rmm_synth.normal((B, Hkv, L, D), seed + 2)
    O, idx, blocks, k, kc, _ = run_ctx(rmm, Q, K, V, r, r_ctx, block)
    Oo, io, bo = oracle.attention_ctx(Q, K, V, k, block, kc, causal=True)
    assert np.array_equal(idx, io)
    assert np.array_equal(blocks, bo)
    assert_close(O, Oo, f"L={L} r={r} r_ctx={r_ctx}")


@pytest.mark.parametrize("T,L,block,r_ctx,causal", [
    (1, 37, 32, 0.5, True),       # one ragged block pair
    (5, 1000, 64, 0.3, True),     # causal chunk, ragged last block
    (16, 2000, 128, 0.5, True),   # the longest chunk the call takes
    (3, 777, 256, 0.75, False),
    (2, 65, 64, 0.5, True),       # the kept block may be the ragged one of one key
])
@pytest.mark.parametrize("per_head", [False, True])
def test_ctx_chunks_and_sets(rmm, T, L, block, r_ctx, causal, per_head):
    B, Hq, Hkv = 2, 8, 2
    seed = rmm_synth.seed_for(13, T, L % 97)
    Q = rmm_synth.normal((B, Hq, T, D), seed)
    K = rmm_synth.normal((B, Hkv, L, D), seed + 1)
    V = rmm_synth.normal((B, Hkv, L, D), seed + 2)
    O, idx, blocks, k, kc, _ = run_ctx(rmm, Q, K, V, 0.5, r_ctx, block, causal, per_head)
    Oo, io, bo = oracle.attention_ctx(Q, K, V, k, block, kc, causal=causal, per_query_head=per_head)
    assert np.array_equal(idx, io)
    assert np.array_equal(blocks, bo)
    assert_close(O, Oo, f"T={T} L={L} block={block} r_ctx={r_ctx} per_head={per_head}")


def test_ctx_all_blocks_equals_head_dim_reduction(rmm):
    """r_ctx = 1 keeps every block: the result is rmm_attn_qk's."""
    B, Hq, Hkv, T, L = 1, 8, 2, 3, 900
    Q = rmm_synth.normal((B, Hq, T, D), 14)
    K = rmm_synth.normal((B, Hkv, L, D), 15)
    V = rmm_synth.normal((B, Hkv, L, D), 16)
    O, idx, blocks, k, kc, _ = run_ctx(rmm, Q, K, V, 0.5, 1.0, 64)
    assert np.array_equal(blocks, np.tile(np.arange(15, dtype=np.int32), (1, 2, 1)))
    Oa, ia = oracle.attention(Q, K, V, k, causal=True)
    assert np.array_equal(idx, ia)
    assert_close(O, Oa, "r_ctx = 1")
    Kt, Vp = to_device_cache(K, V)
    Oq = rmm.rmm_attn_qk(Q.cuda(), Kt, Vp, L, 0.5, opts=rmm.options(attn_path=1)).cpu()
    assert torch.allclose(O.float(), Oq.float(), rtol=1e-2, atol=1e-2)


def test_ctx_row_without_kept_keys_is_zero(rmm):
    """Causal chunk whose first query precedes every kept key: that row is zero."""
    B, Hq, Hkv, T, L, block = 1, 1, 1, 3, 130, 64
    Q = rmm_synth.normal((B, Hq, T, D), 17)
    K = rmm_synth.normal((B, Hkv, L, D), 18) * 0.01
    K[0, 0, 128:130] = (Q[0, 0, 2] * 8).to(torch.bfloat16)  # the ragged block 2 wins the score
    V = rmm_synth.normal((B, Hkv, L, D), 19)
    O, idx, blocks, k, kc, _ = run_ctx(rmm, Q, K, V, 1.0, 0.25, block)  # kc = 1
    Oo, io, bo = oracle.attention_ctx(Q, K, V, k, block, kc, causal=True)
    assert blocks.tolist() == bo.tolist() == [[[2]]]
    assert torch.all(O[0, 0, 0] == 0)
    assert_close(O, Oo, "unseen row")


def test_ctx_rejects_unsupported(rmm):
    B, Hq, Hkv, L, block = 1, 4, 1, 256, 64
    Q = torch.zeros(B, Hq, 17, D, dtype=torch.bfloat16, device="cuda")
    Kt = torch.zeros(B, Hkv, D, L, dtype=torch.bfloat16, device="cuda")
    V = torch.zeros(B, Hkv, L, D, dtype=torch.bfloat16, device="cuda")
    means = rmm.new_ctx_means(Kt, block)
    with pytest.raises(rmm.RmmError):
        rmm.rmm_attn_ctx(Q, Kt, V, means, L, 0.5, 0.5, block)  # T = 17 > 16
    Q1 = torch.zeros(B, Hq, 1, D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rmm.RmmError):  # block 48 (the means buffer sized for it)
        rmm.rmm_attn_ctx(Q1, Kt, V, rmm.new_ctx_means(Kt, 48), L, 0.5, 0.5, 48)
    with pytest.raises(rmm.RmmError):
        rmm.rmm_ctx_block_means(Kt, L, block, blk_begin=3, blk_end=5)  # past ceil(L / block)


@pytest.mark.parametrize("L,block,r_ctx", [(65536, 32, 0.125), (4000, 256, 0.5), (65535, 64, 0.5)])
def test_ctx_large_block_counts(rmm, L, block, r_ctx):
    """2048 blocks of 32 keys (the most the block select sorts), a ragged 256-key last
    block, and a ragged cache just under 64K keys."""
    B, Hq, Hkv, T = 1, 4, 1, 1
    seed = rmm_synth.seed_for(14, L % 1000, block)
    Q = rmm_synth.normal((B, Hq, T, D), seed)
    K = rmm_synth.normal((B, Hkv, L, D), seed + 1)
    V = rmm_synth.normal((B, Hkv, L, D), seed + 2)
    O, idx, blocks, k, kc, _ = run_ctx(rmm, Q, K, V, 0.5, r_ctx, block)
    Oo, io, bo = oracle.attention_ctx(Q, K, V, k, block, kc, causal=True)
    assert np.array_equal(idx, io)
    assert np.array_equal(blocks, bo)
    assert_close(O, Oo, f"L={L} block={block} r_ctx={r_ctx}")
