"""GPU parity of the reduced attention (Q K^T reduced along the head dimension, then softmax . V).

Every call goes through the C ABI.  Kept head-dimension sets are compared bit
for bit with the oracle; outputs within the float bar of tests/parity.py.
The key cache is handed to the library d-major (K^T [B, Hkv, d, ldL]) with a
padded leading dimension; the oracle takes K in its natural [B, Hkv, L, d].
"""
import math

import numpy as np
import pytest
import torch

import oracle
import rmm_synth
from parity import assert_close, row_head_pairs, sample_indices, tile_rows

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
    """K, V [B, Hkv, L, d] (CPU) -> d-major K^T [B, Hkv, d, ldL] and V [B, Hkv, ldL, d] on the GPU."""
    B, Hkv, L, d = K.shape
    ldL = (L + pad - 1) // pad * pad
    Kt = torch.zeros(B, Hkv, d, ldL, dtype=torch.bfloat16)
    Kt[..., :L] = K.transpose(-1, -2)
    Vp = torch.zeros(B, Hkv, ldL, d, dtype=torch.bfloat16)
    Vp[:, :, :L] = V
    return Kt.cuda(), Vp.cuda()


def run_attn(rmm, Q, K, V, r, causal=True, per_head=False, opts=None):
    B, Hq, T, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    Kt, Vp = to_device_cache(K, V)
    k = rmm.rmm_k_for(d, r)
    nsets = Hq if per_head else Hkv
    idx = torch.full((B, nsets, k), -1, dtype=torch.int32, device="cuda")
    o = opts if opts is not None else rmm.options(attn_per_query_head=per_head)
    ws = rmm.new_workspace(rmm.rmm_attn_workspace_bytes(B, Hq, Hkv, T, L, d, o))
    O = rmm.rmm_attn_qk(Q.cuda(), Kt, Vp, L, r, causal=causal, idx_out=idx, workspace=ws, opts=o)
    torch.cuda.synchronize()
    assert rmm.rmm_get_status(ws) == rmm.RMM_OK
    return O.cpu(), idx.cpu().numpy(), k


@pytest.mark.parametrize("T,L", [(1, 37), (1, 1000), (2, 4100), (5, 5), (5, 300), (33, 2100), (64, 64)])
@pytest.mark.parametrize("r", [0.25, 0.5, 1.0])
@pytest.mark.parametrize("causal", [True, False])
def test_attention_small(rmm, T, L, r, causal):
    B, Hq, Hkv = 2, 8, 2
    seed = rmm_synth.seed_for(7, T, L % 10)
    Q = rmm_synth.normal((B, Hq, T, D), seed)
    K = rmm_synth.normal((B, Hkv, L, D), seed + 1)
    V = rmm_synth.normal((B, Hkv, L, D), seed + 2)
    O, idx, k = run_attn(rmm, Q, K, V, r, causal)
    Oo, io = oracle.attention(Q, K, V, k, causal=causal)
    assert np.array_equal(idx, io)
    assert_close(O, Oo, f"T={T} L={L} r={r} causal={causal}")


@pytest.mark.parametrize("T", [1, 7])
def test_attention_per_query_head(rmm, T):
    B, Hq, Hkv, L = 1, 12, 3, 513
    Q = rmm_synth.normal((B, Hq, T, D), 41)
    K = rmm_synth.normal((B, Hkv, L, D), 42)
    V = rmm_synth.normal((B, Hkv, L, D), 43)
    O, idx, k = run_attn(rmm, Q, K, V, 0.25, True, per_head=True)
    Oo, io = oracle.attention(Q, K, V, k, causal=True, per_query_head=True)
    assert np.array_equal(idx, io)
    assert_close(O, Oo, "per-query-head")


def test_attention_tie_heavy_queries(rmm):
    B, Hq, Hkv, T, L = 1, 4, 1, 3, 200
    Q = rmm_synth.tie_heavy((B, Hq, T, D), 5)
    K = rmm_synth.normal((B, Hkv, L, D), 6)
    V = rmm_synth.normal((B, Hkv, L, D), 7)
    O, idx, k = run_attn(rmm, Q, K, V, 0.5, True)
    Oo, io = oracle.attention(Q, K, V, k, causal=True)
    assert np.array_equal(idx, io)
    assert_close(O, Oo, "ties")


def oracle_kept_sets(Q, K, V, k):
    """The oracle's kept head-dimension sets for Q (per KV group): they depend on Q alone, so
    the oracle runs them against the cache's first T keys and computes one output row."""
    T = Q.shape[2]
    _, io = oracle.attention(Q, K[:, :, :T], V[:, :, :T], k, causal=True, t_rows=[0])
    return io


def check_pairs(O, Q, K, V, k, idx, pairs, what, causal=True):
    """O[b, h, t] against the oracle for each sampled (t, h), with the kept sets given (one
    oracle call per query head: that head and its KV group alone)."""
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    by_head = {}
    for t, h in pairs:
        by_head.setdefault(h, []).append(t)
    got, ref = [], []
    for h, rows in sorted(by_head.items()):
        g = h // G
        Oo, _ = oracle.attention(Q[:, h:h + 1].contiguous(), K[:, g:g + 1].contiguous(), V[:, g:g + 1].contiguous(),
                                 k, causal=causal, t_rows=rows, idx_in=idx[:, g:g + 1])
        got.append(O[:, h, rows].double().numpy())
        ref.append(Oo[:, 0])
    assert_close(np.concatenate(got, axis=1), np.concatenate(ref, axis=1), what)


def check_large(rmm, cfg, B, Hq, Hkv, T, L, r, heads_per_row=2, opts=None):
    """Kept sets in full; O on one query row of every 128-row query tile (plus the first and
    last rows), each on `heads_per_row` query heads spread over the KV groups."""
    seed = rmm_synth.seed_for(cfg, T % 100, L % 97)
    Q = rmm_synth.normal((B, Hq, T, D), seed)
    K = rmm_synth.normal((B, Hkv, L, D), seed + 1)
    V = rmm_synth.normal((B, Hkv, L, D), seed + 2)
    O, idx, k = run_attn(rmm, Q, K, V, r, True, opts=opts)
    assert np.array_equal(idx, oracle_kept_sets(Q, K, V, k)), "kept sets"
    rows = tile_rows(T, 128, seed=L + T)
    check_pairs(O, Q, K, V, k, idx, row_head_pairs(rows, Hq, Hkv, heads_per_row), f"cfg{cfg} T={T} L={L} r={r}")


@pytest.mark.parametrize("L", [4096, 16384, 32768])
@pytest.mark.parametrize("T", [1, 512])
@pytest.mark.parametrize("r", [0.25, 0.5])
def test_attention_llama3_8b(rmm, L, T, r):
    """Batch 1, 32 query / 8 KV heads, d = 128, decode and a prefill chunk of 512."""
    check_large(rmm, 2, 1, 32, 8, T, L, r, heads_per_row=8 if T == 1 else 2)


@pytest.mark.parametrize("r", [0.25, 0.5])
def test_attention_layer_prefill_shape(rmm, r):
    """The decoder layer's own prefill attention: T = L = 2048, causal, 32 query / 8 KV
    heads (16 query tiles per head on the tensor cores)."""
    check_large(rmm, 3, 1, 32, 8, 2048, 2048, r, heads_per_row=4)


@pytest.mark.parametrize("T", [1, 4096])
@pytest.mark.parametrize("r", [0.125, 0.25, 0.5, 1.0])
def test_attention_llama3_70b(rmm, T, r):
    """64 query / 8 KV heads, d = 128, KV length 65536; decode and a 4096-token chunk
    (32 query tiles per head) across the retention sweep."""
    check_large(rmm, 4, 1, 64, 8, T, 65536, r, heads_per_row=8 if T == 1 else 1)


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("B,T,L,r,causal,per_head", [
    (1, 16, 16, 0.5, True, False),      # one ragged query tile, one key block
    (2, 130, 300, 0.3, True, False),    # k = 39 (padded to 48 on the tensor cores), two query tiles
    (1, 200, 200, 0.25, False, False),  # non-causal, ragged tile
    (1, 129, 700, 1.0, True, True),     # all dims, per-query-head sets, chunk at the end of the cache
    (1, 256, 1000, 0.5, True, False),   # key blocks past the diagonal and a ragged last key block
])
def test_attention_both_paths(rmm, path, B, T, L, r, causal, per_head):
    """The tensor-core prefill kernel (path 2) and the CUDA-core split pass (path 1)
    against the oracle on the same inputs."""
    Hq, Hkv = 8, 2
    seed = rmm_synth.seed_for(7, T, 5)
    Q = rmm_synth.normal((B, Hq, T, D), seed)
    K = rmm_synth.normal((B, Hkv, L, D), seed + 1)
    V = rmm_synth.normal((B, Hkv, L, D), seed + 2)
    opts = rmm.options(attn_per_query_head=per_head, attn_path=path)
    O, idx, k = run_attn(rmm, Q, K, V, r, causal, per_head=per_head, opts=opts)
    rows = sample_indices(T, 24, seed=T)
    Oo, io = oracle.attention(Q, K, V, k, causal=causal, per_query_head=per_head, t_rows=rows)
    assert np.array_equal(idx, io)
    assert_close(O[:, :, rows], Oo, f"path={path} B={B} T={T} L={L} r={r} causal={causal}")


def test_attention_rejects_bad_head_dim(rmm):
    L = rmm.lib()
    Q = torch.zeros(1, 2, 1, 64, dtype=torch.bfloat16, device="cuda")
    Kt = torch.zeros(1, 1, 64, 16, dtype=torch.bfloat16, device="cuda")
    V = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    ws = rmm.new_workspace(4096)
    p = rmm._ptr
    rc = L.rmm_attn_qk(p(Q), p(Kt), p(V), 1, 2, 1, 1, 16, 16, 64, 0.5, 1, 1.0 / math.sqrt(64), p(Q), None,
                       p(ws), ws.numel(), rmm._stream(None), None)
    assert rc == rmm.RMM_ERR_UNSUPPORTED


def test_fma_exponential_meets_its_stated_bound(rmm):
    """The softmax's FMA-pipe 2^x against the exact value (fp64 on the host) over its whole
    input range [-126, 8]: relative error below the stated 6e-5, every integer exact, and
    the hardware 2^x (torch.exp2) within the same bound; below -126 it clamps to 2^-126."""
    g = torch.Generator().manual_seed(11)
    dense = torch.linspace(-126.0, 8.0, 1 << 20, dtype=torch.float64)
    rand = torch.rand(1 << 20, generator=g, dtype=torch.float64) * 134.0 - 126.0
    near = (torch.arange(-126, 9, dtype=torch.float64)[:, None] +
            torch.tensor([-0.5, -0.4999999, -1e-6, 0.0, 1e-6, 0.4999999, 0.5], dtype=torch.float64)[None, :]).reshape(-1)
    x = torch.cat([dense, rand, near]).clamp(-126.0, 8.0).to(torch.float32)
    y = rmm.rmm_selftest_exp2_fma(x.cuda())
    hw = torch.exp2(x.cuda())
    torch.cuda.synchronize()
    exact = torch.exp2(x.double())
    rel = ((y.cpu().double() - exact) / exact).abs()
    assert float(rel.max()) < 6e-5, f"max relative error {float(rel.max()):.3e}"
    ints = torch.arange(-126, 9, dtype=torch.float32)
    assert torch.equal(rmm.rmm_selftest_exp2_fma(ints.cuda()).cpu(), torch.exp2(ints.double()).float())
    assert float(((hw.cpu().double() - exact) / exact).abs().max()) < 6e-5
    low = rmm.rmm_selftest_exp2_fma(torch.tensor([-130.0, -1000.0, -126.0], device="cuda")).cpu()
    assert torch.equal(low, torch.full((3,), 2.0 ** -126))
