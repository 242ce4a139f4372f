"""Pins of the CPU oracle against facts the method and the mathematics fix.

Nothing here compares the oracle with itself or retypes its formulas: every
check goes through another route -- hand-worked golden fixtures, exhaustive
brute force over all subsets, library dense products and library softmax
attention (numpy), exact algebraic identities.  Each plausible mistake (a
floor for the ceil, the wrong tie rule, a transposed weight, a dropped
scale, an off-by-one causal mask, the wrong GQA group) fails at least one.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import rmm_synth
from input_adaptive_reduced_rmm_b200 import metrics


def f64(t):
    return t.to(torch.float64).numpy()


def key_to_float(keys):
    """bf16 magnitude keys (sign cleared) back to their float values."""
    k = np.asarray(keys, dtype=np.uint16).astype(np.uint32) << 16
    return k.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- k = ceil(r H)

def test_k_for_golden(golden):
    g = golden("k_for.json")
    for H, r, k in g["cases"]:
        assert oracle.k_for(H, r) == k, (H, r)
        assert metrics.k_for(H, r) == k, (H, r)
    for H, r in g["rejected"]:
        assert oracle.k_for(H, r) == -1


def test_flop_formula_golden(golden):
    g = golden("flops_gemm_example.json")
    f = metrics.gemm_flops(g["m"], g["n"], g["k"])
    assert f == g["flops_exact"]
    assert abs(f - g["flops_quoted_approx"]) / g["flops_quoted_approx"] < 1e-3


# ---------------------------------------------------------------- score

def test_score_matches_float_brute_force():
    X = rmm_synth.activations(9, 37, seed=11)
    xs = X.to(torch.float64).tolist()
    want = [max(abs(xs[t][h]) for t in range(9)) for h in range(37)]
    got = key_to_float(oracle.score(X))
    assert got.tolist() == want


def test_score_signed_zero_and_ties():
    X = rmm_synth.tie_heavy((5, 64), seed=3)
    xs = X.to(torch.float64).tolist()
    want = [max(abs(xs[t][h]) for t in range(5)) for h in range(64)]
    assert key_to_float(oracle.score(X)).tolist() == want
    z = torch.tensor([[-0.0, 0.0, -0.0]], dtype=torch.bfloat16)
    assert oracle.score(z).tolist() == [0, 0, 0]


def test_score_rejects_nonfinite():
    X = torch.tensor([[1.0, float("inf")]], dtype=torch.bfloat16)
    with pytest.raises(oracle.OracleError):
        oracle.score(X)


# ---------------------------------------------------------------- select

def brute_force_kept_set(scores, k):
    """The unique k-subset whose every member beats every non-member under (score desc, index asc)."""
    H = len(scores)
    found = []
    for sub in itertools.combinations(range(H), k):
        inside = set(sub)
        ok = True
        for a in inside:
            for b in range(H):
                if b in inside:
                    continue
                # a must beat b: larger score, or equal score and lower index
                if not (scores[a] > scores[b] or (scores[a] == scores[b] and a < b)):
                    ok = False
                    break
            if not ok:
                break
        if ok:
            found.append(list(sub))
    assert len(found) == 1, found
    return found[0]


@pytest.mark.parametrize("H", [1, 2, 3, 5, 7, 8, 10, 12])
def test_select_brute_force(H):
    rng = np.random.default_rng(H)
    for trial in range(4):
        if trial % 2 == 0:
            s = rng.integers(0, 4, size=H).astype(np.uint16)  # heavy ties
        else:
            s = rng.integers(0, 0x7F80, size=H).astype(np.uint16)
        for k in range(1, H + 1):
            assert oracle.select(s, k).tolist() == brute_force_kept_set(s.tolist(), k)


def test_select_nested_over_r():
    X = rmm_synth.activations(4, 300, seed=5)
    s = oracle.score(X)
    prev = set()
    for k in range(1, 301):
        cur = set(oracle.select(s, k).tolist())
        assert prev < cur and len(cur) == k
        prev = cur


def test_select_all_zero_and_dominant():
    s = np.zeros(50, dtype=np.uint16)
    for k in (1, 7, 50):
        assert oracle.select(s, k).tolist() == list(range(k))
    s[33] = 0x4000
    assert oracle.select(s, 1).tolist() == [33]
    assert oracle.select(s, 3).tolist() == [0, 1, 33]


def test_select_output_ascending_and_size():
    X = rmm_synth.activations(3, 777, seed=8)
    s = oracle.score(X)
    for r in (0.125, 0.5, 0.9, 1.0):
        k = oracle.k_for(777, r)
        idx = oracle.select(s, k)
        assert len(idx) == k == math.ceil(r * 777)
        assert np.all(np.diff(idx) > 0)


# ---------------------------------------------------------------- reduced product

def test_tiny_linear_golden(golden):
    g = golden("tiny_linear.json")
    X = torch.tensor(g["X"], dtype=torch.bfloat16)
    W = torch.tensor(g["W"], dtype=torch.bfloat16)
    for case in g["cases"]:
        Y, idx = oracle.linear(X, W, case["r"])
        assert idx.tolist() == case["idx"]
        assert Y.tolist() == case["Y"]
    t = g["ties"]
    Xt = torch.tensor(t["X"], dtype=torch.bfloat16)
    _, idx = oracle.linear(Xt, W, t["r"])
    assert idx.tolist() == t["idx"]


def test_r1_equals_library_dense_product():
    X = rmm_synth.activations(13, 96, seed=21)
    W = rmm_synth.weights(40, 96, seed=22)
    Y, idx = oracle.linear(X, W, 1.0)
    assert idx.tolist() == list(range(96))
    ref = f64(X) @ f64(W).T
    assert np.max(np.abs(Y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_kept_plus_dropped_is_full():
    X = rmm_synth.activations(7, 130, seed=31)
    W = rmm_synth.weights(33, 130, seed=32)
    Yk, idx = oracle.linear(X, W, 0.4)
    drop = np.setdiff1d(np.arange(130), idx).astype(np.int32)
    Yd = oracle.reduced_product(X, W, drop)
    full = f64(X) @ f64(W).T
    assert np.max(np.abs(Yk + Yd - full)) <= 1e-12 * np.max(np.abs(full))
    # the kept set alone equals the library product of the gathered operands
    ref = f64(X)[:, idx] @ f64(W)[:, idx].T
    assert np.max(np.abs(Yk - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_exact_scaling_and_row_subset():
    X = rmm_synth.activations(6, 64, seed=41)
    W = rmm_synth.weights(20, 64, seed=42)
    Y, idx = oracle.linear(X, W, 0.5)
    Y2, idx2 = oracle.linear((X.float() * 2).to(torch.bfloat16), W, 0.5)
    assert idx.tolist() == idx2.tolist()
    assert np.array_equal(Y2, 2 * Y)
    rows = [5, 0, 3]
    Ys, _ = oracle.linear(X, W, 0.5, rows=rows)
    assert np.array_equal(Ys, Y[rows])


def test_outlier_channels_are_kept():
    # the 2 % outlier columns (x20) dominate the max-magnitude score
    X = rmm_synth.activations(32, 512, seed=0)
    _, idx = oracle.linear(X, rmm_synth.weights(8, 512, seed=1), 0.5)
    xs = f64(X)
    colmax = np.abs(xs).max(axis=0)
    top10 = np.argsort(-colmax, kind="stable")[:10]
    assert set(top10.tolist()) <= set(idx.tolist())


# ---------------------------------------------------------------- attention

def numpy_attention(q, K, V, scale, causal):
    """Library softmax attention for one head: q [T,d], K/V [L,d]."""
    T, L = q.shape[0], K.shape[0]
    logits = scale * (q @ K.T)
    if causal:
        pos = np.arange(T)[:, None] + (L - T)
        logits = np.where(np.arange(L)[None, :] <= pos, logits, -np.inf)
    logits = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ V


def test_attention_golden(golden):
    g = golden("tiny_attention.json")
    Q = torch.tensor(g["Q"], dtype=torch.bfloat16).reshape(1, 1, 1, 4)
    K = torch.tensor(g["K"], dtype=torch.bfloat16).reshape(1, 1, 2, 4)
    V = torch.tensor(g["V"], dtype=torch.bfloat16).reshape(1, 1, 2, 4)
    O, idx = oracle.attention(Q, K, V, g["k"], causal=True, scale=1.0)
    assert idx.reshape(-1).tolist() == g["idx"]
    assert np.allclose(O.reshape(-1), g["O_reduced"], rtol=0, atol=1e-15)
    O4, _ = oracle.attention(Q, K, V, 4, causal=True, scale=1.0)
    assert np.allclose(O4.reshape(-1), g["O_full"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("T,L,causal", [(1, 37, True), (5, 23, True), (4, 19, False)])
def test_attention_equals_library_attention_on_masked_q(T, L, causal, per_head):
    B, Hq, Hkv, d, k = 2, 6, 2, 16, 6
    Q = rmm_synth.normal((B, Hq, T, d), seed=51)
    K = rmm_synth.normal((B, Hkv, L, d), seed=52)
    V = rmm_synth.normal((B, Hkv, L, d), seed=53)
    scale = 1.0 / math.sqrt(d)
    O, idx = oracle.attention(Q, K, V, k, causal=causal, scale=scale, per_query_head=per_head)
    q, Kf, Vf = f64(Q), f64(K), f64(V)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            g = h // G
            heads = [h] if per_head else list(range(g * G, (g + 1) * G))
            s = np.abs(q[b, heads]).max(axis=(0, 1))
            order = np.lexsort((np.arange(d), -s))  # score desc, index asc
            S = np.sort(order[:k])
            assert idx[b, h if per_head else g].tolist() == S.tolist()
            qm = np.zeros_like(q[b, h])
            qm[:, S] = q[b, h][:, S]
            ref = numpy_attention(qm, Kf[b, g], Vf[b, g], scale, causal)
            assert np.max(np.abs(O[b, h] - ref)) <= 1e-12


def test_attention_given_sets_are_followed():
    """With kept sets supplied (not the top-k of Q), the oracle equals library
    attention on Q masked to those dimensions; supplying its own selection
    reproduces its own result."""
    B, Hq, Hkv, T, L, d, k = 1, 4, 2, 3, 13, 16, 5
    Q = rmm_synth.normal((B, Hq, T, d), seed=71)
    K = rmm_synth.normal((B, Hkv, L, d), seed=72)
    V = rmm_synth.normal((B, Hkv, L, d), seed=73)
    scale = 1.0 / math.sqrt(d)
    rng = np.random.default_rng(74)
    given = np.stack([np.sort(rng.choice(d, k, replace=False)) for _ in range(Hkv)]).astype(np.int32)[None]
    O, idx = oracle.attention(Q, K, V, k, causal=True, scale=scale, idx_in=given)
    assert np.array_equal(idx, given)
    q, Kf, Vf = f64(Q), f64(K), f64(V)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        qm = np.zeros_like(q[0, h])
        qm[:, given[0, g]] = q[0, h][:, given[0, g]]
        ref = numpy_attention(qm, Kf[0, g], Vf[0, g], scale, True)
        assert np.max(np.abs(O[0, h] - ref)) <= 1e-12
    O_own, idx_own = oracle.attention(Q, K, V, k, causal=True, scale=scale)
    O_again, _ = oracle.attention(Q, K, V, k, causal=True, scale=scale, idx_in=idx_own)
    assert np.array_equal(O_own, O_again)


def test_attention_full_head_dim_is_standard_attention():
    B, Hq, Hkv, T, L, d = 1, 4, 1, 3, 11, 8
    Q = rmm_synth.normal((B, Hq, T, d), seed=61)
    K = rmm_synth.normal((B, Hkv, L, d), seed=62)
    V = rmm_synth.normal((B, Hkv, L, d), seed=63)
    O, _ = oracle.attention(Q, K, V, d, causal=True)
    for h in range(Hq):
        ref = numpy_attention(f64(Q)[0, h], f64(K)[0, 0], f64(V)[0, 0], 1 / math.sqrt(d), True)
        assert np.max(np.abs(O[0, h] - ref)) <= 1e-12


def test_attention_decode_mask_is_noop_and_rows_subset():
    Q = rmm_synth.normal((1, 4, 1, 16), seed=71)
    K = rmm_synth.normal((1, 2, 29, 16), seed=72)
    V = rmm_synth.normal((1, 2, 29, 16), seed=73)
    Oc, ic = oracle.attention(Q, K, V, 8, causal=True)
    On, inn = oracle.attention(Q, K, V, 8, causal=False)
    assert np.array_equal(Oc, On) and np.array_equal(ic, inn)
    Q5 = rmm_synth.normal((1, 4, 5, 16), seed=74)
    Of, _ = oracle.attention(Q5, K, V, 8, causal=True)
    Os, _ = oracle.attention(Q5, K, V, 8, causal=True, t_rows=[4, 1])
    assert np.array_equal(Os, Of[:, :, [4, 1]])


# ---------------------------------------------------------------- layer glue

def test_rmsnorm_closed_form():
    x = torch.full((2, 8), 2.0, dtype=torch.bfloat16)
    x[1] = -0.5
    y = oracle.rmsnorm(x, eps=1e-5)
    assert np.allclose(y[0], 2.0 / math.sqrt(4.0 + 1e-5), rtol=0, atol=1e-15)
    assert np.allclose(y[1], -0.5 / math.sqrt(0.25 + 1e-5), rtol=0, atol=1e-15)


def test_swiglu_closed_form():
    g = torch.tensor([0.0, 1.0, -2.0, 3.0], dtype=torch.bfloat16)
    u = torch.tensor([5.0, 2.0, 1.0, -1.0], dtype=torch.bfloat16)
    out = oracle.swiglu(g, u)
    want = [0.0, 2.0 / (1 + math.exp(-1.0)), -2.0 / (1 + math.exp(2.0)), -3.0 / (1 + math.exp(-3.0))]
    assert np.allclose(out, want, rtol=0, atol=1e-15)


def test_row_and_column_subsets():
    X = rmm_synth.activations(9, 70, seed=81)
    W = rmm_synth.weights(30, 70, seed=82)
    Y, idx = oracle.linear(X, W, 0.3)
    rows, cols = [8, 2, 5], [29, 0, 13, 7]
    Ys, idx2 = oracle.linear(X, W, 0.3, rows=rows, cols=cols)
    assert idx.tolist() == idx2.tolist()
    assert np.array_equal(Ys, Y[np.ix_(rows, cols)])


# ---------------------------------------------------------------- block-granular kept sets

def test_block_select_with_unit_blocks_is_the_slice_select():
    s = rmm_synth.tie_heavy((97,), 81).view(torch.int16).numpy().view(np.uint16) & 0x7FFF
    for k in (1, 13, 50, 97):
        assert oracle.block_select(s, 1, k).tolist() == oracle.select(s, k).tolist()


@pytest.mark.parametrize("block,nb", [(4, 6), (3, 7)])
def test_block_select_brute_force(block, nb):
    """The kept blocks are the unique subset of size kb in which every kept block beats
    every dropped one under (block max desc, block index asc) -- checked over all subsets."""
    rng = np.random.default_rng(82 + block)
    s = rng.integers(0, 6, size=block * nb).astype(np.uint16)  # few values: many ties
    bmax = s.reshape(nb, block).max(axis=1).astype(np.int64)
    for kb in range(1, nb + 1):
        got = oracle.block_select(s, block, kb).tolist()
        valid = []
        for sub in itertools.combinations(range(nb), kb):
            kept, dropped = set(sub), set(range(nb)) - set(sub)
            if all((bmax[a] > bmax[d]) or (bmax[a] == bmax[d] and a < d) for a in kept for d in dropped):
                valid.append(list(sub))
        assert valid == [got]


def test_block_select_nested_over_kb():
    s = rmm_synth.activations(9, 640, 83)
    sc = oracle.score(s)
    prev = set()
    for kb in range(1, 11):
        cur = set(oracle.block_select(sc, 64, kb).tolist())
        assert prev <= cur and len(cur) == kb
        prev = cur


def test_linear_blocks_full_ratio_is_the_dense_product():
    X = rmm_synth.activations(5, 256, 84)
    W = rmm_synth.weights(40, 256, 85)
    Y, blocks = oracle.linear_blocks(X, W, 1.0, block=64)
    assert blocks.tolist() == [0, 1, 2, 3]
    assert np.allclose(Y, f64(X) @ f64(W).T, rtol=0, atol=1e-12)


def test_linear_blocks_keeps_the_outlier_block_and_splits_the_product():
    """A single large value makes its block the best one; kept plus dropped blocks
    sum to the dense product."""
    T, H, N = 3, 512, 24
    X = (rmm_synth.normal((T, H), 86) * 0.01).to(torch.bfloat16)
    X[1, 5 * 64 + 17] = 40.0
    W = rmm_synth.weights(N, H, 87)
    Y, blocks = oracle.linear_blocks(X, W, 1 / 8, block=64)
    assert blocks.tolist() == [5]
    dropped = np.array([j for j in range(H) if j // 64 != 5], dtype=np.int32)
    Yd = oracle.reduced_product(X, W, dropped)
    assert np.allclose(Y + Yd, f64(X) @ f64(W).T, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- context blocks
# cf-1.com post §3.1: keys cut into blocks of consecutive positions, a cheap
# per-block score (here: the best dot product of a query row with the block's
# mean key), Q K^T on the kept blocks only.


def small_ints(shape, lo, hi, seed):
    g = np.random.default_rng(seed)
    return torch.tensor(g.integers(lo, hi + 1, size=shape), dtype=torch.bfloat16)


def test_ctx_block_means_exact_on_integers_and_ragged_block():
    """Integer keys: every float sum is exact; blocks of 64 divide by a power of two, and the
    ragged last block (3 keys) holds one repeated value, so every mean is exact."""
    B, Hkv, L, d, bc = 2, 3, 131, 16, 64
    K = small_ints((B, Hkv, L, d), -8, 8, 81)
    K[:, :, 128:] = K[:, :, 128:129]  # the last block: three copies of one key
    m = oracle.ctx_block_means(K, bc)
    Ki = K.to(torch.int64).numpy()
    assert m.shape == (B, Hkv, 3, d)
    assert np.array_equal(m[:, :, 0], Ki[:, :, 0:64].sum(axis=2) / 64)
    assert np.array_equal(m[:, :, 1], Ki[:, :, 64:128].sum(axis=2) / 64)
    assert np.array_equal(m[:, :, 2], Ki[:, :, 128])


def test_ctx_block_means_close_to_fp64_mean():
    K = rmm_synth.normal((1, 2, 200, 32), seed=82)
    m = oracle.ctx_block_means(K, 48)
    Kf = f64(K)
    for j in range(5):
        ref = Kf[:, :, 48 * j:min(200, 48 * (j + 1))].mean(axis=2)
        assert np.max(np.abs(m[:, :, j] - ref)) <= 1e-5


@pytest.mark.parametrize("per_head", [False, True])
def test_ctx_block_scores_exact_on_integers(per_head):
    """Integer queries and integer block means (constant keys per block): every fmaf is
    exact, so the score is the integer max over the set's query rows of the dot product."""
    B, Hq, Hkv, T, L, d, bc = 1, 4, 2, 3, 256, 16, 64
    Q = small_ints((B, Hq, T, d), -4, 4, 83)
    Kb = small_ints((B, Hkv, L // bc, 1, d), -8, 8, 84)
    K = Kb.expand(B, Hkv, L // bc, bc, d).reshape(B, Hkv, L, d).contiguous()
    m = oracle.ctx_block_means(K, bc)
    sc = oracle.ctx_block_scores(Q, m, Hkv, per_query_head=per_head)
    Qi, Mi = Q.to(torch.int64).numpy(), Kb.to(torch.int64).numpy()[:, :, :, 0]
    G = Hq // Hkv
    for s in range(Hq if per_head else Hkv):
        heads = [s] if per_head else list(range(s * G, (s + 1) * G))
        g = s // G if per_head else s
        dots = np.einsum("htd,jd->htj", Qi[0, heads], Mi[0, g])
        assert np.array_equal(sc[0, s], dots.max(axis=(0, 1)))


def test_ctx_block_scores_close_to_fp64():
    Q = rmm_synth.normal((1, 4, 2, 64), seed=85)
    K = rmm_synth.normal((1, 1, 320, 64), seed=86)
    m = oracle.ctx_block_means(K, 64)
    sc = oracle.ctx_block_scores(Q, m, 1)
    ref = np.einsum("htd,jd->htj", f64(Q)[0], m[0, 0].astype(np.float64)).max(axis=(0, 1))
    assert np.max(np.abs(sc[0, 0] - ref)) <= 1e-4


@pytest.mark.parametrize("nblk", [1, 4, 7, 10])
def test_ctx_select_brute_force(nblk):
    """Over every kc-subset: the kept set is the unique one whose every member beats every
    dropped block under (score desc, index asc); tie-heavy scores, signed zeros included."""
    g = np.random.default_rng(87 + nblk)
    for trial in range(6):
        sc = g.integers(-2, 3, size=nblk).astype(np.float32)
        sc[sc == 0] = np.where(g.random(int((sc == 0).sum())) < 0.5, -0.0, 0.0)
        for kc in range(1, nblk + 1):
            got = oracle.ctx_select(sc, kc).tolist()
            valid = []
            for S in itertools.combinations(range(nblk), kc):
                out = [j for j in range(nblk) if j not in S]
                if all(sc[i] > sc[j] or (sc[i] == sc[j] and i < j) for i in S for j in out):
                    valid.append(list(S))
            assert valid == [got]


def test_ctx_all_blocks_is_the_head_dim_reduction():
    B, Hq, Hkv, T, L, d = 1, 4, 2, 2, 150, 32
    Q = rmm_synth.normal((B, Hq, T, d), seed=88)
    K = rmm_synth.normal((B, Hkv, L, d), seed=89)
    V = rmm_synth.normal((B, Hkv, L, d), seed=90)
    O, idx, blocks = oracle.attention_ctx(Q, K, V, 16, 64, 3, causal=True)
    Oa, ia = oracle.attention(Q, K, V, 16, causal=True)
    assert np.array_equal(O, Oa) and np.array_equal(idx, ia)
    assert blocks.tolist() == [[[0, 1, 2], [0, 1, 2]]]


@pytest.mark.parametrize("T,causal", [(1, True), (3, True), (2, False)])
def test_ctx_given_blocks_equal_library_attention_on_gathered_keys(T, causal):
    """Attention over the kept blocks equals library softmax attention over a cache that
    holds only those blocks' keys and values (causal mask by original position), with Q
    masked to the kept head dimensions."""
    B, Hq, Hkv, L, d, k, bc = 1, 4, 2, 200, 16, 8, 32
    Q = rmm_synth.normal((B, Hq, T, d), seed=91)
    K = rmm_synth.normal((B, Hkv, L, d), seed=92)
    V = rmm_synth.normal((B, Hkv, L, d), seed=93)
    nblk = -(-L // bc)
    given = np.array([[[1, 4, 6], [0, 5, 6]]], dtype=np.int32)  # block 6 is the ragged one (8 keys)
    scale = 1.0 / math.sqrt(d)
    O, idx, blocks = oracle.attention_ctx(Q, K, V, k, bc, 3, causal=causal, scale=scale, blocks_in=given)
    assert np.array_equal(blocks, given) and nblk == 7
    q, Kf, Vf = f64(Q), f64(K), f64(V)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        pos = np.concatenate([np.arange(j * bc, min(L, (j + 1) * bc)) for j in given[0, g]])
        qm = np.zeros_like(q[0, h])
        qm[:, idx[0, g]] = q[0, h][:, idx[0, g]]
        logits = scale * (qm @ Kf[0, g, pos].T)
        if causal:
            last = L - T + np.arange(T)
            logits = np.where(pos[None, :] <= last[:, None], logits, -np.inf)
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        ref = (p / p.sum(axis=1, keepdims=True)) @ Vf[0, g, pos]
        assert np.max(np.abs(O[0, h] - ref)) <= 1e-12


def test_ctx_dropped_blocks_do_not_matter():
    """With the kept blocks fixed, keys and values inside dropped blocks leave O unchanged;
    values there never enter the score, so changing them keeps the selection too."""
    B, Hq, Hkv, T, L, d = 1, 2, 1, 1, 256, 32
    Q = rmm_synth.normal((B, Hq, T, d), seed=94)
    K = rmm_synth.normal((B, Hkv, L, d), seed=95)
    V = rmm_synth.normal((B, Hkv, L, d), seed=96)
    O, idx, blocks = oracle.attention_ctx(Q, K, V, 16, 64, 2)
    drop = [j for j in range(4) if j not in blocks[0, 0]]
    V2 = V.clone()
    K2 = K.clone()
    for j in drop:
        V2[:, :, 64 * j:64 * (j + 1)] = rmm_synth.normal((1, 1, 64, d), seed=97 + j)
        K2[:, :, 64 * j:64 * (j + 1)] = rmm_synth.normal((1, 1, 64, d), seed=197 + j)
    O_v, _, b_v = oracle.attention_ctx(Q, K, V2, 16, 64, 2)
    assert np.array_equal(b_v, blocks) and np.array_equal(O_v, O)
    O_k, _, _ = oracle.attention_ctx(Q, K2, V2, 16, 64, 2, idx_in=idx, blocks_in=blocks)
    assert np.array_equal(O_k, O)


def test_ctx_dominant_block_is_kept_and_unseen_rows_are_zero():
    B, Hq, Hkv, T, L, d = 1, 1, 1, 3, 130, 16
    Q = rmm_synth.normal((B, Hq, T, d), seed=98)
    K = rmm_synth.normal((B, Hkv, L, d), seed=99) * 0.01
    K[0, 0, 64:128] = (Q[0, 0, 0] * 4).to(torch.bfloat16)  # block 1 points along a query row
    V = rmm_synth.normal((B, Hkv, L, d), seed=100)
    _, _, blocks = oracle.attention_ctx(Q, K, V, d, 64, 1, causal=False)
    assert blocks.tolist() == [[[1]]]
    # only the ragged block 2 (positions 128, 129) kept: the query at position 127 sees none
    O, _, _ = oracle.attention_ctx(Q, K, V, d, 64, 1, causal=True, blocks_in=[[[2]]])
    assert np.all(O[0, 0, 0] == 0.0) and np.any(O[0, 0, 1] != 0.0)


# ---------------------------------------------------------------- mean-magnitude blocks
# cf-1.com post §5.1 / §6.1: a block's importance is its mean absolute activation.


def test_block_mean_exact_on_integers():
    """Small-integer activations: every float sum and the division by a power of two
    are exact, so the kept blocks are the integer ranking (ties to the lower block)."""
    for T in (1, 4):
        X = small_ints((T, 512), -6, 6, 111 + T)
        Xi = np.abs(X.to(torch.int64).numpy())
        sums = Xi.reshape(T, 8, 64).sum(axis=(0, 2))
        for kb in (1, 3, 8):
            order = sorted(range(8), key=lambda j: (-sums[j], j))
            assert oracle.block_select_mean(X, 64, kb).tolist() == sorted(order[:kb])


def test_block_mean_unit_blocks_at_one_token_is_the_slice_select():
    """block = 1, T = 1: the mean magnitude of a slice is |x|, whose order is the order
    of the per-slice max score."""
    X = rmm_synth.activations(1, 300, 112)
    for k in (1, 37, 150, 300):
        assert oracle.block_select_mean(X, 1, k).tolist() == oracle.select(oracle.score(X), k).tolist()


@pytest.mark.parametrize("nb", [3, 6, 9])
def test_block_mean_brute_force(nb):
    """Every kb-subset of blocks: the kept set is the unique one whose members all beat
    every dropped block under (mean desc, index asc), the means taken in fp64 (distinct
    enough here that fp32 rounding cannot reorder them)."""
    X = rmm_synth.activations(3, 16 * nb, 113 + nb)
    m = np.abs(f64(X)).reshape(3, nb, 16).mean(axis=(0, 2))
    for kb in range(1, nb + 1):
        got = oracle.block_select_mean(X, 16, kb).tolist()
        valid = [list(S) for S in itertools.combinations(range(nb), kb)
                 if all(m[i] > m[j] or (m[i] == m[j] and i < j) for i in S for j in range(nb) if j not in S)]
        assert valid == [got]


def test_block_mean_linear_full_ratio_is_dense_and_keeps_the_loud_block():
    X = rmm_synth.activations(2, 256, 114)
    W = rmm_synth.weights(64, 256, 115)
    Y1, b1 = oracle.linear_blocks(X, W, 1.0, block=64, block_score="mean")
    assert b1.tolist() == [0, 1, 2, 3]
    assert np.max(np.abs(Y1 - f64(X) @ f64(W).T)) <= 1e-12 * max(1.0, np.abs(Y1).max())
    X2 = X.clone()
    X2[:, 128:192] = (X2[:, 128:192].float() * 50).to(torch.bfloat16)  # block 2 is loud
    _, b2 = oracle.linear_blocks(X2, W, 0.25, block=64, block_score="mean")
    assert b2.tolist() == [2]


# ---------------------------------------------------------------- invariances
# Relabelling the contraction index, exact rescaling and reordering keys are
# symmetries of the method's definitions; a dropped or swapped index anywhere
# in the oracle breaks one of them.


def test_linear_is_equivariant_under_a_column_permutation():
    """Distinct scores (no ties): permuting X's and W's columns by p permutes the kept
    set by p and leaves Y unchanged."""
    T, H, N = 5, 96, 40
    g = np.random.default_rng(121)
    # small random entries, and one distinct, exactly representable maximum per column
    X = (rmm_synth.activations(T, H, 122).float() * 0.01)
    X[2] = torch.tensor(g.permutation(H) + 1, dtype=torch.float32) / 16
    X = X.to(torch.bfloat16)
    W = rmm_synth.weights(N, H, 123)
    s = oracle.score(X)
    assert len(set(s.tolist())) == H, "the test wants distinct scores"
    perm = g.permutation(H)
    Xp, Wp = X[:, perm].contiguous(), W[:, perm].contiguous()
    for r in (0.25, 0.5, 0.8):
        Y, idx = oracle.linear(X, W, r)
        Yp, idxp = oracle.linear(Xp, Wp, r)
        assert sorted(perm[idxp].tolist()) == idx.tolist()
        assert np.max(np.abs(Y - Yp)) <= 1e-12 * max(1.0, np.abs(Y).max())


def test_linear_scales_exactly_with_a_power_of_two():
    X = rmm_synth.activations(4, 128, 124)
    W = rmm_synth.weights(32, 128, 125)
    Y, idx = oracle.linear(X, W, 0.5)
    Y2, idx2 = oracle.linear((X.float() * 2).to(torch.bfloat16), W, 0.5)
    assert idx.tolist() == idx2.tolist()
    assert np.array_equal(Y2, 2 * Y)


def test_attention_is_invariant_under_a_key_permutation():
    """Non-causal attention: reordering the cache's keys (K and V together) changes
    nothing; with the causal mask of a decode step (T = 1) neither."""
    B, Hq, Hkv, T, L, d = 1, 4, 2, 1, 50, 32
    Q = rmm_synth.normal((B, Hq, T, d), 126)
    K = rmm_synth.normal((B, Hkv, L, d), 127)
    V = rmm_synth.normal((B, Hkv, L, d), 128)
    perm = np.random.default_rng(129).permutation(L)
    Kp, Vp = K[:, :, perm].contiguous(), V[:, :, perm].contiguous()
    for causal in (False, True):
        O, idx = oracle.attention(Q, K, V, 16, causal=causal)
        Op, idxp = oracle.attention(Q, Kp, Vp, 16, causal=causal)
        assert np.array_equal(idx, idxp)
        assert np.max(np.abs(O - Op)) <= 1e-12


def test_context_blocks_follow_their_keys_under_a_block_permutation():
    """Non-causal: reordering whole blocks of keys reorders the block scores the same way,
    so the kept set maps through the permutation and O is unchanged."""
    B, Hq, Hkv, T, bc, nb, d = 1, 4, 1, 2, 32, 8, 32
    L = bc * nb
    Q = rmm_synth.normal((B, Hq, T, d), 130)
    K = rmm_synth.normal((B, Hkv, L, d), 131)
    V = rmm_synth.normal((B, Hkv, L, d), 132)
    bperm = np.random.default_rng(133).permutation(nb)
    pos = (bperm[:, None] * bc + np.arange(bc)[None, :]).reshape(-1)  # new block j holds old block bperm[j]
    Kp, Vp = K[:, :, pos].contiguous(), V[:, :, pos].contiguous()
    O, idx, blocks = oracle.attention_ctx(Q, K, V, 16, bc, 3, causal=False)
    Op, idxp, blocksp = oracle.attention_ctx(Q, Kp, Vp, 16, bc, 3, causal=False)
    assert np.array_equal(idx, idxp)
    assert sorted(bperm[blocksp[0, 0]].tolist()) == blocks[0, 0].tolist()
    assert np.max(np.abs(O - Op)) <= 1e-12


def test_openmp_build_gives_the_same_bits():
    """The parallel CPU baseline: each output row computed by one thread in the same
    order as the plain build, so the two builds agree bit for bit."""
    X = rmm_synth.activations(37, 512, 141)
    W = rmm_synth.weights(300, 512, 142)
    Y1, i1 = oracle.linear(X, W, 0.5)
    Y2, i2 = oracle.linear(X, W, 0.5, parallel=True)
    assert np.array_equal(i1, i2) and np.array_equal(Y1, Y2)
    rows = [36, 0, 5]
    assert np.array_equal(oracle.reduced_product(X, W, i1, rows=rows),
                          oracle.reduced_product(X, W, i1, rows=rows, parallel=True))
    assert oracle.parallel_threads() >= 1
