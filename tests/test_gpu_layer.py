"""Decoder layer (prefill then decode steps) on the GPU against the oracle.

Per op, the oracle gets the GPU's own bf16 input to that op, so a last-bit
difference upstream cannot flip a near-tie in a downstream score: kept sets
must then match bit for bit, products and attention meet the float bar, the
relayouts (heads, KV-cache append) and the residual sums are exact.  End to
end, an oracle layer that follows the GPU's kept sets reproduces the layer
output within the float bar.
"""
import numpy as np
import pytest
import torch

import oracle
import rmm_synth
from parity import assert_close, bits_u16, tile_rows

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module")
def rmm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from input_adaptive_reduced_rmm_b200 import rmm as _rmm

    _rmm.lib()
    return _rmm


def make_weights(H, Hq, Hkv, F, seed):
    shapes = {"q": (Hq * D, H), "k": (Hkv * D, H), "v": (Hkv * D, H), "o": (H, Hq * D),
              "gate": (F, H), "up": (F, H), "down": (H, F)}
    return {n: rmm_synth.weights(N, K, rmm_synth.seed_for(3, seed, i), std=0.02)
            for i, (n, (N, K)) in enumerate(shapes.items())}


def bf16(a):
    """fp64 numpy -> bf16 torch (round to nearest even through fp32)."""
    return torch.from_numpy(np.asarray(a, np.float64)).to(torch.float32).to(torch.bfloat16)


def cpu(t):
    return t.detach().cpu()


def check_step(tr, W, r, Hq, Hkv, rows=None):
    """Per-op parity of one forward call, from its trace.  Kept sets are compared in full
    (their scores run over every token row); float outputs on the token rows `rows`
    (None: all of them), each computed by the oracle from the GPU's own inputs."""
    T, H = tr["x"].shape
    rs = slice(None) if rows is None else rows
    par = rows is not None

    def prod(X, Wn, idx):
        return oracle.reduced_product(X, Wn, idx, rows=rows, parallel=par)

    k_h = oracle.k_for(H, r)
    # RMSNorm
    assert_close(cpu(tr["xn"])[rs], oracle.rmsnorm(cpu(tr["x"])[rs]), "rmsnorm")
    # q, k, v: one kept set from xn
    idx = oracle.select(oracle.score(cpu(tr["xn"])), k_h)
    assert cpu(tr["idx_qkv"])[:k_h].numpy().tolist() == idx.tolist(), "q/k/v kept set"
    for n in ("q", "k", "v"):
        assert_close(cpu(tr["y" + n])[rs], prod(cpu(tr["xn"]), W[n], idx), f"{n} projection")
    # heads and the KV-cache append: exact relayouts
    L0, L = tr["L0"], tr["L"]
    yq, yk, yv = cpu(tr["yq"]), cpu(tr["yk"]), cpu(tr["yv"])
    assert torch.equal(cpu(tr["Q"]), yq.view(T, Hq, D).transpose(0, 1)), "Q heads"
    Kt, V = cpu(tr["Kt"]), cpu(tr["V"])
    assert torch.equal(Kt[:, :, L0:L], yk.view(T, Hkv, D).permute(1, 2, 0)), "K cache append"
    assert torch.equal(V[:, L0:L], yv.view(T, Hkv, D).transpose(0, 1)), "V cache append"
    # attention over the cache, kept sets over the head dim from Q
    k_d = oracle.k_for(D, r)
    Kc = Kt[:, :, :L].permute(0, 2, 1).contiguous().unsqueeze(0)
    Vc = V[:, :L].contiguous().unsqueeze(0)
    O_ref, idx_a = oracle.attention(cpu(tr["Q"]).unsqueeze(0), Kc, Vc, k_d, causal=True, t_rows=rows)
    assert np.array_equal(cpu(tr["idx_attn"]).numpy(), idx_a[0]), "attention kept sets"
    assert_close(cpu(tr["O"])[:, rs], O_ref[0], "attention")
    assert torch.equal(cpu(tr["a"]), cpu(tr["O"]).transpose(0, 1).reshape(T, Hq * D)), "heads to tokens"
    # o projection
    k_o = oracle.k_for(Hq * D, r)
    idx = oracle.select(oracle.score(cpu(tr["a"])), k_o)
    assert cpu(tr["idx_o"])[:k_o].numpy().tolist() == idx.tolist(), "o kept set"
    assert_close(cpu(tr["yo"])[rs], prod(cpu(tr["a"]), W["o"], idx), "o projection")
    # residual add (exact: both addends are bf16, their fp32 sum rounds once) + RMSNorm
    h2 = (cpu(tr["x"]).float() + cpu(tr["yo"]).float()).to(torch.bfloat16)
    assert np.array_equal(bits_u16(tr["h2"]), bits_u16(h2)), "residual add"
    assert_close(cpu(tr["xn2"])[rs], oracle.rmsnorm(cpu(tr["h2"])[rs]), "rmsnorm after attention")
    # gate, up (one kept set), SwiGLU, down
    idx = oracle.select(oracle.score(cpu(tr["xn2"])), k_h)
    assert cpu(tr["idx_gu"])[:k_h].numpy().tolist() == idx.tolist(), "gate/up kept set"
    for n, key in (("gate", "g"), ("up", "u")):
        assert_close(cpu(tr[key])[rs], prod(cpu(tr["xn2"]), W[n], idx), f"{n} projection")
    assert_close(cpu(tr["hh"])[rs], oracle.swiglu(cpu(tr["g"])[rs], cpu(tr["u"])[rs]), "swiglu")
    F = tr["hh"].shape[1]
    k_f = oracle.k_for(F, r)
    idx = oracle.select(oracle.score(cpu(tr["hh"])), k_f)
    assert cpu(tr["idx_down"])[:k_f].numpy().tolist() == idx.tolist(), "down kept set"
    assert_close(cpu(tr["yd"])[rs], prod(cpu(tr["hh"]), W["down"], idx), "down projection")
    out = (cpu(tr["h2"]).float() + cpu(tr["yd"]).float()).to(torch.bfloat16)
    assert np.array_equal(bits_u16(tr["out"]), bits_u16(out)), "final residual add"


def oracle_layer_prefill(x, W, r, Hq, Hkv, tr, rows=None):
    """The layer on an empty cache in oracle arithmetic (fp64 ops, bf16 between ops),
    following the GPU's kept sets from the trace.  rows (None: all) restricts the output
    to those token rows: keys and values are still projected for every token (each row
    attends to all earlier ones), queries and everything after attention only for `rows`."""
    T, H = x.shape
    k_h, k_o, k_f = oracle.k_for(H, r), oracle.k_for(Hq * D, r), oracle.k_for(W["down"].shape[1], r)
    par = rows is not None
    rs = slice(None) if rows is None else rows
    xn = bf16(oracle.rmsnorm(x))
    i_qkv = cpu(tr["idx_qkv"])[:k_h].numpy()
    yk, yv = (bf16(oracle.reduced_product(xn, W[n], i_qkv, parallel=par)) for n in ("k", "v"))
    yq = torch.zeros(T, Hq * D, dtype=torch.bfloat16)  # rows not asked for stay zero: the kept sets are given
    yq[rs] = bf16(oracle.reduced_product(xn, W["q"], i_qkv, rows=rows, parallel=par))
    Q = yq.view(T, Hq, D).transpose(0, 1).contiguous().unsqueeze(0)
    K = yk.view(T, Hkv, D).transpose(0, 1).contiguous().unsqueeze(0)
    V = yv.view(T, Hkv, D).transpose(0, 1).contiguous().unsqueeze(0)
    O, _ = oracle.attention(Q, K, V, oracle.k_for(D, r), causal=True, idx_in=cpu(tr["idx_attn"]).numpy()[None],
                            t_rows=rows)
    n = O.shape[2]
    a = bf16(O[0]).transpose(0, 1).reshape(n, Hq * D).contiguous()
    yo = bf16(oracle.reduced_product(a, W["o"], cpu(tr["idx_o"])[:k_o].numpy()))
    h2 = (x[rs].float() + yo.float()).to(torch.bfloat16)
    xn2 = bf16(oracle.rmsnorm(h2))
    i_gu = cpu(tr["idx_gu"])[:k_h].numpy()
    g, u = (bf16(oracle.reduced_product(xn2, W[n], i_gu)) for n in ("gate", "up"))
    hh = bf16(oracle.swiglu(g, u))
    yd = bf16(oracle.reduced_product(hh, W["down"], cpu(tr["idx_down"])[:k_f].numpy()))
    return (h2.double() + yd.double()).numpy()


@pytest.mark.parametrize("T", [24, 40])
def test_layer_prefill_then_decode(rmm, T):
    from input_adaptive_reduced_rmm_b200.layer import DecoderLayer, LayerDims

    H, Hq, Hkv, F, r = 512, 4, 2, 1024, 0.5
    W = make_weights(H, Hq, Hkv, F, T)
    dims = LayerDims(H=H, Hq=Hq, Hkv=Hkv, F=F)
    layer = DecoderLayer(dims, W, max_len=T + 8, r=r, device=torch.device("cuda"))
    x = rmm_synth.activations(T, H, rmm_synth.seed_for(3, T, 9))
    tr = {}
    y = layer.forward(x.cuda(), trace=tr)
    torch.cuda.synchronize()
    check_step(tr, W, r, Hq, Hkv)
    assert_close(y, oracle_layer_prefill(x, W, r, Hq, Hkv, tr), "layer output (prefill, GPU kept sets)")
    # decode steps: one token at a time against the growing cache
    for step in range(3):
        xt = rmm_synth.activations(1, H, rmm_synth.seed_for(3, T, 10 + step))
        tr = {}
        layer.forward(xt.cuda(), trace=tr)
        torch.cuda.synchronize()
        assert tr["L"] == T + step + 1
        check_step(tr, W, r, Hq, Hkv)


def test_layer_llama3_8b_full_size(rmm):
    """The decoder layer at its Llama-3-8B size (hidden 4096, 32 query / 8 KV heads, d = 128,
    MLP 14336), prefill of T = 2048 tokens then decode steps against the 2048+ cache, r = 0.5.
    Kept sets in full; float outputs on one token row per 128-row tile (the products' and the
    attention's query tiles) and the first and last rows."""
    from input_adaptive_reduced_rmm_b200.layer import DecoderLayer, LayerDims

    H, Hq, Hkv, F, r, T = 4096, 32, 8, 14336, 0.5, 2048
    W = make_weights(H, Hq, Hkv, F, 77)
    dims = LayerDims(H=H, Hq=Hq, Hkv=Hkv, F=F)
    layer = DecoderLayer(dims, W, max_len=T + 8, r=r, device=torch.device("cuda"))
    x = rmm_synth.activations(T, H, rmm_synth.seed_for(3, 77, 9))
    tr = {}
    y = layer.forward(x.cuda(), trace=tr)
    torch.cuda.synchronize()
    rows = tile_rows(T, 128, seed=7)
    check_step(tr, W, r, Hq, Hkv, rows=rows)
    assert_close(cpu(y)[rows], oracle_layer_prefill(x, W, r, Hq, Hkv, tr, rows=rows),
                 "layer output (prefill T=2048, GPU kept sets)")
    del tr
    for step in range(3):
        xt = rmm_synth.activations(1, H, rmm_synth.seed_for(3, 77, 10 + step))
        tr = {}
        layer.forward(xt.cuda(), trace=tr)
        torch.cuda.synchronize()
        assert tr["L"] == T + step + 1
        check_step(tr, W, r, Hq, Hkv)


def test_glue_ops_exact_and_edges(rmm):
    """RMSNorm with a weight, SwiGLU against its closed form, argument checks."""
    T, H = 5, 264
    x = rmm_synth.activations(T, H, 91).cuda()
    w = rmm_synth.normal((H,), 92).cuda()
    _, y = rmm.rmm_add_rmsnorm(x, weight=w)
    ref = oracle.rmsnorm(cpu(x)) * cpu(w).double().numpy()[None, :]
    assert_close(y, ref, "rmsnorm with weight")
    g = rmm_synth.normal((3, 64), 93).cuda()
    u = rmm_synth.normal((3, 64), 94).cuda()
    assert_close(rmm.rmm_swiglu(g, u), oracle.swiglu(cpu(g), cpu(u)), "swiglu")
    L = rmm.lib()
    assert L.rmm_add_rmsnorm(rmm._ptr(x), None, T, 12, 1e-5, None, None, rmm._ptr(y), None) == rmm.RMM_ERR_INVALID_ARG
    assert L.rmm_swiglu(rmm._ptr(g), rmm._ptr(u), 7, rmm._ptr(g), None) == rmm.RMM_ERR_INVALID_ARG
    z = torch.empty(8, 8, dtype=torch.bfloat16, device="cuda")
    assert L.rmm_heads_to_tokens(rmm._ptr(z), 1, 8, 64, rmm._ptr(z), None) == rmm.RMM_ERR_UNSUPPORTED
    assert L.rmm_qkv_heads(rmm._ptr(z), rmm._ptr(z), rmm._ptr(z), 8, 1, 1, 128, rmm._ptr(z), rmm._ptr(z),
                           rmm._ptr(z), 8, 4, None) == rmm.RMM_ERR_INVALID_ARG  # L0 + T > ldL
