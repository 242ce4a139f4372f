"""One Llama-style decoder layer built on the reduced products (batch 1).

    x -> RMSNorm -> q, k, v (one kept set: they share their input)
      -> heads + KV-cache append -> reduced attention (head-dim sets) -> o
      -> residual add + RMSNorm -> gate, up (one kept set) -> SwiGLU -> down
      -> residual add
(without a trace, SwiGLU is applied as gate and up are produced)

The anatomy (RMSNorm, a residual stream through every block, a SwiGLU MLP)
follows the 'Numerical Linear Algebra for LLMs' paper digest (ai-feeds.com),
section 'Method: key modules'; the reduced products and the reduced QK^T
follow the reduced-matrix-multiplication pages (input-adaptive slices of the
contraction dimension kept at ratio r).  RoPE is not applied and the norm
weights are 1.  Every op runs in this package's kernels through the C ABI;
this module only sequences the calls and owns the buffers (PyTorch device
memory).  Intermediates are bf16 between ops.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

from . import rmm

D_HEAD = 128


@dataclass
class LayerDims:
    H: int = 4096        # hidden size
    Hq: int = 32         # query heads
    Hkv: int = 8         # key/value heads
    F: int = 14336       # MLP width
    eps: float = 1e-5

    @property
    def q_cols(self) -> int:
        return self.Hq * D_HEAD

    @property
    def kv_cols(self) -> int:
        return self.Hkv * D_HEAD


class DecoderLayer:
    """Weights pre-transposed once (W^T [in, out]); KV caches for max_len tokens."""

    def __init__(self, dims: LayerDims, weights: dict, max_len: int, r: float, device):
        self.d = dims
        self.r = float(r)
        self.dev = device
        self.Wt = {n: rmm.rmm_transpose_weight(weights[n].to(device)) for n in
                   ("q", "k", "v", "o", "gate", "up", "down")}
        self.ldL = (max_len + 7) // 8 * 8
        self.Kt = torch.zeros(dims.Hkv, D_HEAD, self.ldL, dtype=torch.bfloat16, device=device)
        self.V = torch.zeros(dims.Hkv, self.ldL, D_HEAD, dtype=torch.bfloat16, device=device)
        self.pos = 0
        self._ws = {}
        self._bufs = {}
        self._opts_swiglu = rmm.options(swiglu_pair=True)

    # workspaces and activations are kept per token count, so repeated calls
    # (decode steps) allocate nothing
    def _ws_for(self, key, nbytes):
        w = self._ws.get(key)
        if w is None or w.numel() < nbytes:
            w = rmm.new_workspace(nbytes, self.dev)
            self._ws[key] = w
        return w

    def _buf(self, name, shape):
        key = (name, tuple(shape))
        b = self._bufs.get(key)
        if b is None:
            b = torch.empty(*shape, dtype=torch.bfloat16, device=self.dev)
            self._bufs[key] = b
        return b

    def reset(self):
        self.pos = 0

    def forward(self, x: torch.Tensor, trace: dict | None = None, events: list | None = None) -> torch.Tensor:
        """x [T, H] bf16 at cache positions pos .. pos+T-1 (causal).  Returns the layer output.
        trace (optional) receives every intermediate and kept set; events (optional) receives
        (op name, start event, end event) per op."""
        dm, T, r = self.d, x.shape[0], self.r
        L0 = self.pos
        if L0 + T > self.ldL:
            raise ValueError("KV cache full")
        H, F = dm.H, dm.F

        def op(name):
            if events is None:
                return _NullCtx()
            return _EventCtx(events, name)

        with op("rmsnorm"):
            _, xn = rmm.rmm_add_rmsnorm(x, eps=dm.eps, Y=self._buf("xn", (T, H)))
        idx_qkv = self._idx("qkv", H)
        with op("qkv"):
            yq, yk, yv = self._buf("yq", (T, dm.q_cols)), self._buf("yk", (T, dm.kv_cols)), self._buf("yv", (T, dm.kv_cols))
            rmm.rmm_linear_group(xn, [self.Wt["q"], self.Wt["k"], self.Wt["v"]], r, Ys=[yq, yk, yv],
                                 idx_out=idx_qkv,
                                 workspace=self._ws_for(("qkv", T), rmm.rmm_linear_group_workspace_bytes(
                                     T, H, [dm.q_cols, dm.kv_cols, dm.kv_cols])))
        Q = self._buf("Q", (dm.Hq, T, D_HEAD))
        with op("kv_append"):
            rmm.rmm_qkv_heads(yq, yk, yv, Q, self.Kt, self.V, L0)
        L = L0 + T
        idx_attn = torch.empty(1, dm.Hkv, rmm.rmm_k_for(D_HEAD, r), dtype=torch.int32, device=self.dev)
        O = self._buf("O", (1, dm.Hq, T, D_HEAD))
        with op("attention"):
            rmm.rmm_attn_qk(Q.unsqueeze(0), self.Kt.unsqueeze(0), self.V.unsqueeze(0), L, r, causal=True,
                            O=O, idx_out=idx_attn,
                            workspace=self._ws_for(("attn", T), rmm.rmm_attn_workspace_bytes(
                                1, dm.Hq, dm.Hkv, T, self.ldL, D_HEAD)))
        with op("heads_to_tokens"):
            a = rmm.rmm_heads_to_tokens(O[0], A=self._buf("a", (T, dm.q_cols)))
        idx_o = self._idx("o", dm.q_cols)
        with op("o"):
            yo = rmm.rmm_linear(a, self.Wt["o"], r, Y=self._buf("yo", (T, H)), idx_out=idx_o,
                                workspace=self._ws_for(("o", T), rmm.rmm_linear_workspace_bytes(T, dm.q_cols, H)))
        with op("add_rmsnorm"):
            h2, xn2 = rmm.rmm_add_rmsnorm(x, yo, eps=dm.eps, Hsum=self._buf("h2", (T, H)),
                                          Y=self._buf("xn2", (T, H)))
        idx_gu = self._idx("gu", H)
        ws_gu = self._ws_for(("gu", T), rmm.rmm_linear_group_workspace_bytes(T, H, [F, F]))
        g, u = self._buf("g", (T, F)), self._buf("u", (T, F))
        if trace is None:
            # SwiGLU applied as gate/up are produced (folded into the decode GEMV's
            # split sums; after the products on the GEMM path): hh directly, the
            # same bits as the two steps below
            with op("gate_up_swiglu"):
                hh = self._buf("hh", (T, F))
                rmm.rmm_linear_group(xn2, [self.Wt["gate"], self.Wt["up"]], r, Ys=[hh, u], idx_out=idx_gu,
                                     workspace=ws_gu, opts=self._opts_swiglu)
        else:
            with op("gate_up"):
                rmm.rmm_linear_group(xn2, [self.Wt["gate"], self.Wt["up"]], r, Ys=[g, u], idx_out=idx_gu,
                                     workspace=ws_gu)
            with op("swiglu"):
                hh = rmm.rmm_swiglu(g, u, out=self._buf("hh", (T, F)))
        idx_d = self._idx("down", F)
        with op("down"):
            yd = rmm.rmm_linear(hh, self.Wt["down"], r, Y=self._buf("yd", (T, H)), idx_out=idx_d,
                                workspace=self._ws_for(("down", T), rmm.rmm_linear_workspace_bytes(T, F, H)))
        out = torch.empty(T, H, dtype=torch.bfloat16, device=self.dev)
        with op("residual"):
            rmm.rmm_add_rmsnorm(h2, yd, eps=dm.eps, Hsum=out, want_y=False)
        self.pos = L
        if trace is not None:
            # copies: the activation buffers are reused by the next call
            vals = dict(x=x, xn=xn, yq=yq, yk=yk, yv=yv, Q=Q, L0=L0, L=L, O=O[0], a=a, yo=yo, h2=h2, xn2=xn2,
                        g=g, u=u, hh=hh, yd=yd, out=out, idx_qkv=idx_qkv, idx_attn=idx_attn[0], idx_o=idx_o,
                        idx_gu=idx_gu, idx_down=idx_d, Kt=self.Kt, V=self.V)
            for key, v in vals.items():
                trace[key] = v.clone() if torch.is_tensor(v) else v
        return out

    def _idx(self, name, H):
        return torch.empty(H, dtype=torch.int32, device=self.dev)


class DenseLayer:
    """The same layer with dense products (cuBLAS through torch.matmul) and dense
    attention (torch scaled_dot_product_attention): the comparison, not the product.
    Like the reduced layer, which runs q/k/v and gate/up as one grouped launch each,
    it runs q|k|v and gate|up as one product each over concatenated weights."""

    def __init__(self, dims: LayerDims, weights: dict, max_len: int, device):
        self.d = dims
        self.dev = device
        Wt = {n: weights[n].to(device).t().contiguous() for n in ("q", "k", "v", "o", "gate", "up", "down")}
        self.Wt = {"qkv": torch.cat([Wt["q"], Wt["k"], Wt["v"]], dim=1), "o": Wt["o"],
                   "gate_up": torch.cat([Wt["gate"], Wt["up"]], dim=1), "down": Wt["down"]}
        self.K = torch.zeros(1, dims.Hkv, max_len, D_HEAD, dtype=torch.bfloat16, device=device)
        self.V = torch.zeros(1, dims.Hkv, max_len, D_HEAD, dtype=torch.bfloat16, device=device)
        self.pos = 0

    def reset(self):
        self.pos = 0

    def forward(self, x, events: list | None = None):
        dm, T = self.d, x.shape[0]
        L0, L = self.pos, self.pos + x.shape[0]

        def op(name):
            return _NullCtx() if events is None else _EventCtx(events, name)

        with op("rmsnorm"):
            _, xn = rmm.rmm_add_rmsnorm(x, eps=dm.eps)
        with op("qkv"):
            q, k, v = (xn @ self.Wt["qkv"]).split([dm.q_cols, dm.kv_cols, dm.kv_cols], dim=1)
        with op("kv_append"):
            Q = q.view(T, dm.Hq, D_HEAD).transpose(0, 1).unsqueeze(0)
            self.K[0, :, L0:L] = k.view(T, dm.Hkv, D_HEAD).transpose(0, 1)
            self.V[0, :, L0:L] = v.view(T, dm.Hkv, D_HEAD).transpose(0, 1)
        with op("attention"):
            O = torch.nn.functional.scaled_dot_product_attention(
                Q, self.K[:, :, :L], self.V[:, :, :L], is_causal=(T > 1 and L0 == 0), enable_gqa=True,
                scale=1.0 / math.sqrt(D_HEAD))
        with op("heads_to_tokens"):
            a = O[0].transpose(0, 1).reshape(T, dm.q_cols)
        with op("o"):
            yo = a @ self.Wt["o"]
        with op("add_rmsnorm"):
            h2, xn2 = rmm.rmm_add_rmsnorm(x, yo, eps=dm.eps)
        with op("gate_up"):
            g, u = (xn2 @ self.Wt["gate_up"]).split([dm.F, dm.F], dim=1)
        with op("swiglu"):
            hh = torch.nn.functional.silu(g) * u
        with op("down"):
            yd = hh @ self.Wt["down"]
        with op("residual"):
            out, _ = rmm.rmm_add_rmsnorm(h2, yd, eps=dm.eps, want_y=False)
        self.pos = L
        return out


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


class _EventCtx:
    """Timing events around one op; recorded as graph nodes when the call is being
    captured (external events), so a replayed graph reports per-op device time."""

    def __init__(self, events, name):
        self.events, self.name = events, name

    def __enter__(self):
        ext = torch.cuda.is_current_stream_capturing()
        self.e0 = torch.cuda.Event(enable_timing=True, external=ext)
        self.e1 = torch.cuda.Event(enable_timing=True, external=ext)
        self.e0.record()
        return self

    def __exit__(self, *a):
        self.e1.record()
        self.events.append((self.name, self.e0, self.e1))
        return False
