"""The FFN of the cf-1.com post's demo as a workload of this package's kernels.

Input-adaptive matrix-product reduction for LLM inference (cf-1.com post),
§6.1: a gated FFN whose gate and up projections run in full, h = silu(gate)
* up, and whose down projection keeps only the blocks of 64 intermediate
neurons with the largest mean |h| (keep ratio 0.5; the kept blocks depend on
the current token); §6.2: the down projection's work drops with the keep
ratio while gate and up stay full.  The demo's sizes are H = 1024, M = 4096.

Every op runs in the package's kernels through the C ABI: gate and up as one
reduced-product group at ratio 1 (every slice kept: the full products) with
the SwiGLU applied as the split products are folded (or, unfused, the SwiGLU
kernel after them), then the down projection with mean-magnitude
block-granular kept sets.  This module only sequences the calls and owns the buffers.
"""
from __future__ import annotations

import torch

from . import rmm


class FfnBlockReduce:
    """Gate/up full, down projection reduced by mean-|h| blocks.

    W_gate, W_up: [M, H]; W_down: [H, M] (each the model's [out, in] weight),
    bf16 on the device.  forward(x [T, H], T <= 16) returns (y [T, H], kept blocks
    [kb], h [T, M])."""

    def __init__(self, W_gate: torch.Tensor, W_up: torch.Tensor, W_down: torch.Tensor, block: int = 64,
                 keep: float = 0.5, fused_swiglu: bool = True):
        self.M, self.H = W_gate.shape
        if W_up.shape != (self.M, self.H) or W_down.shape != (self.H, self.M):
            raise ValueError("gate/up must be [M, H] and down [H, M]")
        self.block, self.keep = int(block), float(keep)
        self.Wg_t = rmm.rmm_transpose_weight(W_gate)
        self.Wu_t = rmm.rmm_transpose_weight(W_up)
        self.Wd_t = rmm.rmm_transpose_weight(W_down)
        self.kb = rmm.rmm_k_for(self.M // self.block, self.keep)
        self.opts_down = rmm.options(block_size=self.block, block_score=1)
        # gate and up with the SwiGLU applied as they are folded (h written directly;
        # the up buffer is scratch), or the three steps one by one (gate, up kept)
        self.fused = bool(fused_swiglu)
        self.opts_gu = rmm.options(swiglu_pair=True) if self.fused else None
        self._bufs = {}

    def _buffers(self, T: int, dev):
        if T not in self._bufs:
            b = {
                "gate": torch.empty(T, self.M, dtype=torch.bfloat16, device=dev),
                "up": torch.empty(T, self.M, dtype=torch.bfloat16, device=dev),
                "h": torch.empty(T, self.M, dtype=torch.bfloat16, device=dev),
                "y": torch.empty(T, self.H, dtype=torch.bfloat16, device=dev),
                "idx": torch.empty(self.kb * self.block, dtype=torch.int32, device=dev),
                "ws_gu": rmm.new_workspace(rmm.rmm_linear_group_workspace_bytes(T, self.H, [self.M, self.M]), dev),
                "ws_d": rmm.new_workspace(rmm.rmm_linear_workspace_bytes(T, self.M, self.H, self.opts_down), dev),
            }
            self._bufs[T] = b
        return self._bufs[T]

    def forward(self, x: torch.Tensor, want_blocks: bool = True):
        """(y, kept blocks, h); want_blocks=False returns (y, None, h) and launches nothing
        beyond the FFN itself (the kept block ids are derived from the kept slices by a
        tensor op)."""
        T = x.shape[0]
        b = self._buffers(T, x.device)
        if self.fused:
            rmm.rmm_linear_group(x, [self.Wg_t, self.Wu_t], 1.0, Ys=[b["h"], b["up"]], workspace=b["ws_gu"],
                                 opts=self.opts_gu)
        else:
            rmm.rmm_linear_group(x, [self.Wg_t, self.Wu_t], 1.0, Ys=[b["gate"], b["up"]], workspace=b["ws_gu"])
            rmm.rmm_swiglu(b["gate"], b["up"], out=b["h"])
        rmm.rmm_linear(b["h"], self.Wd_t, self.keep, Y=b["y"], idx_out=b["idx"], workspace=b["ws_d"],
                       opts=self.opts_down)
        blocks = b["idx"].view(self.kb, self.block)[:, 0] // self.block if want_blocks else None
        return b["y"], blocks, b["h"]

    def forward_dense(self, x: torch.Tensor):
        """The full FFN with cuBLAS products and the same SwiGLU kernel (comparison)."""
        gate = torch.matmul(x, self.Wg_t)
        up = torch.matmul(x, self.Wu_t)
        h = rmm.rmm_swiglu(gate, up)
        return torch.matmul(h, self.Wd_t)
