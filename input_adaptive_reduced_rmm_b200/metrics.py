"""Algorithmic work of each step of the reduced-product path (host-side arithmetic only).

These are the numerators of every throughput and roofline figure the
benchmark reports.  They count the work the method must do, not what a
kernel happens to move.

* FLOPs of a product of an [m, k] and a [k, n] matrix: 2*m*n*k, one multiply
  and one add per term (GEMM primer, tangquanwei.github.io 'GEMM', section 6).
  The reduced product contracts over the k kept slices only, so it costs
  2*T*N*k.
* Bytes of the memory-bound steps: every byte that has to cross HBM once.
"""
from __future__ import annotations

import math


def k_for(H: int, r: float) -> int:
    """k = ceil(r*H) clamped to [1, H]; raises for r outside (0, 1]."""
    if not (0.0 < r <= 1.0) or H < 1:
        raise ValueError(f"bad retention ratio r={r} or H={H}")
    return max(1, min(H, int(math.ceil(r * H))))


def gemm_flops(m: int, n: int, k: int) -> int:
    """2*m*n*k: one multiply and one add per term of an [m,k] x [k,n] product."""
    return 2 * int(m) * int(n) * int(k)


def reduced_linear_flops(T: int, N: int, k: int) -> int:
    """Effective FLOPs of Y ~= X[:,S] W[:,S]^T with |S| = k."""
    return gemm_flops(T, N, k)


def score_bytes(T: int, H: int, write_xt: bool) -> int:
    """Score pass: read X once (T*H*2); on the GEMM path also write X^T once."""
    return T * H * 2 * (2 if write_xt else 1)


def gemv_bytes(T: int, H: int, N: int, k: int) -> int:
    """Decode product: kept weight rows k*N*2, X T*H*2, Y T*N*2, the index list 4*k."""
    return k * N * 2 + T * H * 2 + T * N * 2 + 4 * k


def gemm_min_bytes(T: int, H: int, N: int, k: int) -> int:
    """Prefill product, compulsory traffic: kept rows of W^T and X^T once, Y once."""
    return k * N * 2 + k * T * 2 + T * N * 2 + 4 * k


def attn_decode_bytes(B: int, Hkv: int, L: int, d: int, k: int) -> int:
    """Decode attention: the k kept rows of the d-major K^T cache plus all of V."""
    return B * Hkv * L * 2 * (k + d)


def attn_flops(B: int, Hq: int, T: int, L: int, d: int, k: int, causal: bool = True) -> int:
    """Reduced attention FLOPs: 2*k per logit plus 2*d per P.V term, over the unmasked pairs."""
    if causal:
        # query t sees L - T + t + 1 keys
        pairs = T * (L - T) + T * (T + 1) // 2
    else:
        pairs = T * L
    return 2 * B * Hq * pairs * (k + d)
