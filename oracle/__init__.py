"""CPU oracle for Reduced Matrix Multiplication (RMM) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product library never
loads it, and it never loads the product library: the two share nothing but
the seeded input generators of ``rmm_synth``.

The arithmetic lives in ``rmm_oracle.c`` (plain single-threaded C, fp64
accumulation); this module compiles it with gcc on first use (``build()``)
and marshals numpy arrays of bf16 bit patterns (uint16) into it.

Every function follows the method as the pages describe it:

* Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
  LLM Inference (Lan, Li, Zhou), abstract -- each product keeps the slices of
  its contraction dimension that the input makes most significant, at
  retention ratio r;
* Input-adaptive matrix-product reduction for LLM inference (cf-1.com post),
  §2 (Y ~= X @ W_sub^T), §5.1-§5.3 (score, top-k, gather + smaller product),
  §6.1 (top-k then sort; keep ratio 1 reproduces the full product),
  §3.3 (reduce inside attention heads).

Pins (tests/test_oracle_pins.py): closed forms for k, brute force over all
subsets for the kept set on H <= 12, r = 1 against a library dense product,
kept + dropped = full, exact scaling, attention against a library softmax
attention on a Q whose dropped head dimensions are zeroed, and hand-worked
golden fixtures under tests/golden/.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rmm_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

ERR_ARG = -1
ERR_NONFINITE = -2
ERR_NOMEM = -3

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")


_LIB_OMP = os.path.join(_HERE, "_build", "liboracle_omp.so")


def build(force: bool = False, parallel: bool = False) -> str:
    """Compile rmm_oracle.c into _build/liboracle.so (plain gcc, no fast-math, no FMA contraction);
    parallel=True: the same source with OpenMP (output rows spread over the host's threads, each
    row computed as in the plain build) into _build/liboracle_omp.so."""
    out = _LIB_OMP if parallel else _LIB
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
    cmd += ["-fopenmp"] if parallel else []
    cmd += [_SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


_lib = None
_lib_omp = None


def parallel_threads() -> int:
    """Threads the OpenMP build's product loop uses on this host."""
    return int(_load(parallel=True).oracle_threads())


def _load(parallel: bool = False):
    global _lib, _lib_omp
    if parallel and _lib_omp is not None:
        return _lib_omp
    if not parallel and _lib is not None:
        return _lib
    lib = ctypes.CDLL(build(parallel=parallel))
    L, D, I, P = ctypes.c_long, ctypes.c_double, ctypes.c_int, ctypes.c_void_p
    lib.oracle_k_for.argtypes = [L, D]
    lib.oracle_k_for.restype = I
    lib.oracle_score.argtypes = [_u16p, L, L, _u16p]
    lib.oracle_score.restype = I
    lib.oracle_select.argtypes = [_u16p, L, L, _i32p]
    lib.oracle_select.restype = I
    lib.oracle_reduced_product.argtypes = [_u16p, _u16p, L, L, L, _i32p, L, P, L, P, L, _f64p]
    lib.oracle_reduced_product.restype = I
    lib.oracle_linear.argtypes = [_u16p, _u16p, L, L, L, D, P, L, P, L, _f64p, _i32p]
    lib.oracle_linear.restype = I
    lib.oracle_attention.argtypes = [_u16p, _u16p, _u16p, L, L, L, L, L, L, L, I, D, I, P, L,
                                     _f64p, _i32p, P]
    lib.oracle_attention.restype = I
    lib.oracle_ctx_block_means.argtypes = [_u16p, L, L, L, L, L, _f32p]
    lib.oracle_ctx_block_means.restype = I
    lib.oracle_ctx_block_scores.argtypes = [_u16p, _f32p, L, L, L, L, L, L, I, _f32p]
    lib.oracle_ctx_block_scores.restype = I
    lib.oracle_ctx_select.argtypes = [_f32p, L, L, _i32p]
    lib.oracle_ctx_select.restype = I
    lib.oracle_attention_ctx.argtypes = [_u16p, _u16p, _u16p, L, L, L, L, L, L, L, I, D, I, L, L, P, L,
                                         _f64p, _i32p, _i32p, P, P]
    lib.oracle_attention_ctx.restype = I
    lib.oracle_block_select_mean.argtypes = [_u16p, L, L, L, L, _i32p]
    lib.oracle_block_select_mean.restype = I
    lib.oracle_block_select.argtypes = [_u16p, L, L, L, _i32p]
    lib.oracle_block_select.restype = I
    lib.oracle_rmsnorm.argtypes = [_u16p, L, L, D, _f64p]
    lib.oracle_rmsnorm.restype = I
    lib.oracle_swiglu.argtypes = [_u16p, _u16p, L, _f64p]
    lib.oracle_swiglu.restype = I
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = I
    if parallel:
        _lib_omp = lib
    else:
        _lib = lib
    return lib


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


def _bits(a) -> np.ndarray:
    """Accept a bf16 torch tensor or a uint16 numpy array; return contiguous uint16 bits."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch  # local: the oracle itself needs only numpy

    assert a.dtype == torch.bfloat16
    return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _rows(rows):
    if rows is None:
        return None, 0, None
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r.ctypes.data_as(ctypes.c_void_p), len(r), r


def k_for(H: int, r: float) -> int:
    """k = ceil(r*H) clamped to [1, H]; -1 for r outside (0, 1]."""
    return int(_load().oracle_k_for(int(H), float(r)))


def score(X) -> np.ndarray:
    """s[h] = max_t |X[t,h]| as the bf16 magnitude key (uint16)."""
    x = _bits(X)
    T, H = x.shape
    s = np.zeros(H, dtype=np.uint16)
    _check(_load().oracle_score(x, T, H, s), "oracle_score")
    return s


def select(s, k: int) -> np.ndarray:
    """Top-k of s under (score desc, index asc), in ascending index order (int32)."""
    s = np.ascontiguousarray(np.asarray(s, dtype=np.uint16))
    idx = np.zeros(int(k), dtype=np.int32)
    _check(_load().oracle_select(s, len(s), int(k), idx), "oracle_select")
    return idx


def reduced_product(X, W, idx, rows=None, cols=None, parallel: bool = False) -> np.ndarray:
    """Y[r, c] = sum_{j} X[t_r, idx_j] * W[n_c, idx_j] in fp64.  W is [N, H].

    rows / cols (optional) select the token rows and output features computed.
    parallel=True runs the OpenMP build (same bits, rows spread over the host's threads).
    """
    x, w = _bits(X), _bits(W)
    T, H = x.shape
    N = w.shape[0]
    assert w.shape[1] == H
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    rp, nr, _kr = _rows(rows)
    cp, nc, _kc = _rows(cols)
    Y = np.zeros((nr if rows is not None else T, nc if cols is not None else N), dtype=np.float64)
    _check(_load(parallel).oracle_reduced_product(x, w, T, H, N, idx, len(idx), rp, nr, cp, nc, Y),
           "oracle_reduced_product")
    return Y


def linear(X, W, r: float, rows=None, cols=None, parallel: bool = False):
    """(Y fp64 [nrows, ncols], idx int32 [k]) of the reduced linear map Y ~= X[:,S] W[:,S]^T.
    parallel=True runs the OpenMP build (same bits, rows spread over the host's threads)."""
    x, w = _bits(X), _bits(W)
    T, H = x.shape
    N = w.shape[0]
    k = k_for(H, r)
    if k < 1:
        raise OracleError("r must lie in (0, 1]")
    rp, nr, _kr = _rows(rows)
    cp, nc, _kc = _rows(cols)
    Y = np.zeros((nr if rows is not None else T, nc if cols is not None else N), dtype=np.float64)
    idx = np.zeros(k, dtype=np.int32)
    _check(_load(parallel).oracle_linear(x, w, T, H, N, float(r), rp, nr, cp, nc, Y, idx), "oracle_linear")
    return Y, idx


def block_select(s, block: int, kb: int) -> np.ndarray:
    """The kb best blocks of `block` consecutive slices (block score = max of its
    slices' scores), ascending block indices."""
    sv = np.ascontiguousarray(np.asarray(s, dtype=np.uint16))
    H = sv.size
    out = np.zeros(int(kb), dtype=np.int32)
    _check(_load().oracle_block_select(sv, H, int(block), int(kb), out), "oracle_block_select")
    return out


def block_select_mean(X, block: int, kb: int) -> np.ndarray:
    """The kb best blocks of `block` consecutive slices scored by their mean |X| (single
    precision: tokens ascending, then the block's slices ascending, then / (T*block)),
    ascending block indices."""
    x = _bits(X)
    T, H = x.shape
    out = np.zeros(int(kb), dtype=np.int32)
    _check(_load().oracle_block_select_mean(x, T, H, int(block), int(kb), out), "oracle_block_select_mean")
    return out


def linear_blocks(X, W, r: float, block: int = 64, rows=None, cols=None, block_score: str = "max"):
    """The reduced linear map with a block-granular kept set: kb = ceil(r * H / block)
    blocks scored by the max of their slices' scores ("max") or by their mean |X|
    ("mean"); the product over their slices.  Returns (Y fp64, kept blocks)."""
    x = _bits(X)
    H = x.shape[1]
    kb = k_for(H // block, r)
    if block_score == "mean":
        blocks = block_select_mean(X, block, kb)
    elif block_score == "max":
        blocks = block_select(score(X), block, kb)
    else:
        raise ValueError(block_score)
    idx = (blocks[:, None] * block + np.arange(block, dtype=np.int32)[None, :]).reshape(-1)
    return reduced_product(X, W, idx, rows=rows, cols=cols), blocks


def attention(Q, K, V, k: int, causal: bool = True, scale: float | None = None,
              per_query_head: bool = False, t_rows=None, idx_in=None):
    """Reduced attention.  Q [B,Hq,T,d], K/V [B,Hkv,L,d] (bf16).  idx_in (int32
    [B,Hkv|Hq,k]) supplies the kept sets instead of selecting them from Q.

    Returns (O fp64 [B,Hq,nrows,d], idx int32 [B,Hkv|Hq,k]).
    """
    q, kk, v = _bits(Q), _bits(K), _bits(V)
    B, Hq, T, d = q.shape
    _, Hkv, L, _ = kk.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rp, nr, _keep = _rows(t_rows)
    nrows = nr if t_rows is not None else T
    O = np.zeros((B, Hq, nrows, d), dtype=np.float64)
    nsets = Hq if per_query_head else Hkv
    idx = np.zeros((B, nsets, int(k)), dtype=np.int32)
    given = None
    if idx_in is not None:
        given = np.ascontiguousarray(np.asarray(idx_in, dtype=np.int32).reshape(B, nsets, int(k)))
    _check(_load().oracle_attention(q, kk, v, B, Hq, Hkv, T, L, d, int(k), int(bool(causal)),
                                    float(scale), int(bool(per_query_head)), rp, nr, O, idx,
                                    None if given is None else given.ctypes.data_as(ctypes.c_void_p)),
           "oracle_attention")
    return O, idx


def ctx_block_means(K, bc: int) -> np.ndarray:
    """Mean key of each block of bc consecutive positions.  K [B,Hkv,L,d] (bf16).
    Returns float32 [B,Hkv,ceil(L/bc),d] (float sums over l ascending, then / n)."""
    kk = _bits(K)
    B, Hkv, L, d = kk.shape
    nblk = -(-L // int(bc))
    out = np.zeros((B, Hkv, nblk, d), dtype=np.float32)
    _check(_load().oracle_ctx_block_means(kk, B, Hkv, L, d, int(bc), out), "oracle_ctx_block_means")
    return out


def ctx_block_scores(Q, means, Hkv: int, per_query_head: bool = False) -> np.ndarray:
    """Block scores: for each kept set, the largest fmaf-chain dot of its query rows with
    each block mean.  Q [B,Hq,T,d] (bf16), means float32 [B,Hkv,nblk,d].
    Returns float32 [B,nsets,nblk]."""
    q = _bits(Q)
    B, Hq, T, d = q.shape
    m = np.ascontiguousarray(means, dtype=np.float32)
    nblk = m.shape[2]
    nsets = Hq if per_query_head else Hkv
    out = np.zeros((B, nsets, nblk), dtype=np.float32)
    _check(_load().oracle_ctx_block_scores(q, m, B, Hq, Hkv, T, nblk, d, int(bool(per_query_head)), out),
           "oracle_ctx_block_scores")
    return out


def ctx_select(scores, kc: int) -> np.ndarray:
    """The kc best blocks of one score row under (score desc, index asc), ascending."""
    sc = np.ascontiguousarray(np.asarray(scores, dtype=np.float32).reshape(-1))
    out = np.zeros(int(kc), dtype=np.int32)
    _check(_load().oracle_ctx_select(sc, sc.size, int(kc), out), "oracle_ctx_select")
    return out


def attention_ctx(Q, K, V, k: int, bc: int, kc: int, causal: bool = True, scale: float | None = None,
                  per_query_head: bool = False, t_rows=None, idx_in=None, blocks_in=None):
    """Reduced attention over the kept head dimensions and the kept context blocks.
    Q [B,Hq,T,d], K/V [B,Hkv,L,d] (bf16); bc keys per block, kc blocks kept per set.

    Returns (O fp64 [B,Hq,nrows,d], idx int32 [B,nsets,k], blocks int32 [B,nsets,kc]).
    """
    q, kk, v = _bits(Q), _bits(K), _bits(V)
    B, Hq, T, d = q.shape
    _, Hkv, L, _ = kk.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rp, nr, _keep = _rows(t_rows)
    nrows = nr if t_rows is not None else T
    O = np.zeros((B, Hq, nrows, d), dtype=np.float64)
    nsets = Hq if per_query_head else Hkv
    idx = np.zeros((B, nsets, int(k)), dtype=np.int32)
    blocks = np.zeros((B, nsets, int(kc)), dtype=np.int32)
    gi = gb = None
    if idx_in is not None:
        gi = np.ascontiguousarray(np.asarray(idx_in, dtype=np.int32).reshape(B, nsets, int(k)))
    if blocks_in is not None:
        gb = np.ascontiguousarray(np.asarray(blocks_in, dtype=np.int32).reshape(B, nsets, int(kc)))
    _check(_load().oracle_attention_ctx(
        q, kk, v, B, Hq, Hkv, T, L, d, int(k), int(bool(causal)), float(scale), int(bool(per_query_head)),
        int(bc), int(kc), rp, nr, O, idx, blocks,
        None if gi is None else gi.ctypes.data_as(ctypes.c_void_p),
        None if gb is None else gb.ctypes.data_as(ctypes.c_void_p)), "oracle_attention_ctx")
    return O, idx, blocks


def rmsnorm(x, eps: float = 1e-5) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) row-wise (norm weight 1), fp64."""
    b = _bits(x)
    T, H = b.shape
    y = np.zeros((T, H), dtype=np.float64)
    _check(_load().oracle_rmsnorm(b, T, H, float(eps), y), "oracle_rmsnorm")
    return y


def swiglu(g, u) -> np.ndarray:
    """silu(g) * u elementwise, fp64."""
    gb, ub = _bits(g), _bits(u)
    assert gb.shape == ub.shape
    out = np.zeros(gb.shape, dtype=np.float64)
    _check(_load().oracle_swiglu(gb.reshape(-1), ub.reshape(-1), gb.size, out.reshape(-1)),
           "oracle_swiglu")
    return out
