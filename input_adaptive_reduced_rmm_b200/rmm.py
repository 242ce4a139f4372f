"""Thin ctypes binding of librmm (C ABI in include/rmm.h), with the same names.

Argument marshalling only: tensors become device pointers and sizes, the
current torch stream becomes the cudaStream_t, a non-OK status becomes an
exception.  Every step of the computation runs in librmm's CUDA kernels;
there is no fallback path, and a missing library raises on first use.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librmm.so")

RMM_OK = 0
RMM_ERR_INVALID_ARG = 1
RMM_ERR_UNSUPPORTED = 2
RMM_ERR_WORKSPACE = 3
RMM_ERR_CUDA = 4
RMM_ERR_TIMEOUT = 5

# every symbol include/rmm.h declares
EXPORTED = (
    "rmm_status_string", "rmm_k_for", "rmm_workspace_init", "rmm_get_status",
    "rmm_transpose_weight", "rmm_linear_workspace_bytes", "rmm_linear", "rmm_score",
    "rmm_select", "rmm_gemm_reduced", "rmm_attn_workspace_bytes", "rmm_attn_qk",
    "rmm_linear_decode_noalloc", "rmm_linear_group", "rmm_linear_group_workspace_bytes",
    "rmm_add_rmsnorm", "rmm_swiglu", "rmm_qkv_heads", "rmm_heads_to_tokens",
    "rmm_ctx_block_means", "rmm_attn_ctx_workspace_bytes", "rmm_attn_ctx", "rmm_selftest_exp2_fma",
)


class RmmError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {rmm_status_string(status)} ({status})")
        self.status = status


class rmm_options(ctypes.Structure):
    _fields_ = [
        ("t_gemv", ctypes.c_int),
        ("attn_per_query_head", ctypes.c_int),
        ("gemv_splits", ctypes.c_int),
        ("debug_timeout_test", ctypes.c_int),
        ("gemm_producer", ctypes.c_int),
        ("attn_path", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("block_score", ctypes.c_int),
        ("swiglu_pair", ctypes.c_int),
        ("product_event_begin", ctypes.c_void_p),
        ("product_event_end", ctypes.c_void_p),
    ]


def options(t_gemv: int = 16, attn_per_query_head: bool = False, gemv_splits: int = 0,
            debug_timeout_test: bool = False, gemm_producer: int = 0, attn_path: int = 0,
            block_size: int = 0, block_score: int = 0, swiglu_pair: bool = False,
            product_events=None) -> rmm_options:
    """An rmm_options struct; product_events = (begin, end) torch.cuda.Event pair (enable_timing);
    attn_path 0 = auto, 1 = CUDA-core split pass, 2 = tensor cores; block_size 0 = single-slice
    kept sets, else blocks of that many consecutive slices; block_score 0 = max of the slice
    scores, 1 = mean magnitude of the block (T <= 16); swiglu_pair: for a group of two products
    of one width (gate, up), Ys[0] receives bf16(silu(gate) * up) and Ys[1] is scratch."""
    o = rmm_options(int(t_gemv), int(bool(attn_per_query_head)), int(gemv_splits),
                    int(bool(debug_timeout_test)), int(gemm_producer), int(attn_path), int(block_size),
                    int(block_score), int(bool(swiglu_pair)), None, None)
    if product_events is not None:
        b, e = product_events
        for ev in (b, e):
            if ev.cuda_event == 0:  # torch creates the CUDA event on its first record
                ev.record()
        o.product_event_begin = ctypes.c_void_p(b.cuda_event)
        o.product_event_end = ctypes.c_void_p(e.cuda_event)
    return o


_lib = None


def lib() -> ctypes.CDLL:
    """Load librmm.so (built in-tree by input_adaptive_reduced_rmm_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m input_adaptive_reduced_rmm_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, D, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float, ctypes.c_size_t
    OP = ctypes.POINTER(rmm_options)
    sig = {
        "rmm_status_string": (ctypes.c_char_p, [I]),
        "rmm_k_for": (I, [I, D]),
        "rmm_workspace_init": (I, [P, Z, P]),
        "rmm_get_status": (I, [P, P]),
        "rmm_transpose_weight": (I, [P, P, I, I, P]),
        "rmm_linear_workspace_bytes": (Z, [I, I, I, OP]),
        "rmm_linear": (I, [P, P, I, I, I, D, P, P, P, Z, P, OP]),
        "rmm_score": (I, [P, I, I, P, P, Z, P]),
        "rmm_select": (I, [P, I, I, P, P, Z, P]),
        "rmm_gemm_reduced": (I, [P, P, P, I, I, I, I, P, P, Z, P, OP]),
        "rmm_attn_workspace_bytes": (Z, [I, I, I, I, I, I, OP]),
        "rmm_attn_qk": (I, [P, P, P, I, I, I, I, I, I, I, D, I, F, P, P, P, Z, P, OP]),
        "rmm_linear_decode_noalloc": (I, [P, P, I, I, I, D, P, P, P]),
        "rmm_linear_group_workspace_bytes": (Z, [I, I, I, P, OP]),
        "rmm_linear_group": (I, [P, I, I, D, I, P, P, P, P, P, Z, P, OP]),
        "rmm_add_rmsnorm": (I, [P, P, I, I, F, P, P, P, P]),
        "rmm_swiglu": (I, [P, P, ctypes.c_int64, P, P]),
        "rmm_qkv_heads": (I, [P, P, P, I, I, I, I, P, P, P, I, I, P]),
        "rmm_heads_to_tokens": (I, [P, I, I, I, P, P]),
        "rmm_ctx_block_means": (I, [P, I, I, I, I, I, I, I, I, P, P]),
        "rmm_attn_ctx_workspace_bytes": (Z, [I, I, I, I, I, I, I, D, OP]),
        "rmm_attn_ctx": (I, [P, P, P, P, I, I, I, I, I, I, I, D, D, I, I, F, P, P, P, P, Z, P, OP]),
        "rmm_selftest_exp2_fma": (I, [P, P, I, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _opt(o):
    return None if o is None else ctypes.byref(o)


def _check(rc: int, what: str):
    if rc != RMM_OK:
        raise RmmError(rc, what)


def _bf16_cuda(t, name):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


def _need(t, name, dtype=torch.bfloat16, shape=None, min_numel=None):
    """Structure of a tensor handed to a kernel: dtype, contiguity, exact shape or
    least element count.  The device is checked separately (_on_cuda), after every
    tensor's structure, so that a wrong-sized output is named as such."""
    if t is None:
        return
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs at least {min_numel}")


def _on_cuda(**tensors):
    for name, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")


def _dims(t, name, n):
    if t.dim() != n:
        raise ValueError(f"{name} must have {n} dimensions, has {t.dim()}")


def rmm_status_string(status: int) -> str:
    return lib().rmm_status_string(int(status)).decode()


def rmm_k_for(H: int, r: float) -> int:
    return int(lib().rmm_k_for(int(H), float(r)))


def _kept_count(H: int, r: float, opts=None) -> int:
    """Entries the library writes to idx_out for a linear call: ceil(r*H) kept slices, or
    with block-granular sets (blocks of b slices, b dividing H) ceil(r*H/b) whole blocks."""
    b = int(opts.block_size) if opts is not None else 0
    if b > 0:
        return max(0, rmm_k_for(int(H) // b, r) * b)
    return max(0, rmm_k_for(H, r))


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled device workspace (the status word must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def rmm_workspace_init(workspace: torch.Tensor, stream=None):
    _check(lib().rmm_workspace_init(_ptr(workspace), workspace.numel(), _stream(stream)),
           "rmm_workspace_init")


def rmm_get_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status word."""
    return int(lib().rmm_get_status(_ptr(workspace), _stream(stream)))


def rmm_transpose_weight(W: torch.Tensor, Wt: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W [N, H] -> W^T [H, N] (bf16)."""
    _bf16_cuda(W, "W")
    N, H = W.shape
    if Wt is None:
        Wt = torch.empty(H, N, dtype=torch.bfloat16, device=W.device)
    _check(lib().rmm_transpose_weight(_ptr(W), _ptr(Wt), N, H, _stream(stream)), "rmm_transpose_weight")
    return Wt


def rmm_linear_workspace_bytes(T: int, H: int, N: int, opts: rmm_options | None = None) -> int:
    return int(lib().rmm_linear_workspace_bytes(int(T), int(H), int(N), _opt(opts)))


def rmm_linear(X: torch.Tensor, Wt: torch.Tensor, r: float, Y: torch.Tensor | None = None,
               idx_out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
               opts: rmm_options | None = None, stream=None) -> torch.Tensor:
    """Y ~= X[:,S] W[:,S]^T with S the ceil(r*H) kept slices.  X [T,H], Wt [H,N] bf16;
    idx_out (optional) int32 with room for the kept list (H entries always suffice)."""
    _dims(X, "X", 2)
    _dims(Wt, "Wt", 2)
    T, H = X.shape
    H2, N = Wt.shape
    if H2 != H:
        raise ValueError("X and Wt disagree on H")
    _need(X, "X")
    _need(Wt, "Wt")
    _need(Y, "Y", shape=(T, N))
    _need(idx_out, "idx_out", torch.int32, min_numel=_kept_count(H, r, opts))
    _on_cuda(X=X, Wt=Wt, Y=Y, idx_out=idx_out)
    if Y is None:
        Y = torch.empty(T, N, dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = new_workspace(rmm_linear_workspace_bytes(T, H, N, opts), X.device)
    _check(lib().rmm_linear(_ptr(X), _ptr(Wt), T, H, N, float(r), _ptr(Y), _ptr(idx_out),
                            _ptr(workspace), workspace.numel(), _stream(stream), _opt(opts)),
           "rmm_linear")
    return Y


def rmm_linear_group_workspace_bytes(T: int, H: int, Ns, opts: rmm_options | None = None) -> int:
    arr = (ctypes.c_int * len(Ns))(*[int(n) for n in Ns])
    return int(lib().rmm_linear_group_workspace_bytes(int(T), int(H), len(Ns), arr, _opt(opts)))


def rmm_linear_group(X: torch.Tensor, Wts, r: float, Ys=None, idx_out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, opts: rmm_options | None = None, stream=None):
    """Projections of one activation matrix sharing one kept set: [X[:,S] W_p[:,S]^T for each W_p^T in Wts]."""
    _dims(X, "X", 2)
    _need(X, "X")
    T, H = X.shape
    Ns = []
    for i, Wt in enumerate(Wts):
        _dims(Wt, f"Wts[{i}]", 2)
        _need(Wt, f"Wts[{i}]")
        if Wt.shape[0] != H:
            raise ValueError("X and a weight disagree on H")
        Ns.append(Wt.shape[1])
    if Ys is not None:
        if len(Ys) != len(Ns):
            raise ValueError("Ys and Wts differ in length")
        for i, Y in enumerate(Ys):
            _need(Y, f"Ys[{i}]", shape=(T, Ns[i]))
    _need(idx_out, "idx_out", torch.int32, min_numel=_kept_count(H, r, opts))
    _on_cuda(X=X, idx_out=idx_out, **{f"Wts[{i}]": W for i, W in enumerate(Wts)},
             **{f"Ys[{i}]": Y for i, Y in enumerate(Ys or [])})
    if Ys is None:
        Ys = [torch.empty(T, n, dtype=torch.bfloat16, device=X.device) for n in Ns]
    if workspace is None:
        workspace = new_workspace(rmm_linear_group_workspace_bytes(T, H, Ns, opts), X.device)
    c = len(Ns)
    w_arr = (ctypes.c_void_p * c)(*[W.data_ptr() for W in Wts])
    y_arr = (ctypes.c_void_p * c)(*[Y.data_ptr() for Y in Ys])
    n_arr = (ctypes.c_int * c)(*Ns)
    _check(lib().rmm_linear_group(_ptr(X), T, H, float(r), c, w_arr, n_arr, y_arr, _ptr(idx_out),
                                  _ptr(workspace), workspace.numel(), _stream(stream), _opt(opts)),
           "rmm_linear_group")
    return Ys


def rmm_score(X: torch.Tensor, s_out: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """s[h] = max_t |X[t,h]| as the bf16 magnitude key (int32 tensor holding uint32 values)."""
    _dims(X, "X", 2)
    _need(X, "X")
    T, H = X.shape
    _need(s_out, "s_out", torch.int32, min_numel=H)
    _on_cuda(X=X, s_out=s_out)
    if s_out is None:
        s_out = torch.empty(H, dtype=torch.int32, device=X.device)
    if workspace is None:
        workspace = new_workspace(rmm_linear_workspace_bytes(T, H, 8), X.device)
    _check(lib().rmm_score(_ptr(X), T, H, _ptr(s_out), _ptr(workspace), workspace.numel(),
                           _stream(stream)), "rmm_score")
    return s_out


def rmm_select(s: torch.Tensor, k: int, idx_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The k best indices of s under (score desc, index asc), ascending (int32)."""
    _need(s, "s", torch.int32)
    H = s.numel()
    _need(idx_out, "idx_out", torch.int32, min_numel=int(k))
    _on_cuda(s=s, idx_out=idx_out)
    if idx_out is None:
        idx_out = torch.empty(int(k), dtype=torch.int32, device=s.device)
    _check(lib().rmm_select(_ptr(s), H, int(k), _ptr(idx_out), None, 0, _stream(stream)), "rmm_select")
    return idx_out


def rmm_gemm_reduced(X: torch.Tensor, Wt: torch.Tensor, idx: torch.Tensor, Y: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, opts: rmm_options | None = None,
                     stream=None) -> torch.Tensor:
    """Y[t,n] = sum_j X[t, idx_j] * Wt[idx_j, n] for a given kept list."""
    _dims(X, "X", 2)
    _dims(Wt, "Wt", 2)
    T, H = X.shape
    H2, N = Wt.shape
    if H2 != H:
        raise ValueError("X and Wt disagree on H")
    _need(X, "X")
    _need(Wt, "Wt")
    _need(idx, "idx", torch.int32)
    _need(Y, "Y", shape=(T, N))
    _on_cuda(X=X, Wt=Wt, idx=idx, Y=Y)
    if Y is None:
        Y = torch.empty(T, N, dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = new_workspace(rmm_linear_workspace_bytes(T, H, N, opts), X.device)
    _check(lib().rmm_gemm_reduced(_ptr(X), _ptr(Wt), _ptr(idx), idx.numel(), T, H, N, _ptr(Y),
                                  _ptr(workspace), workspace.numel(), _stream(stream), _opt(opts)),
           "rmm_gemm_reduced")
    return Y


def rmm_attn_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, L: int, d: int = 128,
                             opts: rmm_options | None = None) -> int:
    return int(lib().rmm_attn_workspace_bytes(B, Hq, Hkv, T, L, d, _opt(opts)))


def rmm_attn_qk(Q: torch.Tensor, Kt: torch.Tensor, V: torch.Tensor, L: int, r: float,
                causal: bool = True, scale: float | None = None, O: torch.Tensor | None = None,
                idx_out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                opts: rmm_options | None = None, stream=None) -> torch.Tensor:
    """Reduced attention.  Q [B,Hq,T,d]; Kt [B,Hkv,d,ldL] (d-major keys); V [B,Hkv,ldL,d];
    idx_out (optional) int32 with room for [B, sets, ceil(r*d)] (sets = Hkv, or Hq per query head)."""
    _dims(Q, "Q", 4)
    _dims(Kt, "Kt", 4)
    B, Hq, T, d = Q.shape
    _, Hkv, d2, ldL = Kt.shape
    if d2 != d or Kt.shape[0] != B or tuple(V.shape) != (B, Hkv, ldL, d):
        raise ValueError("Q, Kt, V shapes disagree")
    for t, n in ((Q, "Q"), (Kt, "Kt"), (V, "V")):
        _need(t, n)
    _need(O, "O", shape=tuple(Q.shape))
    nsets = Hq if (opts is not None and opts.attn_per_query_head) else Hkv
    _need(idx_out, "idx_out", torch.int32, min_numel=B * nsets * max(0, rmm_k_for(d, r)))
    _on_cuda(Q=Q, Kt=Kt, V=V, O=O, idx_out=idx_out)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace = new_workspace(rmm_attn_workspace_bytes(B, Hq, Hkv, T, L, d, opts), Q.device)
    _check(lib().rmm_attn_qk(_ptr(Q), _ptr(Kt), _ptr(V), B, Hq, Hkv, T, int(L), ldL, d, float(r),
                             int(bool(causal)), float(scale), _ptr(O), _ptr(idx_out), _ptr(workspace),
                             workspace.numel(), _stream(stream), _opt(opts)), "rmm_attn_qk")
    return O


def ctx_num_blocks(L: int, block: int) -> int:
    return -(-int(L) // int(block))


def new_ctx_means(Kt: torch.Tensor, block: int) -> torch.Tensor:
    """A zeroed block-mean buffer for the key cache Kt [B,Hkv,d,ldL]: fp32 [B,Hkv,ceil(ldL/block),d]."""
    B, Hkv, d, ldL = Kt.shape
    return torch.zeros(B, Hkv, ctx_num_blocks(ldL, block), d, dtype=torch.float32, device=Kt.device)


def rmm_ctx_block_means(Kt: torch.Tensor, L: int, block: int, means: torch.Tensor | None = None,
                        blk_begin: int = 0, blk_end: int | None = None, stream=None) -> torch.Tensor:
    """Mean key of the context blocks [blk_begin, blk_end) of the first L cache positions
    (all of them by default), written into means (fp32 [B,Hkv,ceil(ldL/block),d])."""
    _bf16_cuda(Kt, "Kt")
    B, Hkv, d, ldL = Kt.shape
    if means is None:
        means = new_ctx_means(Kt, block)
    _need(means, "means", torch.float32, shape=(B, Hkv, ctx_num_blocks(ldL, block), d))
    _on_cuda(means=means)
    if blk_end is None:
        blk_end = ctx_num_blocks(L, block)
    _check(lib().rmm_ctx_block_means(_ptr(Kt), B, Hkv, d, int(L), ldL, int(block), int(blk_begin), int(blk_end),
                                     _ptr(means), _stream(stream)), "rmm_ctx_block_means")
    return means


def rmm_attn_ctx_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, L: int, block: int, r_ctx: float,
                                 d: int = 128, opts: rmm_options | None = None) -> int:
    return int(lib().rmm_attn_ctx_workspace_bytes(B, Hq, Hkv, T, L, d, block, float(r_ctx), _opt(opts)))


def rmm_attn_ctx(Q: torch.Tensor, Kt: torch.Tensor, V: torch.Tensor, means: torch.Tensor, L: int, r: float,
                 r_ctx: float, block: int, causal: bool = True, scale: float | None = None,
                 O: torch.Tensor | None = None, idx_out: torch.Tensor | None = None,
                 blocks_out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                 opts: rmm_options | None = None, stream=None) -> torch.Tensor:
    """Reduced attention over the kept head dimensions and the kept context blocks."""
    _dims(Q, "Q", 4)
    _dims(Kt, "Kt", 4)
    B, Hq, T, d = Q.shape
    _, Hkv, d2, ldL = Kt.shape
    if d2 != d or Kt.shape[0] != B or tuple(V.shape) != (B, Hkv, ldL, d):
        raise ValueError("Q, Kt, V shapes disagree")
    for t, n in ((Q, "Q"), (Kt, "Kt"), (V, "V")):
        _need(t, n)
    _need(means, "means", torch.float32, shape=(B, Hkv, ctx_num_blocks(ldL, block), d))
    _need(O, "O", shape=tuple(Q.shape))
    nsets = Hq if (opts is not None and opts.attn_per_query_head) else Hkv
    _need(idx_out, "idx_out", torch.int32, min_numel=B * nsets * max(0, rmm_k_for(d, r)))
    _need(blocks_out, "blocks_out", torch.int32,
          min_numel=B * nsets * max(0, rmm_k_for(ctx_num_blocks(L, block), r_ctx)))
    _on_cuda(Q=Q, Kt=Kt, V=V, means=means, O=O, idx_out=idx_out, blocks_out=blocks_out)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace = new_workspace(rmm_attn_ctx_workspace_bytes(B, Hq, Hkv, T, L, block, r_ctx, d, opts), Q.device)
    _check(lib().rmm_attn_ctx(_ptr(Q), _ptr(Kt), _ptr(V), _ptr(means), B, Hq, Hkv, T, int(L), ldL, d, float(r),
                              float(r_ctx), int(block), int(bool(causal)), float(scale), _ptr(O), _ptr(idx_out),
                              _ptr(blocks_out), _ptr(workspace), workspace.numel(), _stream(stream), _opt(opts)),
           "rmm_attn_ctx")
    return O


def rmm_linear_decode_noalloc(X: torch.Tensor, Wt: torch.Tensor, r: float, Y: torch.Tensor,
                              idx_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The decode-sized reduced linear map (T <= 16) with no workspace, for callers that may
    not allocate device memory.  Y [T, N] must be given (the binding allocates nothing);
    idx_out (optional) int32 with room for ceil(r*H) entries."""
    _dims(X, "X", 2)
    _dims(Wt, "Wt", 2)
    T, H = X.shape
    H2, N = Wt.shape
    if H2 != H:
        raise ValueError("X and Wt disagree on H")
    _need(X, "X")
    _need(Wt, "Wt")
    if Y is None:
        raise ValueError("Y must be given")
    _need(Y, "Y", shape=(T, N))
    _need(idx_out, "idx_out", torch.int32, min_numel=max(0, rmm_k_for(H, r)))
    _on_cuda(X=X, Wt=Wt, Y=Y, idx_out=idx_out)
    _check(lib().rmm_linear_decode_noalloc(_ptr(X), _ptr(Wt), T, H, N, float(r), _ptr(Y), _ptr(idx_out),
                                           _stream(stream)), "rmm_linear_decode_noalloc")
    return Y


# ---------------------------------------------------------------- decoder-layer glue

def rmm_add_rmsnorm(X: torch.Tensor, R: torch.Tensor | None = None, eps: float = 1e-5,
                    weight: torch.Tensor | None = None, Hsum: torch.Tensor | None = None,
                    Y: torch.Tensor | None = None, want_y: bool = True, stream=None):
    """Hsum = bf16(X + R); Y = bf16(RMSNorm(Hsum) * weight).  Returns (Hsum, Y); an output
    not asked for (Hsum None and R None, or want_y False) comes back as None."""
    _bf16_cuda(X, "X")
    T, H = X.shape
    if R is not None:
        _bf16_cuda(R, "R")
        if Hsum is None:
            Hsum = torch.empty_like(X)
    if want_y and Y is None:
        Y = torch.empty_like(X)
    _check(lib().rmm_add_rmsnorm(_ptr(X), _ptr(R), T, H, float(eps), _ptr(weight), _ptr(Hsum), _ptr(Y),
                                 _stream(stream)), "rmm_add_rmsnorm")
    return Hsum, Y


def rmm_swiglu(G: torch.Tensor, U: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out = bf16(silu(G) * U), elementwise."""
    _bf16_cuda(G, "G")
    _bf16_cuda(U, "U")
    if out is None:
        out = torch.empty_like(G)
    _check(lib().rmm_swiglu(_ptr(G), _ptr(U), G.numel(), _ptr(out), _stream(stream)), "rmm_swiglu")
    return out


def rmm_qkv_heads(Yq: torch.Tensor, Yk: torch.Tensor, Yv: torch.Tensor, Q: torch.Tensor, Kt: torch.Tensor,
                  V: torch.Tensor, L0: int, stream=None) -> torch.Tensor:
    """Token-major q/k/v -> Q [Hq,T,d] and the caches Kt [Hkv,d,ldL], V [Hkv,ldL,d] at L0 (batch 1)."""
    T = Yq.shape[0]
    Hq, _, d = Q.shape
    Hkv, _, ldL = Kt.shape
    _check(lib().rmm_qkv_heads(_ptr(Yq), _ptr(Yk), _ptr(Yv), T, Hq, Hkv, d, _ptr(Q), _ptr(Kt), _ptr(V), ldL,
                               int(L0), _stream(stream)), "rmm_qkv_heads")
    return Q


def rmm_heads_to_tokens(O: torch.Tensor, A: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """O [Hq, T, d] -> A [T, Hq*d]."""
    Hq, T, d = O.shape
    if A is None:
        A = torch.empty(T, Hq * d, dtype=torch.bfloat16, device=O.device)
    _check(lib().rmm_heads_to_tokens(_ptr(O), Hq, T, d, _ptr(A), _stream(stream)), "rmm_heads_to_tokens")
    return A


def rmm_selftest_exp2_fma(x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """2^x by the FMA-pipe exponential of the tensor-core softmax (fp32, elementwise)."""
    _need(x, "x", torch.float32)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", torch.float32, shape=tuple(x.shape))
    _on_cuda(x=x, y=y)
    _check(lib().rmm_selftest_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "rmm_selftest_exp2_fma")
    return y
