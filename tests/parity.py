"""Parity helpers shared by the GPU tests: tolerances and sampling.

The float bar (reduced products and attention outputs, fp32 accumulation and
bf16 output against the fp64 oracle):
    ||Y - Y_oracle||_F <= 5e-3 * ||Y_oracle||_F   and
    max |Y - Y_oracle| <= 1e-2 * max |Y_oracle|.
Kept index sets must match bit for bit.
"""
import numpy as np
import torch

REL_FRO = 5e-3
MAX_ABS_FRAC = 1e-2


def assert_close(y_gpu, y_ref, what=""):
    y = y_gpu.detach().to("cpu", torch.float64).numpy() if torch.is_tensor(y_gpu) else np.asarray(y_gpu, np.float64)
    ref = np.asarray(y_ref, np.float64)
    assert y.shape == ref.shape, (what, y.shape, ref.shape)
    d = y - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(d) / nref if nref > 0 else np.linalg.norm(d)
    mx = float(np.abs(d).max()) if d.size else 0.0
    lim = MAX_ABS_FRAC * float(np.abs(ref).max()) if ref.size else 0.0
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mx <= lim, f"{what}: max abs error {mx:.3e} > {lim:.3e}"
    return rel, mx


def sample_indices(n, count, seed):
    """Sorted sample of `count` indices in [0, n) that always includes 0 and n-1."""
    if n <= count:
        return np.arange(n, dtype=np.int64)
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n, size=count - 2, replace=False).tolist())
    pick.update([0, n - 1])
    return np.array(sorted(pick), dtype=np.int64)


def bits_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def tile_rows(T, tile=128, seed=0):
    """One row in every `tile`-row tile (at a seeded offset), plus the first and last rows."""
    rng = np.random.default_rng(seed)
    rows = {0, T - 1}
    for t0 in range(0, T, tile):
        rows.add(int(t0 + rng.integers(0, min(tile, T - t0))))
    return np.array(sorted(rows), dtype=np.int64)


def row_head_pairs(rows, Hq, Hkv, heads_per_row=1):
    """(row, query head) pairs to check: each row on `heads_per_row` heads, rotating over
    the KV groups and over the heads inside a group, so the sample touches every group."""
    G = Hq // Hkv
    pairs = []
    for i, t in enumerate(rows):
        for j in range(heads_per_row):
            g = (i * heads_per_row + j) % Hkv
            pairs.append((int(t), g * G + (i + j) % G))
    return pairs
