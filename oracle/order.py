"""Token orderings of the (T, H, W) latent grid -- oracle (test infrastructure only).

Source: "DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation", trick 1: tokens normally sit in raster order (row by row); a 3D
Hilbert curve re-threads them so that neighbours in the sequence are
neighbours in space and time, which makes each contiguous block coherent.

Reading (the page gives no construction): the grid is embedded in the
smallest enclosing cube of side 2^k, k = ceil(log2(max(T, H, W))); each cell's
position on the Hilbert curve of that cube is computed with Skilling's
transpose method (J. Skilling, "Programming the Hilbert curve", AIP Conf.
Proc. 707, 2004) using axes (X0, X1, X2) = (t, h, w); the N valid cells are
then ordered by that key (keys are distinct, so there are no ties).  The
sequence is padded at its end to a multiple of the 64-token block; pad
positions map to raster id -1.
"""
from __future__ import annotations

import numpy as np

BLOCK = 64


def hilbert_key_3d(t, h, w, k: int) -> np.ndarray:
    """Hilbert-curve index of cells (t, h, w) in the 2^k cube (int64, vectorised).

    Skilling's method in two stages, written out for three axes:
      1. Axes -> "transpose" form.  From the top bit plane Q = 2^(k-1) down to
         Q = 2, with low mask P = Q - 1, visit the axes in order i = 0, 1, 2:
         if bit Q of axis i is set, invert the low bits of axis 0; otherwise
         exchange the low bits of axis 0 and axis i.  Then Gray-encode: each
         axis i >= 1 is xor-ed with axis i-1, and every axis is xor-ed with the
         mask t accumulated from the set bits Q > 1 of the last axis (t ^= Q-1).
      2. The index is the bit interleave of the transposed axes, most
         significant bit plane first, axis 0 first within a plane.
    """
    X = [np.asarray(t, dtype=np.int64).copy(), np.asarray(h, dtype=np.int64).copy(),
         np.asarray(w, dtype=np.int64).copy()]
    n = 3
    if k <= 0:
        return np.zeros_like(X[0])
    top = 1 << (k - 1)
    Q = top
    while Q > 1:
        P = Q - 1
        for i in range(n):
            bit_set = (X[i] & Q) != 0
            if i == 0:
                # exchanging axis 0 with itself is a no-op: only the inversion applies
                X[0] = np.where(bit_set, X[0] ^ P, X[0])
                continue
            swap = (X[0] ^ X[i]) & P
            new0 = np.where(bit_set, X[0] ^ P, X[0] ^ swap)
            newi = np.where(bit_set, X[i], X[i] ^ swap)
            X[0], X[i] = new0, newi
        Q >>= 1
    for i in range(1, n):
        X[i] = X[i] ^ X[i - 1]
    tmask = np.zeros_like(X[0])
    Q = top
    while Q > 1:
        tmask = np.where((X[n - 1] & Q) != 0, tmask ^ (Q - 1), tmask)
        Q >>= 1
    for i in range(n):
        X[i] = X[i] ^ tmask
    key = np.zeros_like(X[0])
    for b in range(k - 1, -1, -1):
        for i in range(n):
            key = (key << 1) | ((X[i] >> b) & 1)
    return key


def _grid(T: int, H: int, W: int):
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    return t.ravel(), h.ravel(), w.ravel()


def _pad(order_ids: np.ndarray, N: int):
    nb = (N + BLOCK - 1) // BLOCK
    perm = np.full(nb * BLOCK, -1, dtype=np.int64)
    perm[:N] = order_ids
    iperm = np.empty(N, dtype=np.int64)
    iperm[order_ids] = np.arange(N)
    return perm, iperm


def perm_raster(T: int, H: int, W: int):
    """Raster order: position i holds raster token i = (t*H + h)*W + w."""
    N = T * H * W
    return _pad(np.arange(N, dtype=np.int64), N)


def perm_hilbert(T: int, H: int, W: int):
    """Hilbert order: valid cells sorted by their key in the enclosing 2^k cube."""
    N = T * H * W
    k = int(np.ceil(np.log2(max(T, H, W)))) if max(T, H, W) > 1 else 0
    t, h, w = _grid(T, H, W)
    key = hilbert_key_3d(t, h, w, k)
    ids = np.argsort(key, kind="stable")          # raster ids in curve order
    return _pad(ids.astype(np.int64), N)


def build_perm(T: int, H: int, W: int, order: str):
    """(perm [Npad] position -> raster id or -1, iperm [N] raster id -> position)."""
    if order == "raster":
        return perm_raster(T, H, W)
    if order == "hilbert":
        return perm_hilbert(T, H, W)
    raise ValueError(order)


def reorder(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """X_p[..., i, :] = X[..., perm[i], :]; pad rows (perm = -1) are zero."""
    out = np.zeros(x.shape[:-2] + (perm.shape[0], x.shape[-1]), dtype=x.dtype)
    valid = perm >= 0
    out[..., valid, :] = x[..., perm[valid], :]
    return out


def inverse_reorder(xp: np.ndarray, perm: np.ndarray, N: int) -> np.ndarray:
    """X[..., perm[i], :] = X_p[..., i, :] for the valid positions i."""
    out = np.zeros(xp.shape[:-2] + (N, xp.shape[-1]), dtype=xp.dtype)
    valid = perm >= 0
    out[..., perm[valid], :] = xp[..., valid, :]
    return out


def locality_stats(perm: np.ndarray, T: int, H: int, W: int) -> dict:
    """Fraction of unit steps and mean L1 jump between consecutive positions."""
    ids = perm[perm >= 0]
    t, rem = np.divmod(ids, H * W)
    h, w = np.divmod(rem, W)
    jump = np.abs(np.diff(t)) + np.abs(np.diff(h)) + np.abs(np.diff(w))
    return {"unit_frac": float(np.mean(jump == 1)) if jump.size else 1.0,
            "mean_l1": float(np.mean(jump)) if jump.size else 0.0}
