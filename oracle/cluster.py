"""Bidirectional query-key co-clustering order -- oracle (test infrastructure only).

Sources (page title, section):
  * "Training-Free Sparse Attention for Fast Video Generation via Offline
    Layer-Wise Sparsity Profiling and Online Bidirectional Co-Clustering"
    (SVOO), technical summary 2.B: instead of clustering queries and keys
    separately, alternate (1) a query-aware partition of the keys -- keys are
    grouped by their affinity to the current query centroids -- and (2) a
    key-aware partition of the queries -- queries are grouped by their
    affinity to the updated key centroids; the refined partitions give
    aligned Q and K blocks; the result is reused for a number of diffusion
    steps.
  * "SVG-EAR", 2.A: tokens are grouped semantically and permuted so that
    similar tokens are contiguous in memory, forming the block structure.

Readings taken where the method description leaves a step open:
  * per (batch, head), C = nb clusters (as many as 64-token blocks);
  * affinity = the dot product q . k (the attention logit up to its 1/sqrt(d)
    scale), taken exactly: bf16 token values and float32 centroids, products
    and sums in float64 (the value that decides each argmax); ties go to the
    lower cluster index;
  * initial query centroids: the means of the 64-token blocks of the raster
    order (valid tokens only);
  * a centroid is the float32 rounding of the exact mean of its tokens (the
    float64 sum of bf16 values is exact); an empty key cluster takes the query
    centroid of the same index, an empty query cluster the key centroid;
  * one round = key assignment, key centroids, query assignment, query
    centroids; `rounds` rounds (3 by default);
  * order: queries sorted by (cluster, raster index), keys likewise -- a
    permutation for Q and one for K and V, pads at the end as for the other
    orders; the output is gathered back with the query permutation.
"""
from __future__ import annotations

import math

import numpy as np

from .order import _pad, BLOCK


def _means(x: np.ndarray, assign: np.ndarray, C: int, fallback: np.ndarray) -> np.ndarray:
    """float32 centroids: exact float64 sums of the members, divided, rounded."""
    sums = np.zeros((C, x.shape[1]), dtype=np.float64)
    np.add.at(sums, assign, x)
    cnt = np.bincount(assign, minlength=C).astype(np.float64)
    out = fallback.copy()
    nz = cnt > 0
    out[nz] = (sums[nz] / cnt[nz, None]).astype(np.float32)
    return out


def _assign(x: np.ndarray, cent: np.ndarray):
    """argmax_j x . c_j (first index on ties) and the top-2 gap, decided on the
    exact affinities.  The products of a bf16 and a float32 value are exact in
    float64, so only the summation rounds: whatever its order, an fp64 dot
    product of length d is within gamma_d * sum_i |x_i c_i| of the exact value
    (gamma_d = d u / (1 - d u), u = 2^-53).  Every centroid whose interval
    reaches the best one's is a candidate; rows with two or more candidates
    are re-decided on the correctly rounded exact sums (math.fsum), so that
    equal centroids always give equal affinities and a cancellation cannot
    flip the argmax."""
    c64 = cent.astype(np.float64)
    a = x @ c64.T
    d = x.shape[1]
    u = 2.0 ** -53
    # twice the a-priori bound: the bound itself is evaluated in fp64
    err = 2.0 * (d * u / (1.0 - d * u)) * (np.abs(x) @ np.abs(c64).T)
    best = np.argmax(a, axis=1)
    rows = np.arange(a.shape[0])
    close = (a + err) >= (a[rows, best] - err[rows, best])[:, None]
    for t in np.nonzero(close.sum(axis=1) > 1)[0]:
        cand = np.nonzero(close[t])[0]
        exact = [math.fsum(x[t] * c64[j]) for j in cand]
        a[t, cand] = exact
        best[t] = cand[int(np.argmax(exact))]
    top = a[rows, best]
    if a.shape[1] > 1:
        a2 = a.copy()
        a2[rows, best] = -np.inf
        gap = top - a2.max(axis=1)
    else:
        gap = np.full(a.shape[0], np.inf)
    return best, gap


def initial_centroids(q: np.ndarray, N: int) -> np.ndarray:
    """float32 means of the raster 64-token blocks of q ([N, d])."""
    nb = (N + BLOCK - 1) // BLOCK
    blk = np.arange(N) // BLOCK
    return _means(np.asarray(q, dtype=np.float64), blk, nb, np.zeros((nb, q.shape[1]), np.float32))


def cocluster(q: np.ndarray, k: np.ndarray, N: int, rounds: int = 3):
    """Cluster ids of the N queries and N keys of one head ([N, d] bf16-valued
    arrays), and the last round's top-2 affinity gaps (for reporting)."""
    q = np.asarray(q[:N], dtype=np.float64)
    k = np.asarray(k[:N], dtype=np.float64)
    cq = initial_centroids(q, N)
    C = cq.shape[0]
    aq = ak = None
    gq = gk = None
    for _ in range(rounds):
        ak, gk = _assign(k, cq)
        ck = _means(k, ak, C, cq)
        aq, gq = _assign(q, ck)
        cq = _means(q, aq, C, ck)
    return aq, ak, gq, gk


def perm_from_clusters(assign: np.ndarray, N: int):
    """(perm [Npad], iperm [N]): tokens sorted by (cluster, raster index)."""
    order = np.lexsort((np.arange(N), assign[:N]))
    return _pad(order.astype(np.int64), N)
