"""Attention over kept block pairs -- oracle (test infrastructure only), fp64.

Sources (page title, section):
  * SVG-EAR, problem statement: sparse attention computes only a subset of the
    attention blocks; 2.A: the keys and values of each block that is not
    computed exactly are replaced by the block centroid (their mean).
  * SPADE, part 3: per-head sparse attention over the chosen blocks.

Definitions (reordered, padded layout; keys at positions >= N never count):
  exact:        O_i = sum_{j in kept(I), j < N} softmax_j(q_i . k_j / sqrt(d)) v_j
  compensated:  every skipped block J contributes n_J copies of (kbar_J, vbar_J):
                O_i = [sum_kept e^{s_ij} v_j + sum_{J skipped} n_J e^{q_i.kbar_J/sqrt(d)} vbar_J]
                      / [sum_kept e^{s_ij}   + sum_{J skipped} n_J e^{q_i.kbar_J/sqrt(d)}]
  Both are materialised softmaxes (one shift by the row maximum).
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64


def _rows_of(I: int, N: int):
    lo = I * BLOCK
    return lo, min(lo + BLOCK, N)


def _kept_positions(keep_row: np.ndarray, N: int) -> np.ndarray:
    blocks = np.nonzero(keep_row)[0]
    pos = (blocks[:, None] * BLOCK + np.arange(BLOCK)[None, :]).ravel()
    return pos[pos < N]


def masked_attention(qp, kp, vp, N: int, keep: np.ndarray, q_blocks=None) -> dict:
    """Exact attention of one head ([Npad, d] arrays) restricted to kept blocks.

    keep: bool [nqb, nkb].  Returns {I: O_I fp64 [n_I, d]} for I in q_blocks
    (default: all query blocks).  Pad query rows are not produced.
    """
    d = qp.shape[-1]
    nb = qp.shape[-2] // BLOCK
    q_blocks = range(nb) if q_blocks is None else q_blocks
    out = {}
    for I in q_blocks:
        lo, hi = _rows_of(I, N)
        q = np.asarray(qp[lo:hi], dtype=np.float64)
        pos = _kept_positions(keep[I], N)
        k = np.asarray(kp[pos], dtype=np.float64)
        v = np.asarray(vp[pos], dtype=np.float64)
        s = q @ k.T / math.sqrt(d)
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[I] = p @ v
    return out


def compensated_attention(qp, kp, vp, N: int, keep: np.ndarray, kbar, vbar, nvalid,
                          q_blocks=None) -> dict:
    """Exact attention on kept blocks plus centroid terms for the skipped ones."""
    d = qp.shape[-1]
    nb = qp.shape[-2] // BLOCK
    q_blocks = range(nb) if q_blocks is None else q_blocks
    out = {}
    for I in q_blocks:
        lo, hi = _rows_of(I, N)
        q = np.asarray(qp[lo:hi], dtype=np.float64)
        pos = _kept_positions(keep[I], N)
        k = np.asarray(kp[pos], dtype=np.float64)
        v = np.asarray(vp[pos], dtype=np.float64)
        skipped = np.nonzero(~keep[I])[0]
        s_exact = q @ k.T / math.sqrt(d)
        s_cent = q @ kbar[skipped].T / math.sqrt(d) + np.log(nvalid[skipped].astype(np.float64))[None, :]
        s = np.concatenate([s_exact, s_cent], axis=1)
        vals = np.concatenate([v, vbar[skipped]], axis=0)
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[I] = p @ vals
    return out


def dense_attention(q, k, v) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v for [n, d] arrays, materialised, fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = q @ k.T / math.sqrt(q.shape[-1])
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p / p.sum(axis=1, keepdims=True)) @ v


def online_block_attention(qp, kp, vp, N: int, keep: np.ndarray, I: int) -> np.ndarray:
    """Same result as masked_attention for block I, by a running max / running sum
    over the kept key blocks in ascending order (the streaming form)."""
    d = qp.shape[-1]
    lo, hi = _rows_of(I, N)
    q = np.asarray(qp[lo:hi], dtype=np.float64)
    m = np.full(hi - lo, -np.inf)
    l = np.zeros(hi - lo)
    acc = np.zeros((hi - lo, d))
    for J in np.nonzero(keep[I])[0]:
        klo, khi = _rows_of(J, N)
        k = np.asarray(kp[klo:khi], dtype=np.float64)
        v = np.asarray(vp[klo:khi], dtype=np.float64)
        s = q @ k.T / math.sqrt(d)
        m_new = np.maximum(m, s.max(axis=1))
        scale = np.exp(m - m_new)
        p = np.exp(s - m_new[:, None])
        l = l * scale + p.sum(axis=1)
        acc = acc * scale[:, None] + p @ v
        m = m_new
    return acc / l[:, None]


def kept_flops(keep: np.ndarray, nvalid, d: int) -> float:
    """4 * d * sum over kept (I, J) of n_I * n_J (QK^T and PV, 2 flops per MAC).

    keep: bool [..., nqb, nkb]; nvalid: valid tokens per block [nb].
    """
    n = np.asarray(nvalid, dtype=np.float64)
    k = np.asarray(keep, dtype=np.float64)
    return 4.0 * d * float(np.einsum("...ij,i,j->", k, n, n))
