"""Block-mask builder -- oracle (test infrastructure only), fp64.

All arrays are in the reordered, padded layout: positions [0, Npad), of which
[0, N) hold tokens and [N, Npad) are zero pads that are never counted.  Block I
is positions [64 I, 64 I + 64); n_I is the number of its positions below N.

Sources (page title, section):
  * DFSAttn, trick 2: a block's importance estimate uses the block "average";
    finer sub-blocks are scored first and their scores are summed into the
    block score.
  * SVG-EAR, 2.A: a cluster's centroid is its mean.
  * SVOO, 2.A: the density needed to cover a cumulative attention mass (e.g.
    95%); SVG-EAR 4: "top-p" selection.
  * LVSA, abstract: structured window pattern with rotating global anchors.
  * SVG-EAR, 2.B: error-aware routing -- query centroids as proxies for the
    individual queries, compensation error estimated per block, greedy pick by
    estimated error divided by block size under a fixed density budget.

Readings taken where the method description leaves a step open:
  * pooled scores P_IJ = softmax_J(qbar_I . kbar_J / sqrt(d)) over all key
    blocks, one entry per block (no block-size weighting);
  * threshold rule: sort a row by (score desc, block index asc), keep the
    shortest prefix whose cumulative fp64 sum reaches tau (the crossing block
    is kept); tau >= 1 keeps every block;
  * top-k rule: k = ceil(keep_frac * nkb), clamped to [1, nkb], same order;
  * no block is forced (no diagonal);
  * sub-block scores: softmax over the non-empty key sub-blocks for every
    non-empty query sub-block, summed over the sub-pairs of (I, J) and divided
    by the number of non-empty query sub-blocks of I (rows still sum to 1);
  * structured window: block coordinates are the (t, h) of the block's first
    token; keep (I, J) iff |t_I - t_J| <= win_t or |h_I - h_J| <= win_rows *
    ceil(64 / W) token rows; anchors are n_anchors evenly spaced key-block
    columns (stride floor(nkb / n_anchors)) shifted by a per-step offset
    o_s = Philox4x32-10(counter = (s, 0, 0, 0), key = (seed mod 2^32,
    seed div 2^32)), first output word, mod stride -- a counter-based draw, so
    the anchors rotate with the step index s and repeat for the same seed;
  * SICS scorer (SPADE, part 2: a coherence check -- the sum of the cosine
    similarities inside a block -- decides per head and step which blocks
    are focused on; blocks whose tokens agree are kept, blocks whose tokens
    disagree are skipped): per head, key block J scores S_J = c_J / sum c with
    c_J = (sum of cos(k_i, k_j) over the pairs of J's valid keys) / n_J^2; the
    same score row serves every query block of the head, and the threshold /
    top-k rules select from it as from pooled scores;
  * routing budget m_I = the count the threshold rule keeps in row I; error
    e_IJ = || sum_{j in J} e^{s_j - M} v_j - n_J e^{qbar.kbar_J/sqrt(d) - M} vbar_J ||_2
    with s_j = qbar_I . k_j / sqrt(d), M = max_j s_j; ratio
    r_IJ = (e_IJ / Z_I) * (64 / n_J), Z_I = sum_j e^{s_j - M}; keep the m_I
    largest ratios (ties: lower block index).
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64
NEAR = 1e-5


def pool(xp: np.ndarray, N: int, size: int = BLOCK):
    """Means of the valid rows of each `size`-row group.

    xp: [..., Npad, d] (any float dtype) -> (mean fp64 [..., Npad/size, d],
    count int64 [Npad/size]); groups with no valid row get mean 0, count 0.
    """
    Npad = xp.shape[-2]
    ng = Npad // size
    x = np.asarray(xp, dtype=np.float64)
    pos = np.arange(Npad)
    valid = (pos < N).astype(np.float64)
    xs = (x * valid[:, None]).reshape(x.shape[:-2] + (ng, size, x.shape[-1])).sum(axis=-2)
    cnt = valid.reshape(ng, size).sum(axis=1).astype(np.int64)
    mean = np.where(cnt[:, None] > 0, xs / np.maximum(cnt, 1)[:, None], 0.0)
    return mean, cnt


def _softmax_rows(logits: np.ndarray) -> np.ndarray:
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=-1, keepdims=True)


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """P[..., I, J] = softmax over J of qbar_I . kbar_J / sqrt(d)."""
    d = qbar.shape[-1]
    logits = np.einsum("...id,...jd->...ij", qbar, kbar) / math.sqrt(d)
    return _softmax_rows(logits)


def subblock_scores(qp: np.ndarray, kp: np.ndarray, N: int, sub: int = 16,
                    rows=None) -> np.ndarray:
    """Block scores aggregated from `sub`-token sub-blocks (one head: [Npad, d]).

    Returns S [len(rows) or nqb, nkb]: S_IJ = (1/m_I) sum_{i in I} sum_{j in J} p_ij
    with p_ij the softmax over the non-empty key sub-blocks j of the pooled
    logits qtilde_i . ktilde_j / sqrt(d), and m_I the number of non-empty query
    sub-blocks of I.
    """
    d = qp.shape[-1]
    Npad = qp.shape[-2]
    nb = Npad // BLOCK
    per = BLOCK // sub
    qs, qc = pool(qp, N, sub)
    ks, kc = pool(kp, N, sub)
    key_ok = kc > 0
    rows = range(nb) if rows is None else rows
    out = []
    for I in rows:
        acc = np.zeros(nb)
        m = 0
        for i in range(I * per, I * per + per):
            if qc[i] == 0:
                continue
            m += 1
            lg = ks[key_ok] @ qs[i] / math.sqrt(d)
            p = np.zeros(ks.shape[0])
            e = np.exp(lg - lg.max())
            p[key_ok] = e / e.sum()
            acc += p.reshape(nb, per).sum(axis=1)
        out.append(acc / m)
    return np.array(out)


def _sorted_order(row: np.ndarray) -> np.ndarray:
    # score descending, block index ascending
    return np.lexsort((np.arange(row.shape[0]), -row))


def _score_window(row: np.ndarray, s_cut: float) -> np.ndarray:
    """Blocks whose score is within 1e-5 of the cut score -- but only when the
    window holds two or more blocks (a lone cut block cannot swap with anyone)."""
    win = np.abs(row - s_cut) <= NEAR
    if int(win.sum()) < 2:
        win[:] = False
    return win


def select_threshold(row: np.ndarray, tau: float):
    """(kept bool [nkb], near bool [nkb]) for one score row.

    Keeps the shortest prefix of the (score desc, index asc) order whose
    cumulative sum reaches tau.  `near` marks the blocks whose membership a
    1e-5 perturbation of the scores could flip: the blocks within 1e-5 of the
    crossing score (when there are two or more), and -- when a cumulative sum
    next to the crossing lies within 1e-5 of tau -- the crossing block and the
    one after it.
    """
    nkb = row.shape[0]
    kept = np.zeros(nkb, dtype=bool)
    near = np.zeros(nkb, dtype=bool)
    if tau >= 1.0:
        kept[:] = True
        return kept, near
    order = _sorted_order(row)
    csum = np.cumsum(row[order])
    reach = np.nonzero(csum >= tau)[0]
    m = int(reach[0]) + 1 if reach.size else nkb        # number kept
    kept[order[:m]] = True
    near |= _score_window(row, row[order[m - 1]])
    c_prev = csum[m - 2] if m >= 2 else 0.0
    if abs(c_prev - tau) <= NEAR or abs(csum[m - 1] - tau) <= NEAR:
        near[order[m - 1]] = True
        if m < nkb:
            near[order[m]] = True
    return kept, near


def topk_count(keep_frac: float, nkb: int) -> int:
    """k = ceil(keep_frac * nkb) clamped to [1, nkb] (keep_frac taken as float32)."""
    k = math.ceil(float(np.float32(keep_frac)) * nkb)
    return max(1, min(nkb, k))


def select_topk(row: np.ndarray, k: int):
    """(kept, near): the k largest scores, ties to the lower index."""
    nkb = row.shape[0]
    kept = np.zeros(nkb, dtype=bool)
    order = _sorted_order(row)
    kept[order[:k]] = True
    near = _score_window(row, row[order[k - 1]])
    if k == nkb:
        near[:] = False
    return kept, near


def select_rows(S: np.ndarray, mode: str, *, tau: float = 0.9, keep_frac: float = 0.25):
    """Apply a selection rule to every row of S [..., nqb, nkb] -> (kept, near) bool."""
    flat = S.reshape(-1, S.shape[-1])
    kept = np.zeros(flat.shape, dtype=bool)
    near = np.zeros(flat.shape, dtype=bool)
    k = topk_count(keep_frac, S.shape[-1])
    for r in range(flat.shape[0]):
        if mode == "threshold":
            kept[r], near[r] = select_threshold(flat[r], tau)
        elif mode == "topk":
            kept[r], near[r] = select_topk(flat[r], k)
        else:
            raise ValueError(mode)
    return kept.reshape(S.shape), near.reshape(S.shape)


# Philox4x32-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel
# random numbers: as easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64-bit
# multiplications on a 4-word counter, the 2-word key bumped by the Weyl
# constants between rounds.
_PHILOX_M = (0xD2511F53, 0xCD9E8D57)
_PHILOX_W = (0x9E3779B9, 0xBB67AE85)
_U32 = 0xFFFFFFFF


def philox4x32_10(counter, key):
    """The four 32-bit output words for a 4-word counter and a 2-word key."""
    c0, c1, c2, c3 = (int(x) & _U32 for x in counter)
    k0, k1 = (int(x) & _U32 for x in key)
    for r in range(10):
        if r > 0:
            k0 = (k0 + _PHILOX_W[0]) & _U32
            k1 = (k1 + _PHILOX_W[1]) & _U32
        p0 = _PHILOX_M[0] * c0
        p1 = _PHILOX_M[1] * c2
        c0, c1, c2, c3 = ((p1 >> 32) ^ c1 ^ k0, p1 & _U32, (p0 >> 32) ^ c3 ^ k1, p0 & _U32)
    return c0, c1, c2, c3


def anchor_offset(seed: int, step: int, nkb: int, n_anchors: int) -> int:
    """Rotation of the anchor columns at denoising step `step`, in [0, stride),
    stride = floor(nkb / n_anchors) (at least 1); 0 without anchors."""
    if n_anchors <= 0 or nkb <= 0:
        return 0
    stride = max(nkb // n_anchors, 1)
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    word = philox4x32_10((int(step), 0, 0, 0), (seed & _U32, seed >> 32))[0]
    return word % stride


def anchor_blocks(nkb: int, n_anchors: int, offset: int) -> np.ndarray:
    """Key-block columns of the rotating anchors for one step."""
    if n_anchors <= 0:
        return np.zeros(0, dtype=np.int64)
    stride = max(nkb // n_anchors, 1)
    return np.array(sorted({(offset + m * stride) % nkb for m in range(n_anchors)}), dtype=np.int64)


def structured_mask(perm: np.ndarray, T: int, H: int, W: int, *, win_t: int, win_rows: int,
                    n_anchors: int, seed: int = 0, step: int = 0, mode: str = "union") -> np.ndarray:
    """bool [nb, nb]: temporal band OR spatial band (OR anchors) on 64-token blocks,
    the anchors rotated for denoising step `step` of the run seeded `seed`.

    mode="union" is the reading used by the library; mode="intersection" keeps
    only pairs inside both bands (reported for comparison, not built on GPU).
    """
    nb = perm.shape[0] // BLOCK
    first = perm[::BLOCK]                        # raster id of each block's first token
    t, rem = np.divmod(first, H * W)
    h = rem // W
    R = win_rows * ((BLOCK + W - 1) // W)
    dt = np.abs(t[:, None] - t[None, :]) <= win_t
    dh = np.abs(h[:, None] - h[None, :]) <= R
    keep = (dt | dh) if mode == "union" else (dt & dh)
    keep = keep.copy()
    keep[:, anchor_blocks(nb, n_anchors, anchor_offset(seed, step, nb, n_anchors))] = True
    return keep


def sics_coherence(kp: np.ndarray, N: int) -> np.ndarray:
    """Block coherence c [nb] of one head's keys ([Npad, d], reordered).

    SPADE, part 2: the sum of intra-block cosine similarities.  Written out as
    the definition: SICS_J = sum over all ordered pairs (i, j) of valid keys of
    block J of cos(k_i, k_j) (the i = j terms included; a zero key has cosine
    0 with every key), and c_J = SICS_J / n_J^2; a block with no valid key has
    c = 0.
    """
    Npad = kp.shape[-2]
    nb = Npad // BLOCK
    x = np.asarray(kp, dtype=np.float64)
    out = np.zeros(nb)
    for J in range(nb):
        rows = [r for r in range(J * BLOCK, min(J * BLOCK + BLOCK, N))]
        n = len(rows)
        if n == 0:
            continue
        blk = x[rows]
        norms = np.sqrt((blk * blk).sum(axis=1))
        total = 0.0
        for i in range(n):
            if norms[i] == 0.0:
                continue
            # cos(k_i, k_j) for every j of the block (zero keys contribute 0)
            dots = blk @ blk[i]
            ok = norms > 0.0
            total += float((dots[ok] / (norms[i] * norms[ok])).sum())
        out[J] = total / (n * n)
    return out


def sics_scores(kp: np.ndarray, N: int) -> np.ndarray:
    """S [nb] = c_J / sum_J' c_J' for one head (all zero if every c is 0): the
    score every query block of the head ranks the key blocks by under the
    SICS scorer."""
    c = sics_coherence(kp, N)
    tot = c.sum()
    return c / tot if tot > 0 else np.zeros_like(c)


def route_ratios(qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, N: int, rows=None) -> np.ndarray:
    """Error-to-size ratios r [len(rows), nkb] for one head ([Npad, d] arrays)."""
    d = qp.shape[-1]
    qbar, n = pool(qp, N)
    kbar, _ = pool(kp, N)
    vbar, _ = pool(vp, N)
    nb = qbar.shape[0]
    K = np.asarray(kp[:N], dtype=np.float64)
    V = np.asarray(vp[:N], dtype=np.float64)
    blk = np.arange(N) // BLOCK
    rows = range(nb) if rows is None else rows
    out = []
    for I in rows:
        s = K @ qbar[I] / math.sqrt(d)
        M = s.max()
        e = np.exp(s - M)
        Z = e.sum()
        exact = np.zeros((nb, d))
        np.add.at(exact, blk, e[:, None] * V)
        cent = (n * np.exp(kbar @ qbar[I] / math.sqrt(d) - M))[:, None] * vbar
        err = np.linalg.norm(exact - cent, axis=1)
        out.append(err / Z * (BLOCK / n))
    return np.array(out)


def select_routing(r: np.ndarray, budget: int):
    """(kept, near): the `budget` largest ratios, ties to the lower index."""
    return select_topk(r, budget)


def mask_from_rows(kept: np.ndarray):
    """Compacted lists: (kv_idx list of ascending arrays, kv_cnt) from bool rows."""
    flat = kept.reshape(-1, kept.shape[-1])
    idx = [np.nonzero(r)[0] for r in flat]
    cnt = np.array([len(i) for i in idx], dtype=np.int64).reshape(kept.shape[:-1])
    return idx, cnt
