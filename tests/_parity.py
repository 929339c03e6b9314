"""Helpers for the GPU-vs-oracle parity tests (the oracle side composes
`oracle/` functions; the GPU side calls only the C ABI through the binding)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
from block_sparse_attention_hilbert_b200 import SparseVideoAttention

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def gpu_layer(w: workloads.Workload, q, k, v, *, step=0, seed=0, keep_bits=True, compensate=None):
    """Run the four library calls for workload `w` on cuda tensors at denoising
    step `step` of a run seeded `seed`; return the object."""
    comp = w.compensate if compensate is None else compensate
    attn = SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select,
                                tau=w.tau, keep_frac=w.keep_frac, sub_block=w.sub_block, win_t=w.win_t,
                                win_rows=w.win_rows, n_anchors=w.n_anchors if w.select == "structured" else 0,
                                routing=w.routing, compensate=comp, keep_bits=keep_bits, seed=seed,
                                scorer=w.scorer, device="cuda")
    out = attn(q, k, v, step=step)
    torch.cuda.synchronize()
    attn.out = out
    return attn


def gpu_keep(attn) -> np.ndarray:
    """bool [B*heads, nb, nb] from the compacted lists (also checks list sanity)."""
    b = attn.buf
    idx = b.kv_idx.cpu().numpy().reshape(-1, attn.nb, b.cap)
    cnt = b.kv_cnt.cpu().numpy().reshape(-1, attn.nb)
    keep = np.zeros((idx.shape[0], attn.nb, attn.nb), dtype=bool)
    for bh in range(idx.shape[0]):
        for I in range(attn.nb):
            lst = idx[bh, I, :cnt[bh, I]]
            assert 1 <= cnt[bh, I] <= attn.nb
            assert np.all(np.diff(lst) > 0), "kv list must be strictly ascending"
            assert lst.min() >= 0 and lst.max() < attn.nb
            keep[bh, I, lst] = True
    if b.bits is not None:
        bits = b.bits.cpu().numpy().view(np.uint32).reshape(idx.shape[0], attn.nb, -1)
        unpacked = ((bits[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
        unpacked = unpacked.reshape(idx.shape[0], attn.nb, -1)[..., :attn.nb]
        assert np.array_equal(unpacked, keep), "bit rows disagree with kv lists"
    return keep


def oracle_rows(w: workloads.Workload, qp, kp, vp, perm, rows, step=0, seed=0):
    """Oracle (kept, near) for query-block rows `rows` of one head ([Npad, d] fp64)."""
    N = w.N
    if w.select == "structured":
        keep = oracle.structured_mask(perm, w.T, w.H, w.W, win_t=w.win_t, win_rows=w.win_rows,
                                      n_anchors=w.n_anchors, seed=seed, step=step)
        return keep[rows], np.zeros((len(rows), keep.shape[1]), dtype=bool)
    if w.scorer == "sics":
        S = np.tile(oracle.sics_scores(kp, N), (len(rows), 1))
        return oracle.select_rows(S, w.select, tau=w.tau, keep_frac=w.keep_frac)
    if w.sub_block == 64:
        qb, _ = oracle.pool(qp, N)
        kb, _ = oracle.pool(kp, N)
        S = oracle.block_scores(qb[rows], kb)
    else:
        S = oracle.subblock_scores(qp, kp, N, w.sub_block, rows=rows)
    if not w.routing:
        return oracle.select_rows(S, w.select, tau=w.tau, keep_frac=w.keep_frac)
    r = oracle.route_ratios(qp, kp, vp, N, rows=rows)
    kept = np.zeros(S.shape, dtype=bool)
    near = np.zeros(S.shape, dtype=bool)
    for i in range(len(rows)):
        thr_kept, thr_near = oracle.select_threshold(S[i], w.tau)
        m = int(thr_kept.sum())
        kept[i], near[i] = oracle.select_routing(r[i], m)
        # a budget that a 1e-5 change could move by one flips the m-th / (m+1)-th ratio
        order = np.lexsort((np.arange(r.shape[1]), -r[i]))
        if thr_near.any():
            near[i, order[m - 1]] = True
            if m < r.shape[1]:
                near[i, order[m]] = True
    return kept, near


def compare_mask_rows(gkeep_rows, okept, onear):
    """Rows must agree outside the near set; returns (#near blocks, #differing blocks)."""
    diff = gkeep_rows ^ okept
    assert not np.any(diff & ~onear), f"mask mismatch outside near-threshold set: {np.argwhere(diff & ~onear)[:8]}"
    return int(onear.sum()), int(diff.sum())


def check_attention(gout: np.ndarray, ref: np.ndarray, what=""):
    err = np.abs(gout - ref)
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e} > {MAX_ABS}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean-abs {err.mean():.3e} > {MEAN_ABS}"
    return float(err.max()), float(err.mean())
