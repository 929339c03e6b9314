"""Whole-head oracle evaluation for the full-size parity tests (one head per
call).  Imports only numpy and `oracle/`: it never touches torch or the GPU."""
from __future__ import annotations

import numpy as np

import oracle


def head_parity(task):
    """One head of a layer: the oracle's mask (kept, near) over every query
    block, compared with the GPU's, and the oracle's exact attention on the
    GPU's own mask compared with the GPU's output.

    task: dict with qp, kp, vp ([Npad, d] fp64, reordered), gkeep (bool
    [nb, nb], the GPU mask), gop ([Npad, d], the GPU output), N, select, tau,
    keep_frac, sub_block.  Returns counts and error statistics; raises if a
    mask differs outside the near set.
    """
    qp, kp, vp, gkeep, gop = task["qp"], task["kp"], task["vp"], task["gkeep"], task["gop"]
    N = task["N"]
    nb = qp.shape[0] // 64
    if task["sub_block"] == 64:
        qb, _ = oracle.pool(qp, N)
        kb, _ = oracle.pool(kp, N)
        S = oracle.block_scores(qb, kb)
    else:
        S = oracle.subblock_scores(qp, kp, N, task["sub_block"])
    kept, near = oracle.select_rows(S, task["select"], tau=task["tau"], keep_frac=task["keep_frac"])
    diff = gkeep ^ kept
    bad = diff & ~near
    if bad.any():
        raise AssertionError(f"mask differs outside the near-threshold set at {np.argwhere(bad)[:8].tolist()}")
    ref = oracle.masked_attention(qp, kp, vp, N, gkeep)
    errs = []
    for I in range(nb):
        lo, hi = I * 64, min(I * 64 + 64, N)
        errs.append(np.abs(gop[lo:hi] - ref[I]))
    err = np.concatenate(errs)
    return {"near": int(near.sum()), "differing": int(diff.sum()), "max_abs": float(err.max()),
            "sum_abs": float(err.sum()), "count": int(err.size), "pads_zero": bool(np.all(gop[N:] == 0))}
