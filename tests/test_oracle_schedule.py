"""Pins of the step-schedule oracle (DFSAttn trick 3, SVOO 2.B)."""
import numpy as np
import pytest

import oracle
import workloads


def test_dense_steps_keep_everything_then_endpoints():
    n, dense = 50, 5
    assert all(oracle.step_param(n, dense, 0.97, 0.85, s) == 1.0 for s in range(dense))
    assert oracle.step_param(n, dense, 0.97, 0.85, dense) == float(np.float32(0.97))
    assert oracle.step_param(n, dense, 0.97, 0.85, n - 1) == float(np.float32(0.85))


def test_linear_in_between_and_degenerate_span():
    # midpoint of an odd span is the exact average; a one-step span stays at `start`
    n, dense = 11, 0
    assert oracle.step_param(n, dense, 0.5, 0.3, 5) == float(np.float32(0.4))
    assert oracle.step_param(3, 2, 0.9, 0.1, 2) == float(np.float32(0.9))
    vals = [oracle.step_param(30, 3, 0.99, 0.8, s) for s in range(3, 30)]
    assert all(a >= b for a, b in zip(vals, vals[1:]))          # monotone towards `end`


@pytest.mark.parametrize("n,dense,every", [(20, 4, 5), (10, 0, 3), (7, 7, 2), (12, 3, 1)])
def test_rebuild_pattern_closed_form(n, dense, every):
    r = oracle.rebuilds(n, dense, every)
    expect = [s == 0 or (s >= dense and (s - dense) % every == 0) for s in range(n)]
    assert r == expect
    src = oracle.mask_steps(n, dense, every)
    for s in range(n):
        assert src[s] == max(t for t in range(s + 1) if r[t])


def test_scheduled_masks_get_sparser_on_fixed_inputs():
    # on fixed inputs a falling tau keeps no more blocks at a later rebuild
    w = workloads.WORKLOADS["tiny"].with_(T=4, H=16, W=16)
    q, k, v = (t[0, 0].float().numpy().astype(np.float64) for t in workloads.make_qkv(w))
    perm, _ = oracle.build_perm(w.T, w.H, w.W, "hilbert")
    qp, kp = oracle.reorder(q, perm), oracle.reorder(k, perm)
    qb, _ = oracle.pool(qp, w.N)
    kb, _ = oracle.pool(kp, w.N)
    S = oracle.block_scores(qb, kb)
    kept = []
    for s in range(12):
        tau = oracle.step_param(12, 2, 0.99, 0.6, s)
        keep, _ = oracle.select_rows(S, "threshold", tau=tau)
        kept.append(int(keep.sum()))
    assert kept[0] == kept[1] == S.size                       # dense steps
    assert all(a >= b for a, b in zip(kept[2:], kept[3:]))
    assert kept[-1] < kept[2]
