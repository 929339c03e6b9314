"""Pins for the oracle's mask builder (no GPU)."""
import itertools
import math

import numpy as np
import pytest

import oracle
from oracle.mask import NEAR


def test_pool_constant_and_pads():
    N, d = 100, 3                                   # two blocks, second has 36 valid rows
    xp = np.zeros((128, d))
    xp[:64] = 2.0
    xp[64:N] = -1.5
    xp[N:] = 1e9                                   # pads must never count
    mean, cnt = oracle.pool(xp, N)
    assert cnt.tolist() == [64, 36]
    assert np.allclose(mean[0], 2.0) and np.allclose(mean[1], -1.5)


def test_pool_ramp_closed_form():
    # mean of 0..63 is 31.5; of 64..99 is 81.5
    N = 100
    xp = np.arange(128, dtype=np.float64)[:, None] * np.ones((1, 2))
    mean, _ = oracle.pool(xp, N)
    assert mean[0, 0] == 31.5 and mean[1, 1] == 81.5


def test_scores_d1_hand_case(golden):
    expect = golden("softmax_d1.txt")[0]
    P = oracle.block_scores(np.array([[1.0]]), np.array([[0.0], [1.0], [2.0]]))
    assert np.allclose(P[0], expect, rtol=0, atol=1e-15)


def test_scores_rows_sum_to_one():
    rng = np.random.default_rng(1)
    P = oracle.block_scores(rng.standard_normal((2, 7, 16)), rng.standard_normal((2, 9, 16)))
    assert P.shape == (2, 7, 9)
    assert np.allclose(P.sum(-1), 1.0, atol=1e-14)


def test_subblock_of_64_equals_block_scores():
    rng = np.random.default_rng(2)
    N, d = 200, 8
    qp = np.zeros((256, d)); kp = np.zeros((256, d))
    qp[:N] = rng.standard_normal((N, d)); kp[:N] = rng.standard_normal((N, d))
    S = oracle.subblock_scores(qp, kp, N, sub=64)
    qb, _ = oracle.pool(qp, N); kb, _ = oracle.pool(kp, N)
    assert np.allclose(S, oracle.block_scores(qb, kb), atol=1e-15)


def test_subblock_rows_sum_to_one_and_skip_empty():
    rng = np.random.default_rng(3)
    N, d = 200, 8                                   # 200 = 12.5 sub-blocks of 16: last one empty
    qp = np.zeros((256, d)); kp = np.zeros((256, d))
    qp[:N] = rng.standard_normal((N, d)); kp[:N] = rng.standard_normal((N, d))
    S = oracle.subblock_scores(qp, kp, N, sub=16)
    assert np.allclose(S.sum(-1), 1.0, atol=1e-14)
    # brute force for block row 3 (sub-blocks 12 (8 valid) .. 15 (empty))
    qs, qc = oracle.pool(qp, N, 16); ks, kc = oracle.pool(kp, N, 16)
    acc = np.zeros(4); m = 0
    for i in range(12, 16):
        if qc[i] == 0:
            continue
        m += 1
        lg = np.array([qs[i] @ ks[j] / math.sqrt(d) if kc[j] else -np.inf for j in range(16)])
        p = np.exp(lg - lg.max()); p /= p.sum()
        for j in range(16):
            acc[j // 4] += p[j]
    assert m == 1
    assert np.allclose(S[3], acc / m, atol=1e-15)


def _brute_threshold(row, tau):
    n = len(row)
    for m in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), m):
            mass = sum(row[list(sub)])
            if mass >= tau and (best is None or mass > best[0]):
                best = (mass, sub)
        if best is not None:
            return set(best[1])
    return set(range(n))


def _brute_topk(row, k):
    best = max(itertools.combinations(range(len(row)), k), key=lambda s: sum(row[list(s)]))
    return set(best)


@pytest.mark.parametrize("seed", range(12))
def test_threshold_is_minimal_max_mass_subset(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 9))
    row = rng.dirichlet(np.ones(n) * 0.7)
    for tau in (0.3, 0.5, 0.9, 0.95):
        kept, _ = oracle.select_threshold(row, tau)
        assert set(np.nonzero(kept)[0]) == _brute_threshold(row, tau)


@pytest.mark.parametrize("seed", range(8))
def test_topk_is_max_mass_subset(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 9))
    row = rng.dirichlet(np.ones(n))
    for k in range(1, n + 1):
        kept, _ = oracle.select_topk(row, k)
        assert set(np.nonzero(kept)[0]) == _brute_topk(row, k)


def test_ties_go_to_lower_index():
    row = np.array([0.25, 0.25, 0.25, 0.25])
    kept, _ = oracle.select_threshold(row, 0.5)
    assert kept.tolist() == [True, True, False, False]
    kept, _ = oracle.select_topk(row, 3)
    assert kept.tolist() == [True, True, True, False]


def test_keep_all_cases():
    row = np.array([0.1, 0.6, 0.3])
    assert oracle.select_threshold(row, 1.0)[0].all()
    assert oracle.select_topk(row, 3)[0].all()
    assert oracle.topk_count(0.25, 512) == 128
    assert oracle.topk_count(0.0, 10) == 1 and oracle.topk_count(2.0, 10) == 10
    assert oracle.select_threshold(row, 0.0)[0].tolist() == [False, True, False]


def test_near_threshold_flags():
    # sorted: 0.5 (idx1), 0.3 (idx2), 0.2 (idx0); tau just above 0.8 -> crossing at idx0
    row = np.array([0.2, 0.5, 0.3])
    kept, near = oracle.select_threshold(row, 0.8 + 1e-7)
    assert kept.tolist() == [True, True, True]
    assert near[0] and not near[1]
    kept, near = oracle.select_threshold(row, 0.6)
    assert kept.tolist() == [False, True, True] and not near.any()
    # equal-within-1e-5 scores around the top-k cut are both flagged
    row = np.array([0.4, 0.3 + 2e-6, 0.3 - 2e-6])
    kept, near = oracle.select_topk(row, 2)
    assert kept.tolist() == [True, True, False] and near.tolist() == [False, True, True]


def test_structured_hand_case(golden):
    expect = np.array(golden("structured_3x8x16.txt"), dtype=bool)
    perm, _ = oracle.perm_raster(3, 8, 16)
    keep = oracle.structured_mask(perm, 3, 8, 16, win_t=0, win_rows=0, n_anchors=0)
    assert np.array_equal(keep, expect)


def test_structured_symmetry_and_anchors():
    perm, _ = oracle.perm_raster(12, 10, 20)
    base = oracle.structured_mask(perm, 12, 10, 20, win_t=2, win_rows=1, n_anchors=0)
    assert np.array_equal(base, base.T)
    nb = base.shape[0]
    for seed, step in ((0, 0), (0, 1), (5, 3), (2**40 + 7, 11)):
        keep = oracle.structured_mask(perm, 12, 10, 20, win_t=2, win_rows=1, n_anchors=4, seed=seed, step=step)
        cols = oracle.anchor_blocks(nb, 4, oracle.anchor_offset(seed, step, nb, 4))
        assert keep[:, cols].all()
        extra = keep & ~base
        assert set(np.nonzero(extra.any(axis=0))[0]) <= set(cols.tolist())
    # anchors are evenly spaced, stride floor(nb/4)
    a = oracle.anchor_blocks(37, 4, 2)
    assert a.tolist() == [2, 11, 20, 29]


def _hex_rows(name):
    import os
    rows = []
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(x, 16) for x in line.split()])
    return rows


def test_philox_known_answers():
    # Random123's published philox4x32-10 vectors: a dropped round, a wrong
    # multiplier, Weyl constant or word order fails at least one of them
    for row in _hex_rows("philox4x32_10_kat.txt"):
        ctr, key, out = row[:4], row[4:6], row[6:]
        assert list(oracle.philox4x32_10(ctr, key)) == out


def test_anchor_offset_closed_form_and_range():
    # seed 0, step 0: counter and key all zero, so the offset is the first
    # known-answer word 0x6627e8d5 = 1713891541 modulo the stride
    assert oracle.anchor_offset(0, 0, 3072, 4) == 1713891541 % 768 == 469
    assert oracle.anchor_offset(0, 0, 512, 4) == 1713891541 % 128
    assert oracle.anchor_offset(0, 0, 3, 4) == 0          # stride clamps to 1
    assert oracle.anchor_offset(9, 9, 512, 0) == 0        # no anchors
    rng = np.random.default_rng(3)
    for _ in range(300):
        nkb = int(rng.integers(1, 5000))
        n = int(rng.integers(1, 9))
        off = oracle.anchor_offset(int(rng.integers(0, 2**63)), int(rng.integers(0, 2**31)), nkb, n)
        assert 0 <= off < max(nkb // n, 1)


def test_anchors_rotate_with_the_step_and_repeat_for_the_seed():
    nkb, n = 3072, 4
    stride = nkb // n
    offs = [oracle.anchor_offset(0, s, nkb, n) for s in range(64)]
    # a counter-based draw: the same (seed, step) gives the same anchors ...
    assert offs == [oracle.anchor_offset(0, s, nkb, n) for s in range(64)]
    # ... the anchors move from step to step (64 draws from 768 values) ...
    assert len(set(offs)) > 55
    assert all(offs[s] != offs[s + 1] for s in range(8))
    # ... each step's columns stay evenly spaced, one per stride ...
    for s in range(4):
        cols = oracle.anchor_blocks(nkb, n, offs[s])
        assert np.all(np.diff(cols) == stride) and cols[0] == offs[s]
    # ... and another seed gives another rotation
    assert [oracle.anchor_offset(1, s, nkb, n) for s in range(8)] != offs[:8]
    # the 64-bit seed enters both key words
    assert oracle.anchor_offset(2**32, 0, nkb, n) != oracle.anchor_offset(0, 0, nkb, n)
    assert oracle.anchor_offset(1, 0, nkb, n) != oracle.anchor_offset(0, 0, nkb, n)


def test_structured_density_readings():
    # the long-horizon grid: union reading ~19%, intersection far sparser
    T, H, W = 126, 30, 52
    perm, _ = oracle.perm_raster(T, H, W)
    u = oracle.structured_mask(perm, T, H, W, win_t=2, win_rows=1, n_anchors=0)
    x = oracle.structured_mask(perm, T, H, W, win_t=2, win_rows=1, n_anchors=0, mode="intersection")
    assert 0.17 < u.mean() < 0.22
    assert x.mean() < 0.02


def _routing_inputs(rng, N, d, const_k=False, const_v=False):
    Npad = -(-N // 64) * 64
    qp = np.zeros((Npad, d)); kp = np.zeros((Npad, d)); vp = np.zeros((Npad, d))
    qp[:N] = rng.standard_normal((N, d))
    kp[:N] = rng.standard_normal((N, d))
    vp[:N] = rng.standard_normal((N, d))
    for J in range(Npad // 64):
        lo, hi = J * 64, min(J * 64 + 64, N)
        if const_k:
            kp[lo:hi] = rng.standard_normal(d)
        if const_v:
            vp[lo:hi] = rng.standard_normal(d)
    return qp, kp, vp


def test_routing_error_is_replacement_error():
    # e_IJ equals the change of the un-normalised proxy-query output when block J's
    # keys and values are replaced by n_J copies of the block centroid
    rng = np.random.default_rng(7)
    N, d = 300, 8
    qp, kp, vp = _routing_inputs(rng, N, d)
    r = oracle.route_ratios(qp, kp, vp, N, rows=[2])[0]
    qbar, n = oracle.pool(qp, N)
    kbar, _ = oracle.pool(kp, N)
    vbar, _ = oracle.pool(vp, N)
    def unnorm(K, V):
        s = K @ qbar[2] / math.sqrt(d)
        return np.exp(s) @ V, np.exp(s).sum()
    base, _ = unnorm(kp[:N], vp[:N])
    s_all = kp[:N] @ qbar[2] / math.sqrt(d)
    M = s_all.max(); Z = np.exp(s_all - M).sum()
    for J in range(len(n)):
        lo, hi = J * 64, min(J * 64 + 64, N)
        K2 = kp[:N].copy(); V2 = vp[:N].copy()
        K2[lo:hi] = kbar[J]; V2[lo:hi] = vbar[J]
        repl, _ = unnorm(K2, V2)
        e = np.linalg.norm(base - repl) * np.exp(-M)
        assert np.isclose(r[J], e / Z * 64 / n[J], rtol=1e-9, atol=1e-14)


def test_routing_constant_keys_gives_zero_error():
    rng = np.random.default_rng(8)
    qp, kp, vp = _routing_inputs(rng, 256, 8, const_k=True)
    r = oracle.route_ratios(qp, kp, vp, 256)
    assert np.all(r < 1e-12)
    # rounding leaves ~1e-17 residues, so every block sits in the near set; with the
    # errors exactly zero the pick reduces to the index tie-break
    _, near = oracle.select_routing(r[0], 2)
    assert near.all()
    kept, _ = oracle.select_routing(np.zeros(4), 2)
    assert kept.tolist() == [True, True, False, False]


def test_routing_constant_values_jensen_gap():
    # V constant per block: error = ||v_J|| * (sum_j e^{s_j-M} - n e^{sbar-M}) >= 0 (Jensen)
    rng = np.random.default_rng(9)
    N, d = 256, 8
    qp, kp, vp = _routing_inputs(rng, N, d, const_v=True)
    r = oracle.route_ratios(qp, kp, vp, N, rows=[1])[0]
    assert np.all(r >= 0)
    qbar, n = oracle.pool(qp, N)
    kbar, _ = oracle.pool(kp, N)
    s = kp[:N] @ qbar[1] / math.sqrt(d)
    M = s.max(); Z = np.exp(s - M).sum()
    for J in range(4):
        gap = np.exp(s[J * 64:(J + 1) * 64] - M).sum() - 64 * np.exp(kbar[J] @ qbar[1] / math.sqrt(d) - M)
        assert gap >= -1e-12
        assert np.isclose(r[J], abs(gap) * np.linalg.norm(vp[J * 64]) / Z, rtol=1e-8, atol=1e-14)


def test_mask_from_rows():
    kept = np.array([[True, False, True], [False, False, True]])
    idx, cnt = oracle.mask_from_rows(kept)
    assert cnt.tolist() == [2, 1] and idx[0].tolist() == [0, 2] and idx[1].tolist() == [2]


# ---- SICS coherence (SPADE, part 2) -------------------------------------------------
def test_sics_constant_block_is_fully_coherent():
    # n identical keys: every cosine is 1, SICS = n^2, c = 1
    kp = np.zeros((128, 8))
    kp[:64] = np.array([1.0, -2.0, 0.5, 3.0, 0.0, 1.0, 1.0, -1.0])
    kp[64:128] = 0.25
    c = oracle.sics_coherence(kp, 128)
    assert np.allclose(c, [1.0, 1.0], atol=1e-12)


def test_sics_orthogonal_keys_give_one_over_n():
    # n mutually orthogonal keys (scaled basis vectors): only the n diagonal
    # terms survive, SICS = n, c = 1 / n
    d = 64
    kp = np.zeros((64, d))
    kp[np.arange(64), np.arange(64)] = np.linspace(0.5, 3.0, 64)
    assert abs(oracle.sics_coherence(kp, 64)[0] - 1.0 / 64) < 1e-14


def test_sics_antipodal_keys_cancel_and_scale_does_not_matter():
    # keys s_i * x with s_i = +-1 in equal numbers: SICS = (sum s_i)^2 = 0
    x = np.array([0.3, -1.0, 2.0, 0.7])
    kp = np.tile(x, (64, 1)) * np.repeat([1.0, -1.0], 32)[:, None]
    assert abs(oracle.sics_coherence(kp, 64)[0]) < 1e-12
    # 48 keys along +x and 16 along -x: SICS = (48 - 16)^2 = 1024, c = 1/4;
    # positive rescaling of individual keys changes nothing
    s = np.where(np.arange(64) < 48, 1.0, -1.0) * np.linspace(0.1, 5.0, 64)
    assert abs(oracle.sics_coherence(np.outer(s, x), 64)[0] - 0.25) < 1e-12


def test_sics_zero_key_ragged_block_and_closed_form():
    rng = np.random.default_rng(11)
    N, d = 64 + 40, 16                                 # second block: 40 valid keys, 24 pads
    kp = np.zeros((128, d))
    kp[:N] = rng.standard_normal((N, d))
    kp[5] = 0.0                                        # a zero key counts in n, adds nothing
    kp[N:] = 9.0                                       # pads must be ignored
    c = oracle.sics_coherence(kp, N)
    # identity: sum_{i,j} cos(k_i, k_j) = || sum_i k_i / ||k_i|| ||^2 over nonzero keys
    for J, (lo, hi) in enumerate([(0, 64), (64, N)]):
        blk = kp[lo:hi]
        nrm = np.linalg.norm(blk, axis=1)
        u = (blk[nrm > 0] / nrm[nrm > 0, None]).sum(axis=0)
        assert abs(c[J] - (u @ u) / (hi - lo) ** 2) < 1e-12
    # one zero key among n - 1 identical ones: SICS = (n - 1)^2
    kq = np.zeros((64, d))
    kq[1:] = 2.0
    assert abs(oracle.sics_coherence(kq, 64)[0] - (63 / 64) ** 2) < 1e-14
    # an empty block (all pads) scores 0
    assert oracle.sics_coherence(np.ones((128, 4)), 64)[1] == 0.0


def test_sics_scores_rank_the_coherent_blocks():
    rng = np.random.default_rng(12)
    d, nb = 16, 6
    kp = rng.standard_normal((nb * 64, d))
    # blocks 1 and 4 made coherent: a shared direction plus a little noise
    for J, a in ((1, 0.1), (4, 0.3)):
        kp[J * 64:(J + 1) * 64] = rng.standard_normal(d) + a * rng.standard_normal((64, d))
    S = oracle.sics_scores(kp, nb * 64)
    assert abs(S.sum() - 1.0) < 1e-12 and np.all(S >= 0)
    kept, _ = oracle.select_topk(S, 2)
    assert np.nonzero(kept)[0].tolist() == [1, 4]
    assert np.all(oracle.sics_scores(np.zeros((128, 4)), 128) == 0.0)
