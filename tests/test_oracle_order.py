"""Pins for the oracle's token orderings (no GPU)."""
import numpy as np
import pytest

import oracle
from oracle.order import hilbert_key_3d


def _coords(ids, H, W):
    t, rem = np.divmod(ids, H * W)
    h, w = np.divmod(rem, W)
    return t, h, w


def test_order1_is_gray_code(golden):
    expect = [int(x) for x in golden("hilbert_order1.txt")[0]]
    perm, _ = oracle.perm_hilbert(2, 2, 2)
    assert perm[:8].tolist() == expect


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_full_cube_unit_steps(k):
    s = 1 << k
    perm, iperm = oracle.perm_hilbert(s, s, s)
    ids = perm[: s ** 3]
    t, h, w = _coords(ids, s, s)
    step = np.abs(np.diff(t)) + np.abs(np.diff(h)) + np.abs(np.diff(w))
    assert np.all(step == 1)
    assert ids[0] == 0                      # the curve starts at the origin


@pytest.mark.parametrize("j", [1, 2, 3])
def test_aligned_runs_fill_aligned_subcubes(j):
    # every aligned run of 8^j consecutive cells is an aligned 2^j sub-cube
    k = 4
    s = 1 << k
    perm, _ = oracle.perm_hilbert(s, s, s)
    ids = perm[: s ** 3]
    t, h, w = _coords(ids, s, s)
    run = 8 ** j
    side = 1 << j
    for r in range(0, s ** 3, run):
        tt, hh, ww = t[r:r + run], h[r:r + run], w[r:r + run]
        for a in (tt, hh, ww):
            assert a.max() - a.min() == side - 1
            assert a.min() % side == 0
        assert len(set(zip(tt.tolist(), hh.tolist(), ww.tolist()))) == run


@pytest.mark.parametrize("shape", [(4, 8, 8), (3, 5, 7), (21, 30, 52), (1, 1, 1), (1, 3, 1), (62, 45, 80)])
def test_bijection_and_padding(shape):
    T, H, W = shape
    N = T * H * W
    for order in ("raster", "hilbert"):
        perm, iperm = oracle.build_perm(T, H, W, order)
        nb = -(-N // 64)
        assert perm.shape == (nb * 64,)
        assert np.array_equal(np.sort(perm[:N]), np.arange(N))
        assert np.all(perm[N:] == -1)
        assert np.array_equal(perm[iperm], np.arange(N))


def test_crop_is_filtered_cube_order():
    # the crop reading: a non-power-of-two grid follows the enclosing cube's curve
    T, H, W = 5, 3, 7
    s = 8
    full, _ = oracle.perm_hilbert(s, s, s)
    t, h, w = _coords(full[: s ** 3], s, s)
    inside = (t < T) & (h < H) & (w < W)
    expect = (t[inside] * H + h[inside]) * W + w[inside]
    perm, _ = oracle.perm_hilbert(T, H, W)
    assert np.array_equal(perm[: T * H * W], expect)


def test_tiny_crop_keeps_unit_steps():
    # 4x8x8: t is the first axis, so t < 4 is the first half of the 8^3 curve
    perm, _ = oracle.perm_hilbert(4, 8, 8)
    st = oracle.locality_stats(perm, 4, 8, 8)
    assert st["unit_frac"] == 1.0


def test_hilbert_beats_raster_locality():
    T, H, W = 21, 30, 52
    ph, _ = oracle.perm_hilbert(T, H, W)
    pr, _ = oracle.perm_raster(T, H, W)
    # mean spatial extent (bounding box volume) of 64-token blocks
    def extent(perm):
        vols = []
        for b in range(0, T * H * W - 63, 64):
            t, h, w = _coords(perm[b:b + 64], H, W)
            vols.append((np.ptp(t) + 1) * (np.ptp(h) + 1) * (np.ptp(w) + 1))
        return np.mean(vols)
    assert extent(ph) < extent(pr)


def test_reorder_roundtrip():
    rng = np.random.default_rng(0)
    T, H, W, d = 3, 5, 7, 4
    N = T * H * W
    x = rng.standard_normal((2, N, d))
    perm, _ = oracle.perm_hilbert(T, H, W)
    xp = oracle.reorder(x, perm)
    assert np.all(xp[:, N:] == 0)
    assert np.array_equal(oracle.inverse_reorder(xp, perm, N), x)
    # position i really holds raster token perm[i]
    assert np.array_equal(xp[1, 5], x[1, perm[5]])


def test_keys_distinct():
    k = 3
    t, h, w = np.meshgrid(np.arange(8), np.arange(8), np.arange(8), indexing="ij")
    key = hilbert_key_3d(t.ravel(), h.ravel(), w.ravel(), k)
    assert np.array_equal(np.sort(key), np.arange(512))


def test_block_counts(golden):
    for T, H, W, N, nb, pads in golden("block_counts.txt"):
        perm, _ = oracle.perm_hilbert(int(T), int(H), int(W))
        assert perm.shape[0] == 64 * int(nb)
        assert int(np.sum(perm < 0)) == int(pads)
        assert int(np.sum(perm >= 0)) == int(N)
