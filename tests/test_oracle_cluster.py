"""Pins of the co-clustering order oracle (SVOO 2.B, SVG-EAR 2.A)."""
import numpy as np

import oracle
from oracle import cluster


def _bf16(x):
    """Round float64 values to bf16 (round to nearest even) and back."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def test_initial_centroids_are_raster_block_means():
    rng = np.random.default_rng(0)
    N, d = 150, 4                                     # blocks of 64, 64, 22 tokens
    q = _bf16(rng.normal(size=(N, d)))
    c = cluster.initial_centroids(q, N)
    assert c.shape == (3, d) and c.dtype == np.float32
    assert np.array_equal(c[2], (q[128:150].sum(0) / 22).astype(np.float32))
    assert np.array_equal(c[0], (q[:64].sum(0) / 64).astype(np.float32))


def test_planted_coclusters_are_recovered():
    # queries and keys drawn around C shared directions, shuffled: every token
    # lands in the cluster of its direction after the rounds
    rng = np.random.default_rng(1)
    C, d, per = 4, 16, 64
    N = C * per
    dirs = np.linalg.qr(rng.normal(size=(d, d)))[0][:C] * 8.0
    lab = rng.permutation(np.repeat(np.arange(C), per))
    q = _bf16(dirs[lab] + 0.05 * rng.normal(size=(N, d)))
    k = _bf16(dirs[lab] + 0.05 * rng.normal(size=(N, d)))
    aq, ak, gq, gk = cluster.cocluster(q, k, N, rounds=3)
    # same planted direction <-> same cluster, for queries, keys, and across them
    for a in (aq, ak):
        for c in range(C):
            assert len(set(a[lab == c])) == 1
    assert all(aq[lab == c][0] == ak[lab == c][0] for c in range(C))
    perm_q, iperm_q = cluster.perm_from_clusters(aq, N)
    ids = perm_q[perm_q >= 0]
    assert np.all(np.diff(aq[ids]) >= 0)              # contiguous clusters
    assert np.array_equal(np.sort(ids), np.arange(N))


def test_assignment_is_the_exact_argmax_with_lowest_index_ties():
    x = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    c = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 1.0]], dtype=np.float32)
    best, gap = cluster._assign(x, c)
    assert best.tolist() == [0, 1, 0]                 # [2]: tie 1 = 1 = 1 -> index 0
    assert gap.tolist() == [1.0, 0.0, 0.0]


def test_empty_clusters_take_the_partner_centroid():
    x = np.array([[1.0, 2.0], [3.0, 4.0]])
    fallback = np.array([[9, 9], [7, 7], [5, 5]], dtype=np.float32)
    m = cluster._means(x, np.array([2, 2]), 3, fallback)
    assert np.array_equal(m, np.array([[9, 9], [7, 7], [2, 3]], dtype=np.float32))


def test_one_round_fixed_point_on_separated_data():
    # once the planted partition is reached, further rounds change nothing
    rng = np.random.default_rng(2)
    C, d, per = 3, 8, 64
    N = C * per
    dirs = np.eye(d)[:C] * 5.0
    lab = np.repeat(np.arange(C), per)
    q = _bf16(dirs[lab] + 0.01 * rng.normal(size=(N, d)))
    k = _bf16(dirs[lab] + 0.01 * rng.normal(size=(N, d)))
    a3 = cluster.cocluster(q, k, N, rounds=3)
    a5 = cluster.cocluster(q, k, N, rounds=5)
    assert np.array_equal(a3[0], a5[0]) and np.array_equal(a3[1], a5[1])


def test_assignment_survives_cancellation_in_the_fp64_sums():
    # Exact affinities that fp64 summation gets wrong in any usual order: with
    # x = (1, 1, 1) and a centroid holding +-2^60, adding 1 to 2^60 first loses
    # the 1.  The oracle must decide on the exact sums (math.fsum over the
    # exact bf16 x float32 products), so a plain fp64 argmax, or a near-tie
    # window that is relative to the (cancelled) result, fails here.
    big = 2.0 ** 60
    x = np.ones((2, 3))
    # row 0: every permutation of (2^60, 1, -2^60): all exactly 1 -> tie -> index 0
    perms = [(1.0, big, -big), (big, -big, 1.0), (big, 1.0, -big), (-big, big, 1.0), (1.0, -big, big),
             (-big, 1.0, big)]
    c = np.array(perms, dtype=np.float32)
    best, gap = cluster._assign(x[:1], c)
    assert best.tolist() == [0] and gap.tolist() == [0.0]
    # row 1: exactly 1 (cancelling) against exactly 0.5 (plain): the first wins by 0.5
    c2 = np.array([(1.0, big, -big), (0.5, 0.0, 0.0)], dtype=np.float32)
    best, gap = cluster._assign(x[1:], c2)
    assert best.tolist() == [0] and gap.tolist() == [0.5]
    # the candidates' exact values are what decide: swapping the two centroids
    # moves the winner with them
    best, _ = cluster._assign(x[1:], c2[::-1].copy())
    assert best.tolist() == [1]
