"""Pins for the oracle's attention (no GPU)."""
import math

import numpy as np
import pytest
import torch

import oracle


def _sdpa(q, k, v, mask=None):
    """Library softmax attention in fp64 (torch CPU), the textbook definition."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m)[0, 0].numpy()


def _inputs(seed, N, d):
    rng = np.random.default_rng(seed)
    Npad = -(-N // 64) * 64
    a = [np.zeros((Npad, d)) for _ in range(3)]
    for x in a:
        x[:N] = rng.standard_normal((N, d))
    return a


def test_keep_all_is_dense():
    N, d = 200, 16
    qp, kp, vp = _inputs(0, N, d)
    nb = 4
    out = oracle.masked_attention(qp, kp, vp, N, np.ones((nb, nb), bool))
    ref = _sdpa(qp[:N], kp[:N], vp[:N])
    for I in range(nb):
        lo, hi = I * 64, min(I * 64 + 64, N)
        assert np.allclose(out[I], ref[lo:hi], atol=1e-12)
    assert np.allclose(oracle.dense_attention(qp[:N], kp[:N], vp[:N]), ref, atol=1e-12)


def test_masked_is_library_masked_softmax():
    N, d = 230, 8
    qp, kp, vp = _inputs(1, N, d)
    rng = np.random.default_rng(5)
    keep = rng.random((4, 4)) < 0.5
    keep[np.arange(4), np.arange(4)] = True
    out = oracle.masked_attention(qp, kp, vp, N, keep)
    tok_mask = np.repeat(np.repeat(keep, 64, 0), 64, 1)[:N, :N]
    ref = _sdpa(qp[:N], kp[:N], vp[:N], tok_mask)
    for I in range(4):
        lo, hi = I * 64, min(I * 64 + 64, N)
        assert np.allclose(out[I], ref[lo:hi], atol=1e-12)


def test_online_matches_materialised():
    N, d = 256, 16
    qp, kp, vp = _inputs(2, N, d)
    keep = np.array([[1, 0, 1, 1], [0, 1, 0, 0], [1, 1, 1, 1], [0, 0, 0, 1]], bool)
    out = oracle.masked_attention(qp, kp, vp, N, keep)
    for I in range(4):
        assert np.allclose(oracle.online_block_attention(qp, kp, vp, N, keep, I), out[I], atol=1e-12)


def test_single_token_and_constant_values():
    d = 4
    qp, kp, vp = _inputs(3, 1, d)
    out = oracle.masked_attention(qp, kp, vp, 1, np.ones((1, 1), bool))
    assert np.allclose(out[0], vp[:1], atol=0)
    N = 150
    qp, kp, vp = _inputs(4, N, d)
    vp[:N] = 0.375
    out = oracle.masked_attention(qp, kp, vp, N, np.array([[1, 0, 1]] * 3, bool))
    for I in range(3):
        assert np.allclose(out[I], 0.375, atol=1e-15)


def test_compensation_identity_without_skips():
    N, d = 256, 8
    qp, kp, vp = _inputs(5, N, d)
    kb, n = oracle.pool(kp, N)
    vb, _ = oracle.pool(vp, N)
    keep = np.ones((4, 4), bool)
    a = oracle.masked_attention(qp, kp, vp, N, keep)
    b = oracle.compensated_attention(qp, kp, vp, N, keep, kb, vb, n)
    for I in range(4):
        assert np.allclose(a[I], b[I], atol=1e-14)


@pytest.mark.parametrize("seed", [0, 1])
def test_compensation_exact_on_constant_blocks(seed):
    # identical keys and values inside every block: the centroid stands in exactly,
    # so the compensated output equals dense attention whatever the mask
    rng = np.random.default_rng(seed)
    N, d = 220, 8
    qp, kp, vp = _inputs(10 + seed, N, d)
    for J in range(4):
        lo, hi = J * 64, min(J * 64 + 64, N)
        kp[lo:hi] = rng.standard_normal(d)
        vp[lo:hi] = rng.standard_normal(d)
    kb, n = oracle.pool(kp, N)
    vb, _ = oracle.pool(vp, N)
    keep = rng.random((4, 4)) < 0.4
    out = oracle.compensated_attention(qp, kp, vp, N, keep, kb, vb, n)
    ref = _sdpa(qp[:N], kp[:N], vp[:N])
    for I in range(4):
        lo, hi = I * 64, min(I * 64 + 64, N)
        assert np.allclose(out[I], ref[lo:hi], atol=1e-12)


def test_compensation_all_skipped_is_expanded_centroid_attention():
    N, d = 180, 8
    qp, kp, vp = _inputs(6, N, d)
    kb, n = oracle.pool(kp, N)
    vb, _ = oracle.pool(vp, N)
    keep = np.zeros((3, 3), bool)
    out = oracle.compensated_attention(qp, kp, vp, N, keep, kb, vb, n)
    Kx = np.repeat(kb, n, axis=0)
    Vx = np.repeat(vb, n, axis=0)
    ref = _sdpa(qp[:N], Kx, Vx)
    for I in range(3):
        lo, hi = I * 64, min(I * 64 + 64, N)
        assert np.allclose(out[I], ref[lo:hi], atol=1e-12)


def test_kept_flops_closed_form():
    N, d = 200, 128
    n = np.array([64, 64, 64, 8])
    assert oracle.kept_flops(np.ones((4, 4), bool), n, d) == 4.0 * d * N * N
    keep = np.eye(4, dtype=bool)
    assert oracle.kept_flops(keep, n, d) == 4.0 * d * (3 * 64 * 64 + 8 * 8)
