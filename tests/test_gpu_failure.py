"""Failure path and run-to-run reproducibility on the GPU (no fault, no trap:
the timeout comes from a bounded wait that is meant to run out)."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import block_sparse_attention_hilbert_b200 as svsa
from _parity import gpu_layer, gpu_keep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    svsa.lib()


def test_bounded_wait_timeout_is_reported_then_cleared():
    lib = svsa.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.svsa_selftest_timeout(2000, stream) == 0          # a 2 ms wait that nothing ends
    assert lib.svsa_sync_status(stream) == 5                     # SVSA_ERR_TIMEOUT
    assert "site 90" in lib.svsa_last_error().decode()
    assert lib.svsa_sync_status(stream) == 0                     # reported once, then cleared
    assert lib.svsa_selftest_timeout(0, stream) == 1             # out-of-range budget rejected
    # the context is still usable: a layer runs and reports no failure
    w = workloads.WORKLOADS["tiny"]
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    out = svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select,
                                    tau=w.tau)(q, k, v)
    assert lib.svsa_sync_status(stream) == 0
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("kw", [
    dict(select="topk", keep_frac=0.3),
    dict(select="threshold", tau=0.9, sub_block=16),
    dict(select="threshold", tau=0.9, routing=True, compensate=True),
    dict(select="topk", keep_frac=0.3, order="cocluster"),
])
def test_two_runs_are_bit_identical(kw):
    """Masks, orders and outputs do not depend on scheduling: two runs of the
    same layer on the same inputs agree bit for bit."""
    w = workloads.Workload("rep", 1, 3, 128, 6, 12, 20, order=kw.pop("order", "hilbert"), **{
        k: v for k, v in kw.items() if k in ("select", "keep_frac", "tau", "sub_block", "routing", "compensate")})
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=11))
    runs = []
    for _ in range(2):
        attn = gpu_layer(w, q, k, v)
        b = attn.buf
        runs.append((attn.out.clone(), gpu_keep(attn),
                     (b.perm_q.clone(), b.perm_k.clone()) if attn.cocluster else (b.perm.clone(),)))
    assert torch.equal(runs[0][0], runs[1][0])
    assert np.array_equal(runs[0][1], runs[1][1])
    assert all(torch.equal(a, b) for a, b in zip(runs[0][2], runs[1][2]))


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_values_beyond_fp16_are_reported_as_range():
    """A bf16 value of 7e4 given to the fp16 value gather saturates; the call
    succeeds but svsa_sync_status reports SVSA_ERR_RANGE once, then clears."""
    lib = svsa.lib()
    w = workloads.WORKLOADS["tiny"]
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    s = svsa.shape(1, 1, w.T, w.H, w.W, w.d)
    perm = torch.arange(w.Npad, dtype=torch.int32, device="cuda")
    vp = torch.empty(1, 1, w.Npad, w.d, dtype=torch.float16, device="cuda")
    svsa.svsa_reorder_values(v, vp, perm, s)
    assert lib.svsa_sync_status(_stream()) == 0                   # in range: nothing recorded
    v2 = v.clone()
    v2[0, 0, 17, 5] = 7.0e4
    svsa.svsa_reorder_values(v2, vp, perm, s)
    assert lib.svsa_sync_status(_stream()) == 6                   # SVSA_ERR_RANGE
    assert "svsa_reorder_values" in lib.svsa_last_error().decode()
    assert float(vp[0, 0, 17, 5]) == 65504.0                       # saturated, as documented
    assert lib.svsa_sync_status(_stream()) == 0                   # reported once
    v2[0, 0, 3, 0] = float("inf")
    v2[0, 0, 17, 5] = 0.0
    svsa.svsa_reorder_values(v2, vp, perm, s)
    assert lib.svsa_sync_status(_stream()) == 6


def test_block_means_beyond_fp16_are_reported_as_range():
    """Queries whose block mean exceeds the fp16 range of the scores' split."""
    lib = svsa.lib()
    w = workloads.WORKLOADS["tiny"]
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    q2 = q.clone()
    q2[0, 0, :, 3] = 9.0e4                                        # every block's mean is 9e4 in this channel
    attn = svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select, tau=w.tau)
    attn(q, k, v)
    assert lib.svsa_sync_status(_stream()) == 0
    attn(q2, k, v)
    assert lib.svsa_sync_status(_stream()) == 6
    assert "block mean" in lib.svsa_last_error().decode()
    assert lib.svsa_sync_status(_stream()) == 0


@pytest.mark.parametrize("defect", ["descending", "out_of_range", "negative", "count_above_cap", "duplicate"])
def test_malformed_masks_are_reported(defect):
    """mask.check validates caller-built lists before the attention; the
    attention still clamps every count and index to the tensors, so the run
    touches nothing outside them and returns, and svsa_sync_status reports
    SVSA_ERR_MASK."""
    lib = svsa.lib()
    B, heads, T, H, W, d = 1, 2, 4, 8, 16, 128                    # nb = 8
    N = T * H * W
    nb = N // 64
    s = svsa.shape(B, heads, T, H, W, d)
    g = torch.Generator(device="cuda").manual_seed(5)
    qp = torch.randn(B, heads, nb * 64, d, generator=g, device="cuda").to(torch.bfloat16)
    kp = torch.randn(B, heads, nb * 64, d, generator=g, device="cuda").to(torch.bfloat16)
    vp = torch.randn(B, heads, nb * 64, d, generator=g, device="cuda").to(torch.float16)
    op = torch.empty_like(qp)
    cap = nb
    kv_idx = torch.arange(cap, dtype=torch.int32, device="cuda").repeat(B * heads * nb, 1).reshape(B, heads, nb, cap)
    kv_cnt = torch.full((B, heads, nb), 4, dtype=torch.int32, device="cuda")
    good = svsa.make_mask(kv_idx, kv_cnt, cap, check=True)
    svsa.svsa_attn_fwd(qp, kp, vp, good, False, op, None, s)
    assert lib.svsa_sync_status(_stream()) == 0
    bad_idx, bad_cnt = kv_idx.clone(), kv_cnt.clone()
    if defect == "descending":
        bad_idx[0, 1, 3, :4] = torch.tensor([5, 3, 2, 0], dtype=torch.int32)
    elif defect == "out_of_range":
        bad_idx[0, 0, 2, 3] = nb + 5
    elif defect == "negative":
        bad_idx[0, 0, 0, 0] = -1
    elif defect == "count_above_cap":
        bad_cnt[0, 1, 7] = cap + 3
    else:
        bad_idx[0, 0, 6, :4] = torch.tensor([1, 2, 2, 3], dtype=torch.int32)
    bad = svsa.make_mask(bad_idx, bad_cnt, cap, check=True)
    svsa.svsa_attn_fwd(qp, kp, vp, bad, False, op, None, s)
    assert lib.svsa_sync_status(_stream()) == 7                   # SVSA_ERR_MASK
    assert "malformed" in lib.svsa_last_error().decode()
    assert lib.svsa_sync_status(_stream()) == 0
    # a pairing table that is not a permutation
    pairs = torch.arange(nb, dtype=torch.int32, device="cuda").repeat(B * heads, 1).reshape(B, heads, nb)
    goodp = svsa.make_mask(kv_idx, kv_cnt, cap, check=True, pairs=pairs)
    svsa.svsa_attn_fwd(qp, kp, vp, goodp, False, op, None, s)
    assert lib.svsa_sync_status(_stream()) == 0
    badp = pairs.clone()
    badp[0, 1, 5] = badp[0, 1, 2]
    svsa.svsa_attn_fwd(qp, kp, vp, svsa.make_mask(kv_idx, kv_cnt, cap, check=True, pairs=badp), False, op, None, s)
    assert lib.svsa_sync_status(_stream()) == 7
    # without the check the same call is not validated (and still stays in bounds)
    unchecked = svsa.make_mask(bad_idx, bad_cnt, cap)
    svsa.svsa_attn_fwd(qp, kp, vp, unchecked, False, op, None, s)
    assert lib.svsa_sync_status(_stream()) == 0
