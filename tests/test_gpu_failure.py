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
