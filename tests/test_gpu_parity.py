"""GPU path vs the fp64 oracle on small shapes that still span several tiles and
a ragged tail.  Every GPU step runs through the C ABI (libsvsa.so)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import block_sparse_attention_hilbert_b200 as svsa
from block_sparse_attention_hilbert_b200 import SparseVideoAttention
from _parity import (check_attention, compare_mask_rows, gpu_keep, gpu_layer, oracle_rows, to_np)

pytestmark = pytest.mark.gpu

SHAPES = [(4, 8, 8), (3, 5, 7), (5, 7, 9), (1, 1, 1), (1, 3, 50), (2, 9, 13), (6, 12, 20)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    svsa.lib()


@pytest.mark.parametrize("order", ["raster", "hilbert"])
@pytest.mark.parametrize("grid", SHAPES + [(21, 30, 52), (126, 30, 52), (62, 45, 80), (17, 64, 3)])
def test_perm_bit_exact(order, grid):
    T, H, W = grid
    s = svsa.shape(1, 1, T, H, W, 64)
    N = T * H * W
    nb = -(-N // 64)
    perm = torch.full((nb * 64,), 12345, dtype=torch.int32, device="cuda")
    iperm = torch.full((N,), 12345, dtype=torch.int32, device="cuda")
    o = svsa.ORDER_HILBERT if order == "hilbert" else svsa.ORDER_RASTER
    ws = torch.empty(max(svsa.svsa_perm_workspace_bytes(s, o), 16), dtype=torch.uint8, device="cuda")
    svsa.svsa_build_perm(s, o, perm, iperm, ws, ws.numel())
    svsa.svsa_sync_status()
    ep, ei = oracle.build_perm(T, H, W, order)
    assert np.array_equal(perm.cpu().numpy(), ep)
    assert np.array_equal(iperm.cpu().numpy(), ei)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("grid", [(3, 5, 7), (4, 8, 8), (2, 9, 13)])
def test_reorder_inverse_bit_exact(d, grid):
    T, H, W = grid
    B, h = 2, 3
    N = T * H * W
    x = torch.randn(B, h, N, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    attn = svsa.SparseVideoAttention(B, h, T, H, W, d, order="hilbert", select="topk")
    attn.build_perm()
    b = attn.buf
    b.qp.fill_(7.0)
    svsa.svsa_reorder(x, b.qp, b.perm, attn.shape)
    out = torch.zeros_like(x)
    svsa.svsa_inverse_reorder(b.qp, out, b.iperm, attn.shape)
    svsa.svsa_sync_status()
    perm, _ = oracle.build_perm(T, H, W, "hilbert")
    expect = oracle.reorder(x.cpu().view(torch.int16).numpy(), perm)
    assert np.array_equal(b.qp.cpu().view(torch.int16).numpy(), expect)
    assert torch.equal(out.view(torch.int16), x.view(torch.int16))


@pytest.mark.parametrize("d", [64, 128])
def test_reorder_values_fp16_bit_exact(d):
    T, H, W = 2, 9, 13
    B, h = 1, 2
    N = T * H * W
    g = torch.Generator().manual_seed(9)
    v = (torch.randn(B, h, N, d, generator=g) * 3.0)
    v[0, 0, :5, 0] = torch.tensor([1e-6, -3e-7, 6.1e-5, 70000.0, -1e5])     # subnormal and saturating cases
    v = v.to(torch.bfloat16).cuda()
    attn = svsa.SparseVideoAttention(B, h, T, H, W, d, order="hilbert", select="topk")
    attn.build_perm()
    b = attn.buf
    svsa.svsa_reorder_values(v, b.vp, b.perm, attn.shape)
    # the two saturating values are reported (SVSA_ERR_RANGE), and the status clears
    with pytest.raises(svsa.SvsaError) as err:
        svsa.svsa_sync_status()
    assert err.value.status == 6
    svsa.svsa_sync_status()
    perm, _ = oracle.build_perm(T, H, W, "hilbert")
    vf16 = v.float().clamp(-65504, 65504).to(torch.float16).cpu()
    expect = oracle.reorder(vf16.view(torch.int16).numpy(), perm)
    assert np.array_equal(b.vp.cpu().view(torch.int16).numpy(), expect)


def _small(select, sub=64, grid=(5, 7, 9), heads=2, d=128, **kw):
    T, H, W = grid
    return workloads.Workload("small", 1, heads, d, T, H, W, select=select, sub_block=sub, **kw)


def _run_and_compare_masks(w, step=0, seed=0, run_seed=0):
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=seed))
    attn = gpu_layer(w, q, k, v, step=step, seed=run_seed)
    keep = gpu_keep(attn)
    perm, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    near_total = 0
    rows = list(range(attn.nb))
    for eta in range(w.heads):
        kept, near = oracle_rows(w, qp[eta], kp[eta], vp[eta], perm, rows, step=step, seed=run_seed)
        n, _ = compare_mask_rows(keep[eta], kept, near)
        near_total += n
    return attn, keep, (q, k, v), (qp, kp, vp), perm, near_total


@pytest.mark.parametrize("order", ["raster", "hilbert"])
@pytest.mark.parametrize("select,sub", [("topk", 64), ("threshold", 64), ("threshold", 16), ("topk", 16)])
@pytest.mark.parametrize("grid", [(5, 7, 9), (6, 12, 20)])
def test_mask_and_attention_small(order, select, sub, grid):
    w = _small(select, sub, grid=grid, order=order, tau=0.9, keep_frac=0.3)
    attn, keep, _, (qp, kp, vp), _, near = _run_and_compare_masks(w)
    op = to_np(attn.buf.op)[0]
    for eta in range(w.heads):
        ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta])
        gout = np.concatenate([op[eta][I * 64:min(I * 64 + 64, w.N)] for I in range(attn.nb)])
        check_attention(gout, np.concatenate([ref[I] for I in range(attn.nb)]), f"head {eta}")
        assert np.all(op[eta][w.N:] == 0)


@pytest.mark.parametrize("order", ["raster", "hilbert"])
@pytest.mark.parametrize("select", ["topk", "threshold"])
@pytest.mark.parametrize("grid,d", [((5, 7, 9), 128), ((6, 12, 20), 64), ((4, 8, 8), 128)])
def test_sics_mask_and_attention_small(order, select, grid, d):
    """The SICS scorer: per-head coherence scores, one list per head copied to
    every query block, against the oracle's definition (the double sum of
    cosines); outputs on that mask within tolerance."""
    T, H, W = grid
    w = workloads.Workload("sics", 1, 2, d, T, H, W, order=order, select=select, tau=0.6, keep_frac=0.3,
                           scorer="sics")
    attn, keep, _, (qp, kp, vp), _, near = _run_and_compare_masks(w)
    for eta in range(w.heads):
        assert np.all(keep[eta] == keep[eta][:1])              # the same list for every query block
    op = to_np(attn.buf.op)[0]
    for eta in range(w.heads):
        ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta])
        gout = np.concatenate([op[eta][I * 64:min(I * 64 + 64, w.N)] for I in range(attn.nb)])
        check_attention(gout, np.concatenate([ref[I] for I in range(attn.nb)]), f"head {eta}")


def test_sics_zero_keys_and_compensation():
    """All-zero keys: every coherence is 0, so the threshold rule keeps every
    block and top-k the first k; with compensation on a SICS mask, the means
    come from the same call."""
    w = workloads.Workload("sics0", 1, 2, 128, 6, 12, 20, order="hilbert", select="threshold", tau=0.9,
                           scorer="sics")
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=3))
    attn = gpu_layer(w, q, torch.zeros_like(k), v)
    assert gpu_keep(attn).all()
    wk = w.with_(select="topk", keep_frac=0.25)
    attn = gpu_layer(wk, q, torch.zeros_like(k), v)
    keep = gpu_keep(attn)
    kk = oracle.topk_count(wk.keep_frac, attn.nb)
    assert np.all(keep[:, :, :kk]) and not keep[:, :, kk:].any()
    wc = w.with_(select="topk", keep_frac=0.3, compensate=True)
    attn = gpu_layer(wc, q, k, v)
    keep = gpu_keep(attn)
    perm, _ = oracle.build_perm(wc.T, wc.H, wc.W, wc.order)
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    op = to_np(attn.buf.op)[0]
    for eta in range(wc.heads):
        kb, nv = oracle.pool(kp[eta], wc.N)
        vb, _ = oracle.pool(vp[eta], wc.N)
        ref = oracle.compensated_attention(qp[eta], kp[eta], vp[eta], wc.N, keep[eta], kb, vb, nv)
        gout = np.concatenate([op[eta][I * 64:min(I * 64 + 64, wc.N)] for I in range(attn.nb)])
        check_attention(gout, np.concatenate([ref[I] for I in range(attn.nb)]), f"head {eta}")


@pytest.mark.parametrize("size,d,grid", [(64, 128, (5, 7, 9)), (16, 128, (6, 12, 20)), (16, 64, (2, 9, 13)),
                                         (64, 64, (1, 1, 65))])
def test_pool_entry_point(size, d, grid):
    """svsa_pool: fp32 means of the valid rows of every group, pads never
    counted, against the oracle's fp64 means (fp32 sums of <= 64 bf16 values)."""
    T, H, W = grid
    N = T * H * W
    nb = -(-N // 64)
    g = torch.Generator(device="cuda").manual_seed(9)
    xp = torch.zeros(1, 3, nb * 64, d, dtype=torch.bfloat16, device="cuda")
    xp[:, :, :N] = (2.0 * torch.randn(1, 3, N, d, generator=g, device="cuda")).to(torch.bfloat16)
    xp[:, :, N:] = 7.0                                          # pads must not count
    out = torch.empty(1, 3, nb * 64 // size, d, dtype=torch.float32, device="cuda")
    svsa.svsa_pool(xp, out, svsa.shape(1, 3, T, H, W, d), size)
    torch.cuda.synchronize()
    for eta in range(3):
        ref, cnt = oracle.pool(to_np(xp)[0, eta].astype(np.float64), N, size)
        got = out[0, eta].cpu().numpy().astype(np.float64)
        assert np.abs(got - ref).max() <= 1e-5
        assert np.all(got[cnt == 0] == 0.0)


@pytest.mark.parametrize("tau", [0.5, 0.95, 1.0])
def test_threshold_extremes(tau):
    w = _small("threshold", 64, grid=(6, 12, 20), tau=tau)
    _, keep, *_ = _run_and_compare_masks(w)
    if tau >= 1.0:
        assert keep.all()


def test_structured_bit_exact():
    w = workloads.Workload("s", 1, 2, 64, 12, 10, 20, order="raster", select="structured",
                           win_t=2, win_rows=1, n_anchors=4)
    # the anchors rotate with the step index (computed in the library from
    # (seed, step)); each step's mask must equal the oracle's bit for bit
    cols = []
    for run_seed, step in ((0, 0), (0, 1), (0, 2), (0, 3), (12345, 3), (2**40 + 1, 0)):
        _, keep, *_ = _run_and_compare_masks(w, step=step, run_seed=run_seed)
        assert np.array_equal(keep[0], keep[1])          # structure is per layer, not per head
        cols.append(tuple(np.nonzero(keep[0].all(axis=0))[0]))
    assert len(set(cols[:4])) > 1                        # the always-kept columns move with the step
    w0 = w.with_(win_t=0, win_rows=0, n_anchors=0, T=3, H=8, W=16)
    _run_and_compare_masks(w0)


def test_routing_and_compensation_small():
    w = _small("threshold", 64, grid=(6, 12, 20), tau=0.9, routing=True, compensate=True)
    attn, keep, _, (qp, kp, vp), _, near = _run_and_compare_masks(w)
    b = attn.buf
    op = to_np(b.op)[0]
    kbar_g = to_np(b.kbar)[0]
    vbar_g = to_np(b.vbar)[0]
    assert np.array_equal(b.nvalid.cpu().numpy(), oracle.pool(kp[0], w.N)[1])
    for eta in range(w.heads):
        kb, n = oracle.pool(kp[eta], w.N)
        vb, _ = oracle.pool(vp[eta], w.N)
        assert np.allclose(kbar_g[eta], kb, rtol=1e-5, atol=1e-6)
        assert np.allclose(vbar_g[eta], vb, rtol=1e-5, atol=1e-6)
        ref = oracle.compensated_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta], kb, vb, n)
        gout = np.concatenate([op[eta][I * 64:min(I * 64 + 64, w.N)] for I in range(attn.nb)])
        check_attention(gout, np.concatenate([ref[I] for I in range(attn.nb)]), f"comp head {eta}")


@pytest.mark.parametrize("sub,d,grid,heads", [
    (64, 128, (4, 10, 16), 2),      # nb = 10: key ranges of the routing kernel past nb are empty
    (64, 64, (5, 7, 9), 2),         # head dim 64, ragged last block
    (16, 128, (6, 12, 20), 2),      # budget from 16-token sub-block scores, ratios from block means
    (64, 128, (10, 30, 52), 1),     # nb = 244: two tiles of 128 proxies, the second one ragged
])
def test_routing_masks(sub, d, grid, heads):
    w = _small("threshold", sub, grid=grid, heads=heads, d=d, tau=0.9, routing=True)
    _run_and_compare_masks(w)


@pytest.mark.parametrize("select,kw", [
    ("threshold", dict(tau=0.9)),
    ("threshold", dict(tau=0.5)),
    ("threshold", dict(tau=0.0)),                   # shortest prefix: one block
    ("topk", dict(keep_frac=0.3)),
    ("threshold", dict(tau=0.9, routing=True)),
    ("threshold", dict(tau=0.9, sub_block=16)),
])
def test_long_row_selection(select, kw):
    """nb = 1129 (> 1024): rows selected by one CTA each; sampled rows against
    the oracle, every row's list and bit row checked for consistency."""
    sub = kw.pop("sub_block", 64)
    w = _small(select, sub, grid=(10, 20, 361), heads=1, d=64, **kw)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=3))
    attn = gpu_layer(w, q, k, v)
    assert attn.nb == 1129
    keep = gpu_keep(attn)
    perm, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    rows = sorted(set(range(0, attn.nb, 61)) | {attn.nb - 1})
    kept, near = oracle_rows(w, qp[0], kp[0], vp[0], perm, rows)
    compare_mask_rows(keep[0][rows], kept, near)
    if select == "threshold" and kw.get("tau") == 0.0:
        assert np.all(keep[0].sum(axis=1) == 1)


@pytest.mark.parametrize("select,start,end", [("threshold", 0.97, 0.7), ("topk", 0.6, 0.25)])
def test_schedule_run_matches_oracle(select, start, end):
    """An 8-step run under the step schedule (2 dense steps, mask rebuilt every 3
    steps, Q and K drifting between steps): each rebuilt mask is the oracle's
    for that step's parameter and inputs, each reused mask is bit-identical to
    the last built one, and every step's output is the oracle's attention over
    the step's inputs with the mask in use."""
    n, dense, every = 8, 2, 3
    w = _small(select, 64, grid=(6, 12, 20), heads=2)
    q0, k0, v = (t.cuda() for t in workloads.make_qkv(w, seed=5))
    attn = svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=select,
                                     schedule=(n, dense, start, end, every), keep_bits=True, device="cuda")
    perm, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
    flags = oracle.rebuilds(n, dense, every)
    last = None
    for s in range(n):
        q, k = workloads.qk_at_step(q0, k0, sigma=0.05, seed=5, step=s)
        out, rebuilt = attn.step(q, k, v, s)
        torch.cuda.synchronize()
        assert rebuilt == flags[s]
        keep = gpu_keep(attn)
        qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
        if rebuilt:
            p = oracle.step_param(n, dense, start, end, s)
            ws = w.with_(tau=p) if select == "threshold" else w.with_(keep_frac=p)
            for eta in range(w.heads):
                kept, near = oracle_rows(ws, qp[eta], kp[eta], vp[eta], perm, list(range(attn.nb)))
                compare_mask_rows(keep[eta], kept, near)
            if s < dense:
                assert keep.all()
            last = keep
        else:
            assert np.array_equal(keep, last)
        op = to_np(attn.buf.op)[0]
        for eta in range(w.heads):
            ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta])
            gout = np.concatenate([op[eta][I * 64:min(I * 64 + 64, w.N)] for I in range(attn.nb)])
            check_attention(gout, np.concatenate([ref[I] for I in range(attn.nb)]), f"step {s} head {eta}")


@pytest.mark.parametrize("select,groups,kw", [
    ("topk", 3, {}),
    ("threshold", 5, {"routing": True, "compensate": True}),
    ("structured", 2, {"n_anchors": 2}),
])
def test_forward_host_matches_device_call(select, groups, kw):
    """The streamed host-to-host layer (groups of heads on three streams) gives
    bit for bit the output of the device call on the same inputs."""
    w = _small(select, 64, grid=(6, 12, 20), heads=8, tau=0.9, keep_frac=0.3, **kw)   # nb = 23: groups of 4 rows
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=3))
    mk = lambda: svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select,
                                           tau=w.tau, keep_frac=w.keep_frac, n_anchors=w.n_anchors,
                                           routing=w.routing, compensate=w.compensate, device="cuda")
    ref = mk()(q, k, v, step=1)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    attn = mk()
    attn.forward_host(hq, hk, hv, hout, step=1, groups=groups)
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu())
    # a second call reusing the cached mask gives the same output again
    hout2 = torch.empty_like(hout).pin_memory()
    attn.forward_host(hq, hk, hv, hout2, reuse_mask=True, groups=groups)
    torch.cuda.synchronize()
    assert torch.equal(hout2, hout)


@pytest.mark.parametrize("select,groups,kw", [
    ("topk", 1, dict(order="raster")),
    ("threshold", 3, dict(routing=True, compensate=True)),
    ("threshold", 8, dict(sub=16, passes=2)),
    ("structured", 2, dict(n_anchors=2)),
    ("topk", 4, dict(paired=True, d=64)),
])
def test_layer_entry_point_on_host_buffers(select, groups, kw):
    """svsa_layer_forward_host (the C entry point on host buffers, with its own
    copy streams) gives bit for bit the device pipeline's output, over steps
    that rebuild the mask and steps that reuse it."""
    kw = dict(kw)
    sub, passes, paired = kw.pop("sub", 64), kw.pop("passes", 1), kw.pop("paired", False)
    w = _small(select, sub, grid=(6, 12, 20), heads=8, tau=0.9, keep_frac=0.3, **kw)
    mk = lambda: svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select,
                                           tau=w.tau, keep_frac=w.keep_frac, sub_block=sub, n_anchors=w.n_anchors,
                                           routing=w.routing, compensate=w.compensate, attn_passes=passes,
                                           paired_split=paired, device="cuda")
    ref_layer = mk()
    cfg = svsa.layer_config(svsa.ORDER_HILBERT if w.order == "hilbert" else svsa.ORDER_RASTER, ref_layer.params,
                            compensate=w.compensate, attn_passes=passes, paired=paired, groups=groups)
    h = svsa.svsa_layer_create(ref_layer.shape, cfg)
    try:
        for step, reuse in ((0, False), (1, True), (2, False)):
            q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=10 + step))
            ref = ref_layer(q, k, v, step=step, reuse_mask=reuse).cpu()
            hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
            hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()
            svsa.svsa_layer_forward_host(h, hq, hk, hv, hout, step=step,
                                         flags=svsa.LAYER_REUSE_MASK if reuse else 0)
            torch.cuda.synchronize()
            assert torch.equal(hout, ref), f"step {step}"
        # three calls queued back to back with their inputs declared ready (the
        # next call's copies overlap this one's work, the input staging
        # alternates between two sets), one synchronisation at the end
        ins, refs, outs = [], [], []
        for step in (3, 4, 5):
            q3, k3, v3 = (t.cuda() for t in workloads.make_qkv(w, seed=20 + step))
            refs.append(ref_layer(q3, k3, v3, step=step, reuse_mask=step > 3).cpu())
            ins.append(tuple(t.cpu().pin_memory() for t in (q3, k3, v3)))
            outs.append(torch.empty(q3.shape, dtype=q3.dtype).pin_memory())
        torch.cuda.synchronize()
        for i, step in enumerate((3, 4, 5)):
            svsa.svsa_layer_forward_host(h, *ins[i], outs[i], step=step,
                                         flags=svsa.LAYER_INPUTS_READY | (svsa.LAYER_REUSE_MASK if step > 3 else 0))
        torch.cuda.synchronize()
        for i in range(3):
            assert torch.equal(outs[i], refs[i]), f"queued call {i}"
        (hq, hk, hv), ref = ins[2], refs[2]
        # pageable host memory: the copies no longer overlap, the result is the same
        pq, pk, pv = (t.clone() for t in (hq, hk, hv))
        pout = torch.empty(hq.shape, dtype=hq.dtype)
        assert not pq.is_pinned() and not pout.is_pinned()
        svsa.svsa_layer_forward_host(h, pq, pk, pv, pout, step=5, flags=svsa.LAYER_REUSE_MASK)
        torch.cuda.synchronize()
        assert torch.equal(pout, ref)
        svsa.svsa_sync_status()
    finally:
        svsa.svsa_layer_destroy(h)


@pytest.mark.parametrize("d", [64, 128])
def test_dense_and_random_masks(d):
    T, H, W = 5, 7, 9
    w = _small("topk", 64, grid=(T, H, W), heads=2, d=d)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=4))
    # the lists are written here, not by svsa_build_mask, so no pairing table
    # (the attention then pairs query blocks 2p and 2p + 1)
    attn = svsa.SparseVideoAttention(1, 2, T, H, W, d, order="hilbert", select="threshold", tau=1.0,
                                     pair_blocks=False)
    attn.reorder(q, k, v)
    b = attn.buf
    perm, _ = oracle.build_perm(T, H, W, "hilbert")
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    # dense
    attn.attend_dense()
    torch.cuda.synchronize()
    op = to_np(b.op)[0]
    for eta in range(2):
        ref = oracle.dense_attention(qp[eta][:w.N], kp[eta][:w.N], vp[eta][:w.N])
        check_attention(op[eta][:w.N], ref, "dense")
    # random masks fed straight into the kv lists
    nb = attn.nb
    keep = np.stack([workloads.random_mask_lists(nb, nb, density=0.4, seed=s) for s in range(2)])
    idx = np.zeros((1, 2, nb, nb), dtype=np.int32)
    cnt = keep.sum(-1).astype(np.int32)[None]
    for eta in range(2):
        for I in range(nb):
            lst = np.nonzero(keep[eta, I])[0]
            idx[0, eta, I, :len(lst)] = lst
    b.kv_idx.copy_(torch.from_numpy(idx))
    b.kv_cnt.copy_(torch.from_numpy(cnt))
    attn.attend()
    torch.cuda.synchronize()
    op = to_np(b.op)[0]
    for eta in range(2):
        ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta])
        gout = np.concatenate([op[eta][I * 64:min(I * 64 + 64, w.N)] for I in range(nb)])
        check_attention(gout, np.concatenate([ref[I] for I in range(nb)]), "random mask")


def test_single_token_and_single_block():
    for grid in [(1, 1, 1), (1, 3, 5)]:
        w = _small("threshold", 64, grid=grid, heads=1, tau=0.9)
        q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=1))
        attn = gpu_layer(w, q, k, v)
        out = attn.out
        if w.N == 1:
            assert torch.allclose(out.float(), v.float(), atol=0, rtol=0)
        perm, _ = oracle.build_perm(*grid, "hilbert")
        ref = oracle.dense_attention(to_np(q)[0, 0], to_np(k)[0, 0], to_np(v)[0, 0])
        check_attention(to_np(out)[0, 0], ref, "single block")


def test_layer_end_to_end_raster_in_raster_out():
    w = _small("topk", 64, grid=(6, 12, 20), heads=2, keep_frac=0.4, order="hilbert")
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=5))
    attn = gpu_layer(w, q, k, v)
    keep = gpu_keep(attn)
    perm, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    out = to_np(attn.out)[0]
    for eta in range(2):
        ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta])
        refp = np.zeros((attn.Npad, w.d))
        for I in range(attn.nb):
            refp[I * 64:min(I * 64 + 64, w.N)] = ref[I]
        check_attention(out[eta], oracle.inverse_reorder(refp, perm, w.N), "raster out")


def test_masks_are_deterministic():
    w = _small("threshold", 16, grid=(6, 12, 20), tau=0.9)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=6))
    a1 = gpu_layer(w, q, k, v)
    a2 = gpu_layer(w, q, k, v)
    assert torch.equal(a1.buf.kv_cnt, a2.buf.kv_cnt)
    assert np.array_equal(gpu_keep(a1), gpu_keep(a2))
    assert torch.equal(a1.out.view(torch.int16), a2.out.view(torch.int16))


def test_lse_output():
    w = _small("topk", 64, grid=(5, 7, 9), heads=1, keep_frac=0.5)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=7))
    attn = gpu_layer(w, q, k, v)
    keep = gpu_keep(attn)
    lse = torch.full((1, 1, attn.Npad), 99.0, device="cuda")
    attn.attend(lse=lse)
    torch.cuda.synchronize()
    perm, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
    qp, kp = (oracle.reorder(to_np(t)[0, 0].astype(np.float64), perm) for t in (q, k))
    g = lse.cpu().numpy()[0, 0]
    for I in range(attn.nb):
        lo, hi = I * 64, min(I * 64 + 64, w.N)
        pos = np.concatenate([np.arange(J * 64, min(J * 64 + 64, w.N)) for J in np.nonzero(keep[0, I])[0]])
        s = qp[lo:hi] @ kp[pos].T / np.sqrt(w.d)
        ref = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
        assert np.abs(g[lo:hi] - ref).max() < 1e-3
    assert np.all(g[w.N:] == 0)


def _cocluster_case(w, q, k, rounds=3):
    """GPU co-clustering orders next to the oracle's, head by head."""
    attn = svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order="cocluster", select=w.select,
                                     tau=w.tau, keep_frac=w.keep_frac, cluster_rounds=rounds, device="cuda")
    attn.build_perm(q=q, k=k)
    torch.cuda.synchronize()
    b = attn.buf
    qn, kn = to_np(q)[0].astype(np.float64), to_np(k)[0].astype(np.float64)
    for eta in range(w.heads):
        aq, ak, gq, gk = oracle.cocluster(qn[eta], kn[eta], w.N, rounds=rounds)
        pq, ipq = oracle.perm_from_clusters(aq, w.N)
        pk, ipk = oracle.perm_from_clusters(ak, w.N)
        got_pq, got_pk = b.perm_q[eta].cpu().numpy(), b.perm_k[eta].cpu().numpy()
        assert np.array_equal(got_pq, pq), f"head {eta}: query order differs at {np.nonzero(got_pq != pq)[0][:8]}"
        assert np.array_equal(got_pk, pk), f"head {eta}: key order differs at {np.nonzero(got_pk != pk)[0][:8]}"
        assert np.array_equal(b.iperm_q[eta].cpu().numpy(), ipq)
        assert np.array_equal(b.iperm_k[eta].cpu().numpy(), ipk)
    return attn


@pytest.mark.parametrize("d,grid,heads", [(128, (6, 12, 20), 2), (64, (5, 7, 9), 2), (128, (8, 30, 52), 1)])
def test_cocluster_order_bit_exact(d, grid, heads):
    """Both orders (queries; keys and values) equal the oracle's bit for bit."""
    w = _small("topk", 64, grid=grid, heads=heads, d=d, keep_frac=0.3)
    q, k, _ = (t.cuda() for t in workloads.make_qkv(w, seed=6))
    _cocluster_case(w, q, k)


def test_cocluster_exact_ties_take_the_lower_cluster():
    """Repeated tokens make equal centroids and exactly tied affinities: the
    fp64 fix-up must give the lower cluster index, as the oracle does."""
    w = _small("topk", 64, grid=(4, 8, 16), heads=1, d=128, keep_frac=0.3)
    g = torch.Generator().manual_seed(7)
    base = (torch.randn(6, 128, generator=g) * 2).to(torch.bfloat16)
    idx = torch.randint(0, 6, (w.N,), generator=g)
    q = base[idx][None, None].cuda()
    k = base[torch.roll(idx, 5)][None, None].cuda()
    _cocluster_case(w, q, k, rounds=2)


def test_cocluster_all_centroids_tied_recompute_every_centroid():
    """Identical tokens make all 8 centroids equal: every affinity ties across
    more than four centroids, so the fix-up scores every centroid in fp64 and
    keeps cluster 0, as the oracle does."""
    w = _small("topk", 64, grid=(4, 8, 16), heads=1, d=128, keep_frac=0.3)
    g = torch.Generator().manual_seed(11)
    row = (torch.randn(128, generator=g) * 2).to(torch.bfloat16)
    q = row.expand(w.N, 128).contiguous()[None, None].cuda()
    k = (row * 0.5).to(torch.bfloat16).expand(w.N, 128).contiguous()[None, None].cuda()
    _cocluster_case(w, q, k, rounds=2)


@pytest.mark.parametrize("select", ["topk", "threshold"])
def test_cocluster_layer_matches_oracle(select):
    """The whole layer on the co-clustering order: masks bit-exact outside the
    near set, outputs within tolerance, against the oracle on its own orders."""
    w = _small(select, 64, grid=(6, 12, 20), heads=2, tau=0.9, keep_frac=0.3)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=8))
    attn = _cocluster_case(w, q, k)
    out = attn(q, k, v)
    torch.cuda.synchronize()
    keep = gpu_keep(attn)
    qn, kn, vn = (to_np(t)[0].astype(np.float64) for t in (q, k, v))
    on = to_np(out)[0]
    for eta in range(w.heads):
        aq, ak, _, _ = oracle.cocluster(qn[eta], kn[eta], w.N)
        pq, _ = oracle.perm_from_clusters(aq, w.N)
        pk, _ = oracle.perm_from_clusters(ak, w.N)
        qp, kp, vp = oracle.reorder(qn[eta], pq), oracle.reorder(kn[eta], pk), oracle.reorder(vn[eta], pk)
        kept, near = oracle_rows(w, qp, kp, vp, None, list(range(attn.nb)))
        compare_mask_rows(keep[eta], kept, near)
        ref = oracle.masked_attention(qp, kp, vp, w.N, keep[eta])
        ref_raster = oracle.inverse_reorder(np.concatenate([ref[I] for I in range(attn.nb)] +
                                                           [np.zeros((attn.Npad - w.N, w.d))]), pq, w.N)
        check_attention(on[eta], ref_raster, f"head {eta}")


@pytest.mark.parametrize("case", ["topk", "threshold16", "routing_comp", "structured", "cocluster"])
def test_batch_rows_are_independent(case):
    """B = 2: every step treats the (batch, head) rows independently, so the
    two-batch layer equals two one-batch layers (each checked against the
    oracle elsewhere) bit for bit: permutations, masks and outputs."""
    sel = {"topk": "topk", "cocluster": "topk", "structured": "structured"}.get(case, "threshold")
    kw = {"routing": True, "compensate": True} if case == "routing_comp" else {}
    if case == "structured":
        kw = {"n_anchors": 2}
    sub = 16 if case == "threshold16" else 64
    T, H, W = 5, 12, 20
    w2 = workloads.Workload("batch2", 2, 2, 128, T, H, W, select=sel, sub_block=sub, tau=0.9, keep_frac=0.3, **kw)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w2, seed=11))
    w1 = workloads.Workload("batch1", 1, 2, 128, T, H, W, select=sel, sub_block=sub, tau=0.9, keep_frac=0.3, **kw)

    def run(w, q, k, v):
        if case == "cocluster":
            attn = _cocluster_case(w, q, k) if w.B == 1 else svsa.SparseVideoAttention(
                w.B, w.heads, T, H, W, w.d, order="cocluster", select=w.select, tau=w.tau, keep_frac=w.keep_frac,
                cluster_rounds=3, device="cuda")
            if w.B != 1:
                attn.build_perm(q=q, k=k)
            out = attn(q, k, v)
        else:
            attn = gpu_layer(w, q, k, v, step=1)
            out = attn.out
        torch.cuda.synchronize()
        return attn, out

    a2, o2 = run(w2, q, k, v)
    rows = w2.heads
    for bi in range(2):
        a1, o1 = run(w1, *(t[bi:bi + 1].contiguous() for t in (q, k, v)))
        assert torch.equal(o2[bi].view(torch.int16), o1[0].view(torch.int16)), f"batch {bi}: outputs differ"
        assert torch.equal(a2.buf.kv_cnt.view(2 * rows, -1)[bi * rows:(bi + 1) * rows],
                           a1.buf.kv_cnt.view(rows, -1)), f"batch {bi}: kept counts differ"
        assert np.array_equal(gpu_keep(a2)[bi * rows:(bi + 1) * rows], gpu_keep(a1)), f"batch {bi}: masks differ"
        if case == "cocluster":
            assert torch.equal(a2.buf.perm_q[bi * rows:(bi + 1) * rows], a1.buf.perm_q)
            assert torch.equal(a2.buf.perm_k[bi * rows:(bi + 1) * rows], a1.buf.perm_k)


@pytest.mark.parametrize("grid", [(1, 1, 1), (1, 1, 64), (1, 1, 65), (2, 3, 5), (1, 8, 8)])
@pytest.mark.parametrize("case", ["topk", "threshold", "threshold16", "routing_comp", "cocluster", "structured"])
def test_degenerate_grids(grid, case):
    """One token, exactly one block, one token past a block, tiny ragged grids:
    the whole layer through every rule, masks and outputs against the oracle."""
    d = 64 if case == "threshold16" else 128
    sel = {"topk": "topk", "cocluster": "topk", "structured": "structured"}.get(case, "threshold")
    kw = {"routing": True, "compensate": True} if case == "routing_comp" else {}
    if case == "structured":
        kw = {"n_anchors": 1}                                  # at most nb anchor columns
    w = _small(sel, 16 if case == "threshold16" else 64, grid=grid, heads=2, d=d, tau=0.9, keep_frac=0.3, **kw)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=9))
    if case == "cocluster":
        attn = _cocluster_case(w, q, k)
        out = attn(q, k, v)
    else:
        attn = gpu_layer(w, q, k, v)
        out = attn.out
    torch.cuda.synchronize()
    keep = gpu_keep(attn)
    qn, kn, vn = (to_np(t)[0].astype(np.float64) for t in (q, k, v))
    on = to_np(out)[0]
    b = attn.buf
    for eta in range(w.heads):
        if case == "cocluster":
            aq, ak, _, _ = oracle.cocluster(qn[eta], kn[eta], w.N)
            pq, _ = oracle.perm_from_clusters(aq, w.N)
            pk, _ = oracle.perm_from_clusters(ak, w.N)
        else:
            pq, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
            pk = pq
        qp, kp, vp = oracle.reorder(qn[eta], pq), oracle.reorder(kn[eta], pk), oracle.reorder(vn[eta], pk)
        kept, near = oracle_rows(w, qp, kp, vp, pq, list(range(attn.nb)))
        compare_mask_rows(keep[eta], kept, near)
        if w.compensate:
            kb, n = oracle.pool(kp, w.N)
            vb, _ = oracle.pool(vp, w.N)
            ref = oracle.compensated_attention(qp, kp, vp, w.N, keep[eta], kb, vb, n)
        else:
            ref = oracle.masked_attention(qp, kp, vp, w.N, keep[eta])
        full = np.concatenate([ref[I] for I in range(attn.nb)] + [np.zeros((attn.Npad - w.N, w.d))])
        check_attention(on[eta], oracle.inverse_reorder(full, pq, w.N), f"{case} {grid} head {eta}")


@pytest.mark.parametrize("passes,select,kw", [
    (2, "topk", {}),
    (3, "threshold", {"routing": True, "compensate": True}),
    (5, "threshold", {"sub": 16}),
])
@pytest.mark.parametrize("paired", [False, True])
def test_split_attention_matches_single_pass_and_oracle(passes, select, kw, paired):
    """Key-range passes merged by log-sum-exp (svsa_attn_fwd_split, or each
    pass as the paired-block split): the output and the lse agree with the
    single-pass call (up to rounding) and with the oracle."""
    kw = dict(kw)
    sub = kw.pop("sub", 64)
    w = _small(select, sub, grid=(6, 12, 20), heads=2, tau=0.9, keep_frac=0.3, **kw)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=12))
    mk = lambda p, ps: svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=select,
                                                 tau=w.tau, keep_frac=w.keep_frac, sub_block=sub,
                                                 routing=w.routing, compensate=w.compensate, keep_bits=True,
                                                 attn_passes=p, paired_split=ps, device="cuda")
    one, many = mk(1, False), mk(passes, paired)
    one.reorder(q, k, v); one.build_mask()
    many.reorder(q, k, v); many.build_mask()
    lse1 = torch.empty(1, w.heads, one.Npad, dtype=torch.float32, device="cuda")
    lsep = torch.empty_like(lse1)
    one.attend(lse=lse1); many.attend(lse=lsep)
    torch.cuda.synchronize()
    assert np.array_equal(gpu_keep(one), gpu_keep(many))
    a1, ap = to_np(one.buf.op)[0], to_np(many.buf.op)[0]
    assert np.abs(a1 - ap).max() <= 2 * 2 ** -8 * max(1.0, np.abs(a1).max())       # two bf16 roundings apart at most
    valid = np.arange(one.Npad) < w.N
    assert np.allclose(to_np(lse1)[0][:, valid], to_np(lsep)[0][:, valid], atol=1e-4)
    keep = gpu_keep(many)
    perm, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    for eta in range(w.heads):
        if w.compensate:
            kb, n = oracle.pool(kp[eta], w.N)
            vb, _ = oracle.pool(vp[eta], w.N)
            ref = oracle.compensated_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta], kb, vb, n)
        else:
            ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta])
        gout = np.concatenate([ap[eta][I * 64:min(I * 64 + 64, w.N)] for I in range(many.nb)])
        check_attention(gout, np.concatenate([ref[I] for I in range(many.nb)]), f"passes={passes} head {eta}")


@pytest.mark.parametrize("select,kw", [("topk", {}), ("threshold", dict(routing=True, compensate=True)),
                                       ("structured", dict(n_anchors=2))])
def test_captured_layer_replays_the_eager_call(select, kw):
    """A layer captured in a CUDA graph, replayed on new contents of its input
    buffers, gives the eager call's output bit for bit."""
    w = _small(select, 64, grid=(6, 12, 20), heads=2, tau=0.9, keep_frac=0.3, **kw)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=1))
    layer = gpu_layer(w, q, k, v)                         # builds the order, sizes the buffers
    out = torch.empty_like(q)
    g = layer.capture(q, k, v, out)
    for seed in (2, 3):
        q2, k2, v2 = (t.cuda() for t in workloads.make_qkv(w, seed=seed))
        q.copy_(q2)
        k.copy_(k2)
        v.copy_(v2)
        g.replay()
        torch.cuda.synchronize()
        ref = gpu_layer(w, q2, k2, v2).out                 # a fresh layer, eager
        assert torch.equal(out, ref), f"seed {seed}: replay differs from the eager call"
    svsa.svsa_sync_status()


@pytest.mark.parametrize("select,kw", [("topk", {}), ("threshold", dict(sub=16)),
                                       ("threshold", dict(routing=True, compensate=True))])
def test_query_block_pairing(select, kw):
    """The pairing svsa_build_mask writes (mask.pairs) is a permutation of the
    query blocks of every head, pairs blocks that share kept key blocks at
    least as well as the plain adjacent pairs do, and the attention on it
    matches both the unpaired call and the oracle."""
    w = _small(select, grid=(7, 13, 21), heads=2, tau=0.9, keep_frac=0.3, **kw)   # nb = 30
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=4))
    mk = lambda pair: SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select,
                                           tau=w.tau, keep_frac=w.keep_frac, sub_block=w.sub_block,
                                           routing=w.routing, compensate=w.compensate, pair_blocks=pair,
                                           keep_bits=True, paired_split=True, device="cuda")
    paired, plain = mk(True), mk(False)
    out_p, out_u = paired(q, k, v), plain(q, k, v)
    torch.cuda.synchronize()
    nb = paired.nb
    pairs = paired.buf.pairs.cpu().numpy().reshape(w.heads, nb)
    keep = gpu_keep(paired)
    assert np.array_equal(keep, gpu_keep(plain))
    for eta in range(w.heads):
        assert np.array_equal(np.sort(pairs[eta]), np.arange(nb))
        shared = sum((keep[eta, pairs[eta, i]] & keep[eta, pairs[eta, i + 1]]).sum() for i in range(0, nb - 1, 2))
        adjacent = sum((keep[eta, i] & keep[eta, i + 1]).sum() for i in range(0, nb - 1, 2))
        assert shared >= adjacent
    # two independently rounded bf16 outputs may differ by a rounding step
    # (2^-7 relative); each is checked against the oracle below
    a, b = to_np(out_p), to_np(out_u)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 2e-3)
    perm, _ = oracle.build_perm(w.T, w.H, w.W, w.order)
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    op = to_np(paired.buf.op)[0]
    for eta in range(w.heads):
        if w.compensate:
            kb, nv = oracle.pool(kp[eta], w.N)
            vb, _ = oracle.pool(vp[eta], w.N)
            ref = oracle.compensated_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta], kb, vb, nv)
        else:
            ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta])
        gout = np.concatenate([op[eta][I * 64:min(I * 64 + 64, w.N)] for I in range(nb)])
        check_attention(gout, np.concatenate([ref[I] for I in range(nb)]), f"head {eta}")


def _write_lists(attn, keep):
    """Kept sets keep [heads, nb, nb] (bool) into the layer's kv lists and bitmap."""
    heads, nb = keep.shape[0], keep.shape[1]
    b = attn.buf
    idx = np.zeros((1, heads, nb, b.cap), dtype=np.int32)
    for eta in range(heads):
        for I in range(nb):
            lst = np.nonzero(keep[eta, I])[0]
            idx[0, eta, I, :len(lst)] = lst
    words = -(-nb // 32)
    bits = np.zeros((1, heads, nb, words), dtype=np.uint32)
    for J in range(nb):
        bits[..., J >> 5] |= keep[None, :, :, J].astype(np.uint32) << np.uint32(J & 31)
    b.kv_idx.copy_(torch.from_numpy(idx))
    b.kv_cnt.copy_(torch.from_numpy(keep.sum(-1).astype(np.int32)[None]))
    b.bits.copy_(torch.from_numpy(bits.view(np.int32)))


@pytest.mark.parametrize("passes", [1, 2, 3])
@pytest.mark.parametrize("table", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_paired_split_on_written_masks(passes, table, d):
    """svsa_attn_fwd_paired on lists written here, with every shape a pair can
    take: identical lists (all shared), disjoint lists (all exclusive), one
    empty list, both empty, a full row, and (odd nb) the lone last block;
    with and without a pairing table.  Output and lse agree with
    svsa_attn_fwd up to rounding and with the oracle."""
    T, H, W = 7, 13, 20                                   # N = 1820: nb = 29, last block 28 tokens
    heads = 2
    w = _small("topk", 64, grid=(T, H, W), heads=heads, d=d)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w, seed=21))
    nb = -(-w.N // 64)
    rng = np.random.default_rng(5 + passes)
    keep = rng.random((heads, nb, nb)) < 0.35
    keep[:, 4] = keep[:, 5]                               # identical
    keep[:, 6] = ~keep[:, 7]                              # disjoint
    keep[:, 8] = False                                    # one empty
    keep[:, 10] = keep[:, 11] = False                     # both empty
    keep[:, 12] = True                                    # full
    mk = lambda ps: SparseVideoAttention(1, heads, T, H, W, d, order="hilbert", select="threshold", tau=1.0,
                                         keep_bits=True, pair_blocks=table, attn_passes=passes,
                                         paired_split=ps, device="cuda")
    paired, plain = mk(True), mk(False)
    for a in (paired, plain):
        a.reorder(q, k, v)
        _write_lists(a, keep)
    if table:
        # a random order of the query blocks per head, so pairs are far apart
        pt = np.stack([rng.permutation(nb) for _ in range(heads)]).astype(np.int32)
        paired.buf.pairs.copy_(torch.from_numpy(pt)[None])
    lse_p = torch.empty(1, heads, paired.Npad, dtype=torch.float32, device="cuda")
    lse_u = torch.empty_like(lse_p)
    paired.attend(lse=lse_p)
    plain.attend(lse=lse_u)
    torch.cuda.synchronize()
    svsa.svsa_sync_status()
    a, b = to_np(paired.buf.op)[0], to_np(plain.buf.op)[0]
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 2e-3)
    valid = np.arange(paired.Npad) < w.N
    assert np.allclose(to_np(lse_p)[0][:, valid], to_np(lse_u)[0][:, valid], atol=1e-4)
    assert np.all(a[:, ~valid] == 0)
    lp = to_np(lse_p)[0]
    for eta in range(heads):
        for I in (8, 10, 11):                             # no kept key: zero rows, lse 0
            rows = slice(I * 64, I * 64 + 64)
            assert np.all(a[eta, rows] == 0) and np.all(lp[eta, rows] == 0)
    perm, _ = oracle.build_perm(T, H, W, "hilbert")
    qp, kp, vp = (oracle.reorder(to_np(t)[0].astype(np.float64), perm) for t in (q, k, v))
    for eta in range(heads):
        # (the softmax over no key is undefined; those rows were checked above)
        blocks = [I for I in range(nb) if keep[eta, I].any()]
        ref = oracle.masked_attention(qp[eta], kp[eta], vp[eta], w.N, keep[eta], q_blocks=blocks)
        gout = np.concatenate([a[eta][I * 64:min(I * 64 + 64, w.N)] for I in blocks])
        check_attention(gout, np.concatenate([ref[I] for I in blocks]), f"passes={passes} head {eta}")


def test_paired_split_needs_the_bitmap():
    w = _small("topk", 64, grid=(5, 7, 9), heads=1)
    attn = SparseVideoAttention(1, 1, 5, 7, 9, w.d, select="topk", keep_frac=0.3, device="cuda")
    assert attn.buf.bits is None
    ws = torch.empty(svsa.svsa_attn_paired_workspace_bytes(attn.shape, 1), dtype=torch.uint8, device="cuda")
    b = attn.buf
    with pytest.raises(svsa.SvsaError):
        svsa.svsa_attn_fwd_paired(b.qp, b.kp, b.vp, attn._mask, False, b.op, None, attn.shape, 1, ws, ws.numel())
    assert SparseVideoAttention(1, 1, 5, 7, 9, w.d, select="topk", paired_split=True,
                                device="cuda").buf.bits is not None
