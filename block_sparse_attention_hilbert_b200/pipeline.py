"""One attention layer through the four library calls, with its device buffers.

    attn = SparseVideoAttention(B, heads, T, H, W, d, order="hilbert", select="topk", keep_frac=0.25)
    o = attn(q, k, v)               # q, k, v: bf16 [B, heads, T*H*W, d] on the GPU, raster order

A call runs svsa_reorder (Q, K), svsa_reorder_values (V), svsa_build_mask (unless the cached mask is
reused across denoising steps -- "DFSAttn" trick 3), the attention
(svsa_attn_fwd_split: one pass is a plain svsa_attn_fwd, more passes run over
key ranges with a balanced item schedule; svsa_attn_fwd_paired with
paired_split) and svsa_inverse_reorder on the current stream.  The
permutation is built once per object.  Buffers are allocated once with torch
(the library allocates nothing).

    attn.forward_host(q_h, k_h, v_h, o_h)   # pinned host tensors in and out

runs the same calls on groups of (batch, head) rows, with the host->device
copies of one group, the library calls of the previous group and the
device->host copy of the one before overlapping on three streams (every
(batch, head) row is independent in all four steps).  The library's own
host-buffer entry point (svsa_layer_create / svsa_layer_forward_host) does the
same in C with a device arena of its own.
"""
from __future__ import annotations

import math

import torch

from . import (ORDER_HILBERT, ORDER_RASTER, SEL_STRUCTURED, SEL_THRESHOLD, SEL_TOPK, SCORE_POOLED, SCORE_SICS, BLOCK,
               make_mask, mask_params, schedule as make_schedule, shape, svsa_attn_dense_fwd, svsa_attn_fwd,
               svsa_build_mask, svsa_build_perm, svsa_build_perm_cocluster, svsa_cocluster_workspace_bytes,
               svsa_inverse_reorder, svsa_inverse_reorder_heads, svsa_mask_workspace_bytes,
               svsa_perm_workspace_bytes, svsa_reorder, svsa_reorder_heads, svsa_reorder_values,
               svsa_reorder_values_heads, svsa_schedule_step, svsa_attn_fwd_split,
               svsa_attn_split_workspace_bytes, svsa_attn_fwd_paired, svsa_attn_paired_workspace_bytes)

_ORDERS = {"raster": ORDER_RASTER, "hilbert": ORDER_HILBERT}
_SELECTS = {"threshold": SEL_THRESHOLD, "topk": SEL_TOPK, "structured": SEL_STRUCTURED}
_SCORERS = {"pooled": SCORE_POOLED, "sics": SCORE_SICS}


class LayerBuffers:
    """Device buffers of one layer shape (all caller-owned, as the ABI requires)."""

    def __init__(self, B, heads, T, H, W, d, *, cap, need_means, keep_bits, ws_bytes, perm_ws_bytes,
                 device, compensate=False, pair_blocks=False):
        N = T * H * W
        nb = -(-N // BLOCK)
        Npad = nb * BLOCK
        dev = torch.device(device)
        bf = torch.bfloat16
        self.perm = torch.empty(Npad, dtype=torch.int32, device=dev)
        self.iperm = torch.empty(N, dtype=torch.int32, device=dev)
        self.perm_ws = torch.empty(max(perm_ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.qp = torch.empty(B, heads, Npad, d, dtype=bf, device=dev)
        self.kp = torch.empty_like(self.qp)
        self.vp = torch.empty(B, heads, Npad, d, dtype=torch.float16, device=dev)   # values in fp16
        self.op = torch.empty_like(self.qp)
        self.kv_idx = torch.empty(B, heads, nb, cap, dtype=torch.int32, device=dev)
        self.kv_cnt = torch.empty(B, heads, nb, dtype=torch.int32, device=dev)
        self.kbar = torch.empty(B, heads, nb, d, dtype=torch.float32, device=dev) if need_means else None
        self.vbar = torch.empty_like(self.kbar) if need_means else None
        self.nvalid = torch.empty(nb, dtype=torch.int32, device=dev) if need_means else None
        # compensation: kept-block bitmap and the 16-bit centroid scratch of the attention;
        # the query-block pairing reads the bitmap too
        if compensate or pair_blocks:
            keep_bits = True
        self.bits = (torch.empty(B, heads, nb, -(-nb // 32), dtype=torch.int32, device=dev)
                     if keep_bits else None)
        self.cbar = torch.empty(B, heads, nb, 2 * d, dtype=torch.int16, device=dev) if compensate else None
        self.pairs = torch.empty(B, heads, nb, dtype=torch.int32, device=dev) if pair_blocks else None
        self.ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.cap = cap

    def mask(self):
        return make_mask(self.kv_idx, self.kv_cnt, self.cap, self.bits, self.kbar, self.vbar, self.nvalid,
                         self.cbar, pairs=self.pairs)


class CapturedLayer:
    """A layer call captured by SparseVideoAttention.capture()."""

    def __init__(self, graph):
        self.graph = graph

    def replay(self):
        """Run the captured layer on the current stream (asynchronous)."""
        self.graph.replay()


def default_attn_passes(select: int, Npad: int, d: int) -> int:
    """Key-range passes of the attention for a head of Npad reordered tokens:
    one for the structured rule (its windows keep the key blocks of
    neighbouring query blocks together, so they share L2 already) and while
    the head's K and V (Npad * d * 4 bytes) fit in 48 MB of L2, else enough
    passes for at most 32 MB each, at most 8."""
    kv_bytes = Npad * d * 4
    if select == SEL_STRUCTURED or kv_bytes <= 48 * 2**20:
        return 1
    return min(8, -(-kv_bytes // (32 * 2**20)))


class SparseVideoAttention:
    def __init__(self, B, heads, T, H, W, d, *, order="hilbert", select="threshold", tau=0.9,
                 keep_frac=0.25, sub_block=64, win_t=2, win_rows=1, n_anchors=0, routing=False,
                 compensate=False, keep_bits=False, schedule=None, cluster_rounds=3, attn_passes=None,
                 seed=0, scorer="pooled", check_mask=False, pair_blocks=False, paired_split=False, device="cuda"):
        """order: "raster", "hilbert" or "cocluster" (a per-head semantic order from
        bidirectional query-key co-clustering, built from the first inputs and
        kept until `rebuild_order()`).  schedule: optional (n_steps, dense_steps,
        start, end, refresh_every) -- a timestep-adaptive rule for `step()`.
        attn_passes: key-range passes of the attention (svsa_attn_fwd_split); by
        default 1 for the structured rule (its windows keep the key blocks of
        neighbouring query blocks close together, so they share L2 already)
        and while a head's reordered K and V (Npad * d * 4 bytes) fit in 48 MB
        of L2, else enough passes for at most 32 MB each (at most 8).
        seed: the run's seed of the structured rule's anchor rotation (the
        step index of each call picks the rotation).  scorer: "pooled" (block
        scores) or "sics" (per-head block coherence).  check_mask: validate
        the lists before every attention call (svsa_sync_status reports a
        malformed one).  paired_split: run the attention as
        svsa_attn_fwd_paired (the key blocks both query blocks of a pair keep
        on the 128-row kernel, the rest on the 64-row one; it keeps the
        kept-block bitmap).  pair_blocks: let svsa_build_mask pair the query
        blocks by kept-list overlap for that split (else blocks 2p and 2p + 1
        go together).  Both are off by default: on B200 the 64-row kernel
        alone is the faster one on the sparse masks measured."""
        self.B, self.heads, self.T, self.H, self.W, self.d = B, heads, T, H, W, d
        self.N = T * H * W
        self.nb = -(-self.N // BLOCK)
        self.Npad = self.nb * BLOCK
        self.cocluster = order == "cocluster"
        self.cluster_rounds = int(cluster_rounds)
        self.order = ORDER_RASTER if self.cocluster else _ORDERS[order]
        if self.cocluster and select == "structured":
            raise ValueError("the structured rule needs a geometric order (raster or hilbert)")
        self.select = _SELECTS[select]
        self.compensate = bool(compensate)
        self.routing = bool(routing)
        self.shape = shape(B, heads, T, H, W, d)
        self.params = mask_params(self.select, tau, keep_frac, sub_block, win_t, win_rows, n_anchors, 0, seed,
                                  routing, _SCORERS[scorer])
        k = max(1, min(self.nb, math.ceil(float(torch.tensor(keep_frac, dtype=torch.float32)) * self.nb)))
        self.schedule = make_schedule(*schedule) if schedule is not None else None
        # a scheduled top-k rule reaches keep_frac = 1 on its dense steps
        cap = k if (self.select == SEL_TOPK and self.schedule is None) else self.nb
        self.buf = LayerBuffers(B, heads, T, H, W, d, cap=cap, need_means=self.compensate or self.routing,
                                keep_bits=keep_bits or paired_split, ws_bytes=svsa_mask_workspace_bytes(self.shape, self.params),
                                perm_ws_bytes=svsa_perm_workspace_bytes(self.shape, self.order),
                                device=device, compensate=self.compensate, pair_blocks=pair_blocks)
        self._mask = self.buf.mask()
        self._mask.check = int(bool(check_mask))
        if attn_passes is None:
            attn_passes = default_attn_passes(self.select, self.Npad, d)
        self.attn_passes = int(attn_passes)
        self.paired_split = bool(paired_split)
        ws_bytes = (svsa_attn_paired_workspace_bytes if self.paired_split
                    else svsa_attn_split_workspace_bytes)(self.shape, self.attn_passes)
        # (every path has a workspace: at one pass it holds the item schedule)
        self.buf.split_ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=self.buf.qp.device)
        if self.cocluster:
            rows, dev = B * heads, self.buf.qp.device
            b = self.buf
            b.perm_q = torch.empty(rows, self.Npad, dtype=torch.int32, device=dev)
            b.iperm_q = torch.empty(rows, self.N, dtype=torch.int32, device=dev)
            b.perm_k = torch.empty_like(b.perm_q)
            b.iperm_k = torch.empty_like(b.iperm_q)
            b.clu_ws = torch.empty(max(svsa_cocluster_workspace_bytes(self.shape), 16), dtype=torch.uint8, device=dev)
        self._perm_ready = False
        self.mask_ready = False

    # ---- the four steps -------------------------------------------------
    def build_perm(self, stream=None, q=None, k=None):
        b = self.buf
        if self.cocluster:
            if q is None or k is None:
                raise ValueError("the co-clustering order is built from the layer's raster q and k")
            svsa_build_perm_cocluster(q, k, self.shape, self.cluster_rounds, b.perm_q, b.iperm_q, b.perm_k,
                                      b.iperm_k, b.clu_ws, b.clu_ws.numel(), stream)
        else:
            svsa_build_perm(self.shape, self.order, b.perm, b.iperm, b.perm_ws, b.perm_ws.numel(), stream)
        self._perm_ready = True

    def rebuild_order(self):
        """Re-cluster at the next call (the co-clustering order is reused until then)."""
        self._perm_ready = False

    def reorder(self, q, k, v, stream=None):
        if not self._perm_ready:
            self.build_perm(stream, q, k)
        b = self.buf
        if self.cocluster:
            svsa_reorder_heads(q, b.qp, b.perm_q, self.shape, stream)
            svsa_reorder_heads(k, b.kp, b.perm_k, self.shape, stream)
            svsa_reorder_values_heads(v, b.vp, b.perm_k, self.shape, stream)
            return
        svsa_reorder(q, b.qp, b.perm, self.shape, stream)
        svsa_reorder(k, b.kp, b.perm, self.shape, stream)
        svsa_reorder_values(v, b.vp, b.perm, self.shape, stream)

    def build_mask(self, step: int = 0, stream=None):
        """The block mask for denoising step `step` (the structured rule's
        anchors rotate with it; the other rules do not depend on it)."""
        b = self.buf
        self.params.step = int(step)
        svsa_build_mask(b.qp, b.kp, b.vp, None if self.cocluster else b.perm, self.shape, self.params, self._mask,
                        b.ws, b.ws.numel(), stream)
        self.mask_ready = True

    def attend(self, lse=None, stream=None):
        b = self.buf
        if self.paired_split:
            svsa_attn_fwd_paired(b.qp, b.kp, b.vp, self._mask, self.compensate, b.op, lse, self.shape,
                                 self.attn_passes, b.split_ws, b.split_ws.numel(), stream)
        else:
            svsa_attn_fwd_split(b.qp, b.kp, b.vp, self._mask, self.compensate, b.op, lse, self.shape,
                                self.attn_passes, b.split_ws, b.split_ws.numel(), stream)

    def attend_dense(self, lse=None, stream=None):
        b = self.buf
        svsa_attn_dense_fwd(b.qp, b.kp, b.vp, b.op, lse, self.shape, stream)

    def inverse(self, out, stream=None):
        if self.cocluster:
            svsa_inverse_reorder_heads(self.buf.op, out, self.buf.iperm_q, self.shape, stream)
        else:
            svsa_inverse_reorder(self.buf.op, out, self.buf.iperm, self.shape, stream)

    # ---- one denoising step under the schedule ----------------------------
    def step(self, q, k, v, step: int, *, out=None, stream=None):
        """The layer at denoising step `step` of the schedule: the step's rule
        parameter, and a new mask only on the schedule's rebuild steps (the
        others reuse the last mask).  Returns (out, rebuilt)."""
        if self.schedule is None:
            raise ValueError("no schedule given to this layer")
        base = self.params
        p, rebuild = svsa_schedule_step(self.schedule, step, base)
        self.params = p
        if out is None:
            out = torch.empty_like(q)
        build = rebuild or not self.mask_ready
        self.reorder(q, k, v, stream)
        if build:
            self.build_mask(step, stream)
        self.attend(stream=stream)
        self.inverse(out, stream)
        return out, build

    # ---- a group of (batch, head) rows, as a layer of its own -------------
    def _rows(self, t, r0, r1):
        """rows r0..r1 of the flattened (batch, head) dimension of a layer-shaped buffer"""
        return t.reshape((self.B * self.heads,) + tuple(t.shape[2:]))[r0:r1] if t is not None else None

    def _group(self, r0, r1):
        b = self.buf
        sh = shape(1, r1 - r0, self.T, self.H, self.W, self.d)
        m = make_mask(self._rows(b.kv_idx, r0, r1), self._rows(b.kv_cnt, r0, r1), b.cap,
                      self._rows(b.bits, r0, r1), self._rows(b.kbar, r0, r1), self._rows(b.vbar, r0, r1),
                      b.nvalid, self._rows(b.cbar, r0, r1), check=bool(self._mask.check),
                      pairs=self._rows(b.pairs, r0, r1))
        return sh, m

    def forward_host(self, q, k, v, out, *, step: int = 0, reuse_mask: bool = False, groups: int = 12):
        """q, k, v, out: pinned host bf16 [B, heads, N, d] (raster order).  The rows
        are processed in `groups` groups.  Every group's input copies are queued
        first, on one stream, each group ending in an event, so the link stays
        busy whatever the host's launch rate; each group's four library calls
        run on the current stream once its event has fired, and its output is
        copied out on a third stream.  The current stream waits for the last
        copy, so synchronising it covers the layer."""
        b = self.buf
        rows = self.B * self.heads
        if getattr(self, "_stage", None) is None:
            dev = b.qp.device
            self._stage = tuple(torch.empty(rows, self.N, self.d, dtype=torch.bfloat16, device=dev)
                                for _ in range(4))
            self._h2d, self._d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        dq, dk, dv, dout = self._stage
        hq, hk, hv, hout = (t.reshape(rows, self.N, self.d) for t in (q, k, v, out))
        compute = torch.cuda.current_stream()
        if not self._perm_ready:
            if self.cocluster:
                raise ValueError("forward_host needs the co-clustering order built first (a device call)")
            self.build_perm()
        build = not (reuse_mask and self.mask_ready)
        if build:
            self.params.step = int(step)
        # group bounds keep every per-row mask slice 16-byte aligned (the ABI's
        # pointer rule): rows of nb int32 counts must start at a multiple of 4 words
        unit = 4 // math.gcd(self.nb, 4)
        groups = max(1, min(groups, rows))
        bounds = sorted({min(rows, (rows * g // groups) // unit * unit) for g in range(groups)} | {rows})
        # the copy streams start after what the current stream has already queued
        self._h2d.wait_stream(compute)
        self._d2h.wait_stream(compute)
        spans = list(zip(bounds[:-1], bounds[1:]))
        arrived = []
        with torch.cuda.stream(self._h2d):
            for r0, r1 in spans:
                for h, d_ in ((hq, dq), (hk, dk), (hv, dv)):
                    d_[r0:r1].copy_(h[r0:r1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self._h2d)
                arrived.append(ev)
        for (r0, r1), ev in zip(spans, arrived):
            compute.wait_event(ev)
            sh, m = self._group(r0, r1)
            if self.cocluster:
                svsa_reorder_heads(dq[r0:r1], self._rows(b.qp, r0, r1), b.perm_q[r0:r1], sh, compute)
                svsa_reorder_heads(dk[r0:r1], self._rows(b.kp, r0, r1), b.perm_k[r0:r1], sh, compute)
                svsa_reorder_values_heads(dv[r0:r1], self._rows(b.vp, r0, r1), b.perm_k[r0:r1], sh, compute)
            else:
                svsa_reorder(dq[r0:r1], self._rows(b.qp, r0, r1), b.perm, sh, compute)
                svsa_reorder(dk[r0:r1], self._rows(b.kp, r0, r1), b.perm, sh, compute)
                svsa_reorder_values(dv[r0:r1], self._rows(b.vp, r0, r1), b.perm, sh, compute)
            if build:
                svsa_build_mask(self._rows(b.qp, r0, r1), self._rows(b.kp, r0, r1), self._rows(b.vp, r0, r1),
                                None if self.cocluster else b.perm, sh, self.params, m, b.ws, b.ws.numel(),
                                compute)
            if self.paired_split:
                svsa_attn_fwd_paired(self._rows(b.qp, r0, r1), self._rows(b.kp, r0, r1), self._rows(b.vp, r0, r1),
                                     m, self.compensate, self._rows(b.op, r0, r1), None, sh, self.attn_passes,
                                     b.split_ws, b.split_ws.numel(), compute)
            else:
                svsa_attn_fwd_split(self._rows(b.qp, r0, r1), self._rows(b.kp, r0, r1), self._rows(b.vp, r0, r1), m,
                                    self.compensate, self._rows(b.op, r0, r1), None, sh, self.attn_passes,
                                    b.split_ws, b.split_ws.numel(), compute)
            if self.cocluster:
                svsa_inverse_reorder_heads(self._rows(b.op, r0, r1), dout[r0:r1], b.iperm_q[r0:r1], sh, compute)
            else:
                svsa_inverse_reorder(self._rows(b.op, r0, r1), dout[r0:r1], b.iperm, sh, compute)
            self._d2h.wait_stream(compute)
            with torch.cuda.stream(self._d2h):
                hout[r0:r1].copy_(dout[r0:r1], non_blocking=True)
        if build:
            self.mask_ready = True
        compute.wait_stream(self._d2h)
        return out

    # ---- whole layer ----------------------------------------------------
    # ---- the layer as one CUDA graph ---------------------------------------
    def capture(self, q, k, v, out, *, step: int = 0, with_order: bool = False) -> "CapturedLayer":
        """Capture one layer call on these device buffers (reorder, block mask,
        attention, inverse reorder; the token order too with with_order) into
        a CUDA graph.  replay() re-runs it on whatever q, k and v then hold and
        writes `out`, without a host launch per kernel.  The buffers, the
        shape and the mask parameters (the step index included) are fixed at
        capture."""
        if self.cocluster and not with_order and not self._perm_ready:
            raise ValueError("build the co-clustering order first, or capture it with with_order=True")

        def body():
            if with_order or not self._perm_ready:
                self.build_perm(q=q, k=k)
            self.reorder(q, k, v)
            self.build_mask(step)
            self.attend()
            self.inverse(out)

        # allocator-safe warm-up on a side stream, then the capture
        side = torch.cuda.Stream(q.device)
        side.wait_stream(torch.cuda.current_stream(q.device))
        with torch.cuda.stream(side):
            body()
        torch.cuda.current_stream(q.device).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            body()
        return CapturedLayer(graph)

    def __call__(self, q, k, v, *, out=None, step: int = 0, reuse_mask: bool = False, stream=None):
        if out is None:
            out = torch.empty_like(q)
        self.reorder(q, k, v, stream)
        if not (reuse_mask and self.mask_ready):
            self.build_mask(step, stream)
        self.attend(stream=stream)
        self.inverse(out, stream)
        return out
