"""Benchmark of the block-sparse video attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload hunyuan_2x] [--order hilbert]
    python bench.py --impl reference ...      # the fp64 CPU oracle as the reference arm

One step = the whole path over one synthetic layer already resident in HBM,
for one mask cycle of the layer: svsa_build_perm, then at each of the layer's
reuse_steps denoising steps svsa_reorder (Q, K), svsa_reorder_values (V),
svsa_attn_fwd and svsa_inverse_reorder, with svsa_build_mask at the first of
them (the HunyuanVideo layer reuses its mask over 4 steps while Q and K
drift; the other layers build a mask every step).  Each timed step is
bracketed by CUDA events on the launching stream, with an L2 flush (a
512 MiB write) between steps, outside the events.  `value` = kept-block
attention FLOPs of all ranks / the slowest rank's time (TFLOP/s).  Ranks run
independent layers (weak scaling, no collective on the data path; only the
timing max is reduced).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "block-sparse attn fwd ms & kept-FLOP TFLOP/s (% BF16 peak); speedup vs dense"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LONG_STEP_MS = 100.0
ATTN_KERNEL_SRCS = [os.path.join(ROOT, "block_sparse_attention_hilbert_b200", "csrc", f)
                    for f in ("attn_tc.cu", "tcgen05.cuh")]


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="svsa", choices=["svsa", "reference"])
    ap.add_argument("--workload", default="hunyuan_2x", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--secondary", default="wan13b",
                    help="a second, short layer whose attention / dense figures ride along in the line ('' = none)")
    ap.add_argument("--scorer", default=None, choices=["pooled", "sics"])
    ap.add_argument("--attn", default="transposed", choices=["paired", "transposed"],
                    help="sparse attention: the 64-row kernel alone (default) or the paired-block split")
    ap.add_argument("--order", default=None, choices=["raster", "hilbert", "cocluster"])
    ap.add_argument("--heads", type=int, default=None, help="override the layer's head count (profiling captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay of the step")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--schedule", default=None, metavar="N,DENSE,START,END,EVERY",
                    help="time whole denoising runs of the layer under the step schedule "
                         "(svsa_schedule_step): N steps, DENSE dense ones, the rule parameter "
                         "from START to END, the mask rebuilt every EVERY steps")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, ws, local


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _workload(args):
    _LAYER_OPTS["paired_split"] = _LAYER_OPTS["pair_blocks"] = getattr(args, "attn", "transposed") == "paired"
    w = workloads.WORKLOADS[args.workload]
    if args.order:
        w = w.with_(order=args.order)
    if args.heads:
        w = w.with_(heads=args.heads)
    if args.scorer:
        w = w.with_(scorer=args.scorer, sub_block=64 if args.scorer == "sics" else w.sub_block)
    return w


def kept_flops_from_lists(kv_idx: np.ndarray, kv_cnt: np.ndarray, nvalid: np.ndarray, d: int) -> float:
    """4 * d * sum over kept (I, J) of n_I * n_J, from the compacted lists."""
    nb = nvalid.shape[0]
    cap = kv_idx.shape[-1]
    idx = kv_idx.reshape(-1, nb, cap)
    cnt = kv_cnt.reshape(-1, nb)
    mask = np.arange(cap)[None, None, :] < cnt[..., None]
    nJ = np.where(mask, nvalid[np.clip(idx, 0, nb - 1)], 0).sum(-1)       # [BH, nb]
    return 4.0 * d * float((nJ * nvalid[None, :]).sum())


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"svsa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, flag in zip(names, r[3][1:]):
                if flag.lower().startswith("active"):
                    reasons.add(n)
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- traffic
def _attn_traffic(workload: str):
    """dram bytes per attention launch from the committed ncu summary, if it was
    taken on the current kernel source -- attn_tc.cu and tcgen05.cuh, hashed
    together -- (else null)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"attn_{workload}.traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                a, b = line.split(":", 1)
                kv[a.strip()] = b.strip()
    sha = hashlib.sha256()
    for src in ATTN_KERNEL_SRCS:
        with open(src, "rb") as f:
            sha.update(f.read())
    h = sha.hexdigest()[:16]
    if kv.get("kernel_sha256_16") != h:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------------- oracle arm
def _oracle_sample(w, q, k, v, seconds: float, perm_cache=None):
    """Time the fp64 oracle on a bounded sample of the layer: the full permutation,
    then head by head the pooling, the mask rows and the attention of query
    blocks until `seconds` elapse.  Returns (kept_flops, elapsed, description)."""
    import oracle
    from threadpoolctl import threadpool_info
    t0 = time.perf_counter()
    perm, _ = perm_cache if perm_cache is not None else oracle.build_perm(w.T, w.H, w.W, w.order)
    flops = 0.0
    blocks = 0
    heads_done = 0
    nb = w.nb
    k_keep = oracle.topk_count(w.keep_frac, nb)
    for eta in range(min(w.heads, q.shape[1])):
        qp, kp, vp = (oracle.reorder(t[0, eta].float().cpu().numpy().astype(np.float64), perm) for t in (q, k, v))
        qb, nv = oracle.pool(qp, w.N)
        kb, _ = oracle.pool(kp, w.N)
        heads_done += 1
        for I in range(nb):
            if w.select == "structured":
                keep_row = oracle.structured_mask(perm, w.T, w.H, w.W, win_t=w.win_t, win_rows=w.win_rows,
                                                  n_anchors=w.n_anchors, seed=0, step=0)[I]
            else:
                if w.scorer == "sics":
                    if I == 0:
                        S_head = oracle.sics_scores(kp, w.N)
                    S = S_head
                elif w.sub_block == 64:
                    S = oracle.block_scores(qb[I:I + 1], kb)[0]
                else:
                    S = oracle.subblock_scores(qp, kp, w.N, w.sub_block, rows=[I])[0]
                if w.select == "topk":
                    keep_row, _ = oracle.select_topk(S, k_keep)
                else:
                    keep_row, _ = oracle.select_threshold(S, w.tau)
            keep = np.zeros((nb, nb), dtype=bool)
            keep[I] = keep_row
            oracle.masked_attention(qp, kp, vp, w.N, keep, q_blocks=[I])
            flops += oracle.kept_flops(keep, nv, w.d)
            blocks += 1
            if time.perf_counter() - t0 >= seconds:
                break
        if time.perf_counter() - t0 >= seconds:
            break
    elapsed = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    desc = (f"{w.name}: full {w.order} permutation, then per head pooling + mask row + exact attention "
            f"of {blocks} query blocks over {heads_done} head(s) (of {w.heads} x {nb}); "
            f"{flops / 1e12:.4f} kept TFLOP in {elapsed:.1f} s")
    return flops, elapsed, desc, threads


def run_reference(args):
    rank, ws, _ = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0
    if rank != 0:
        return
    import oracle
    w = _workload(args)
    # the sample covers a head or two: generate two heads of the layer's shape
    # (every head has the same shape and input distribution)
    q, k, v = workloads.make_qkv(w.with_(heads=min(w.heads, 2)), device="cpu")
    if w.order not in ("raster", "hilbert"):
        raise SystemExit("the oracle arm samples the geometric orders (raster, hilbert) only")
    perm_cache = oracle.build_perm(w.T, w.H, w.W, w.order)
    per_step = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        _oracle_sample(w, q, k, v, per_step, perm_cache)
    tot_f, tot_t, desc, threads = 0.0, 0.0, "", 1
    for _ in range(args.steps):
        f, t, desc, threads = _oracle_sample(w, q, k, v, per_step, perm_cache)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "heads": w.heads, "d": w.d, "grid": [w.T, w.H, w.W],
                       "N": w.N, "order": w.order, "select": w.select},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"each step: {desc}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU arm
# layer options every GPU arm shares (set from the command line)
_LAYER_OPTS = {"paired_split": False, "pair_blocks": False}


def _layer(svsa, w, dev, seed=0):
    return svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select,
                                     tau=w.tau, keep_frac=w.keep_frac, sub_block=w.sub_block,
                                     win_t=w.win_t, win_rows=w.win_rows,
                                     n_anchors=w.n_anchors if w.select == "structured" else 0,
                                     routing=w.routing, compensate=w.compensate, seed=seed, scorer=w.scorer,
                                     device=dev, **_LAYER_OPTS)


def _timed(fn, stream, flush, warmup, iters):
    """Mean CUDA-event time (ms) of fn() on `stream`, L2 flushed before each call."""
    times = []
    for i in range(warmup + iters):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1))
    return statistics.mean(times)


def _secondary(svsa, name, dev, stream, flush, peaks, steps):
    """Attention and dense figures of a second, short layer (one mask per step)."""
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.make_qkv(w, device=dev)
    attn = _layer(svsa, w, dev)
    out = torch.empty_like(q)
    attn(q, k, v, out=out)
    torch.cuda.synchronize()
    nvalid = np.minimum(64, w.N - 64 * np.arange(w.nb)).astype(np.int64)
    kflops = kept_flops_from_lists(attn.buf.kv_idx.cpu().numpy(), attn.buf.kv_cnt.cpu().numpy(), nvalid, w.d)
    dense_flops = 4.0 * w.d * float(w.N) ** 2 * w.heads * w.B
    step_ms = _timed(lambda: attn(q, k, v, out=out), stream, flush, 3, steps)
    attn_ms = _timed(attn.attend, stream, flush, 3, steps)
    dense_ms = _timed(attn.attend_dense, stream, flush, 3, steps)
    peak = float(peaks["bf16_tflops"])
    res = {"workload": name, "heads": w.heads, "grid": [w.T, w.H, w.W], "select": w.select,
           "keep_frac": w.keep_frac, "step_ms": step_ms, "attn_ms": attn_ms,
           "attn_tflops": kflops / (attn_ms * 1e-3) / 1e12, "dense_ms": dense_ms,
           "dense_tflops": dense_flops / (dense_ms * 1e-3) / 1e12, "speedup_vs_dense": dense_ms / attn_ms,
           "density": kflops / dense_flops}
    res["attn_frac_of_peak"] = res["attn_tflops"] / peak
    res["dense_frac_of_peak"] = res["dense_tflops"] / peak
    res["peak"] = "bf16_tflops (burst)"
    del attn, q, k, v, out
    torch.cuda.empty_cache()
    return res


def run_svsa(args):
    rank, ws, local = _dist()
    import block_sparse_attention_hilbert_b200 as svsa
    assert torch.cuda.is_available(), "bench.py needs a GPU"
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    svsa.lib()
    w = _workload(args)
    stream = torch.cuda.current_stream()
    # one bench step = the layer's mask cycle: the mask is built at the first
    # denoising step and reused for the next reuse_steps - 1, while Q and K
    # drift by sigma * N(0, 1) per step (V does not)
    cycle = max(1, w.reuse_steps)
    q0, k0, v = workloads.make_qkv(w, seed=rank, device=dev)
    qs, ks = [q0], [k0]
    for st in range(1, cycle):
        qs.append(workloads.perturb(qs[-1], sigma=w.sigma, seed=rank, step=st, tensor=workloads.TENSOR_Q))
        ks.append(workloads.perturb(ks[-1], sigma=w.sigma, seed=rank, step=st, tensor=workloads.TENSOR_K))
    attn = _layer(svsa, w, dev)
    out = torch.empty_like(q0)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    phases = ["perm", "reorder", "mask", "attn", "inverse"]

    def cycle_body(acc=None):
        def mark():
            if acc is None:
                return None
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            return e

        def close(phase, e0):
            if acc is not None:
                acc.append((phase, e0, mark()))

        e = mark()
        attn.build_perm(q=q0, k=k0)
        close("perm", e)
        for st in range(cycle):
            e = mark()
            attn.reorder(qs[st], ks[st], v)
            close("reorder", e)
            if st == 0:
                e = mark()
                attn.build_mask(0)
                close("mask", e)
            e = mark()
            attn.attend()
            close("attn", e)
            e = mark()
            attn.inverse(out)
            close("inverse", e)

    for _ in range(max(args.warmup, 3)):
        cycle_body()
    torch.cuda.synchronize()
    nvalid = np.minimum(64, w.N - 64 * np.arange(w.nb)).astype(np.int64)
    kflops = kept_flops_from_lists(attn.buf.kv_idx.cpu().numpy(), attn.buf.kv_cnt.cpu().numpy(), nvalid, w.d)
    dense_flops = 4.0 * w.d * float(w.N) ** 2 * w.heads * w.B
    density = kflops / dense_flops

    times = {p: [] for p in phases}
    attn_launch = []
    launches0 = svsa.svsa_launch_count()
    _barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            flush.fill_(1.0)
            acc = []
            cycle_body(acc)
            torch.cuda.synchronize()
            per = {p: 0.0 for p in phases}
            for phase, e0, e1 in acc:
                ms = e0.elapsed_time(e1)
                per[phase] += ms
                if phase == "attn":
                    attn_launch.append(ms)
            for p in phases:
                times[p].append(per[p])
    torch.cuda.synchronize()
    _barrier(ws)
    launches = svsa.svsa_launch_count() - launches0
    step_ms_local = sum(sum(times[p]) for p in phases) / args.steps
    step_ms = _max_over_ranks(step_ms_local, ws)
    attn_ms = _max_over_ranks(statistics.mean(attn_launch), ws)      # one attention launch

    # the same cycle replayed from a CUDA graph (no host launch per kernel),
    # right after the eager steps so that both see the same clocks; reported
    # beside the eager step, whose per-phase events a graph cannot hold
    graph_ms, graph_err = None, None
    if not args.no_graph:
        try:
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                cycle_body()
            stream.wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                cycle_body()
            graph_ms = _max_over_ranks(_timed(graph.replay, stream, flush, args.warmup, args.steps), ws)
            del graph
        except Exception as exc:                       # reported, not fatal: the eager step is the measure
            graph_err = f"capture failed: {exc}"[:200]

    # pooling on its own (svsa_pool of Q and K at the rule's group size): one HBM pass each
    size = w.sub_block if w.select != "structured" else 64
    pq = torch.empty(w.B, w.heads, w.Npad // size, w.d, dtype=torch.float32, device=dev)
    pk = torch.empty_like(pq)

    def pool_both():
        svsa.svsa_pool(attn.buf.qp, pq, attn.shape, size)
        svsa.svsa_pool(attn.buf.kp, pk, attn.shape, size)

    pool_ms = _max_over_ranks(_timed(pool_both, stream, flush, 3, args.steps), ws)
    pool_bytes = 2 * (w.B * w.heads * w.Npad * w.d * 2 + w.B * w.heads * (w.Npad // size) * w.d * 4)
    del pq, pk

    # dense denominator: same arithmetic over every key block (seconds per launch on
    # the long layers, so at most 3 timed launches there)
    long_layer = attn_ms >= LONG_STEP_MS / 2
    dense_ms = _max_over_ranks(_timed(attn.attend_dense, stream, flush, 1 if long_layer else args.warmup,
                                      min(args.steps, 3) if long_layer else args.steps), ws)

    # end to end through the C entry point on host buffers (svsa_layer_forward_host):
    # pinned host Q, K, V of every step of the cycle in, O of every step back to
    # the host, the copies of one group of heads overlapping the compute of another
    hq = [t.cpu().pin_memory() for t in qs]
    hk = [t.cpu().pin_memory() for t in ks]
    hv = v.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    e2e_groups = min(12, w.B * w.heads)
    # (the co-clustering order is built from the layer's device tensors: that
    # order streams through the Python layer object instead)
    layer = None if attn.cocluster else svsa.svsa_layer_create(attn.shape, svsa.layer_config(
        attn.order, attn.params, compensate=w.compensate, attn_passes=attn.attn_passes,
        paired=attn.paired_split, groups=e2e_groups))

    def e2e_cycle():
        for st in range(cycle):
            if layer is None:
                attn.forward_host(hq[st], hk[st], hv, hout, step=0, reuse_mask=st > 0, groups=e2e_groups)
            else:
                # (the pinned inputs are ready: each step's copies may overlap the previous step's work)
                svsa.svsa_layer_forward_host(layer, hq[st], hk[st], hv, hout, step=0,
                                             flags=svsa.LAYER_INPUTS_READY | (svsa.LAYER_REUSE_MASK if st > 0 else 0),
                                             stream=stream)

    try:
        e2e_ms = _max_over_ranks(_timed(e2e_cycle, stream, flush, args.warmup, args.steps), ws)
    finally:
        if layer is not None:
            svsa.svsa_layer_destroy(layer)
    h2d = cycle * 3 * q0.numel() * q0.element_size()
    d2h = cycle * out.numel() * out.element_size()
    del hq, hk, hv, hout

    peaks, peak_src = _peaks()
    # a kernel inside steps of 100 ms or more runs seconds-long loops under the
    # power cap: its denominator is the sustained GEMM rate, else the burst one
    sustained = step_ms >= LONG_STEP_MS
    peak = float(peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"])
    attn_tflops = kflops / (attn_ms * 1e-3) / 1e12
    cycle_flops = cycle * kflops
    value = ws * cycle_flops / (step_ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        f, t, desc, threads = _oracle_sample(w, q0, k0, v, args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}
    secondary = None
    if rank == 0 and ws == 1 and args.secondary and args.secondary != w.name:
        secondary = _secondary(svsa, args.secondary, dev, stream, flush, peaks, args.steps)

    if rank == 0:
        reorder_bytes = cycle * 3 * (w.B * w.heads * (w.N + w.Npad) * w.d * 2)
        inverse_bytes = cycle * w.B * w.heads * (w.N + w.Npad) * w.d * 2
        reorder_ms = statistics.mean(times["reorder"])
        inverse_ms = statistics.mean(times["inverse"])
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "heads": w.heads, "d": w.d, "grid": [w.T, w.H, w.W],
                       "N": w.N, "order": w.order, "select": w.select, "keep_frac": w.keep_frac,
                       "tau": w.tau, "sub_block": w.sub_block, "routing": w.routing,
                       "compensate": w.compensate, "scorer": w.scorer,
                       "attention": "paired-block split" if _LAYER_OPTS["paired_split"] else "64-row kernel",
                       "step": (f"one mask cycle: perm, mask at the first of {cycle} denoising steps, then "
                                f"reorder + attention + inverse at each of the {cycle} steps (Q, K drift by "
                                f"sigma={w.sigma} between steps)") if cycle > 1 else
                               "perm + reorder + mask + attention + inverse",
                       "l2": "flushed (512 MiB write) between timed steps",
                       "parallelism": f"independent layer per GPU x{ws}"},
            "attn_ms": attn_ms, "attn_tflops": attn_tflops, "attn_frac_of_peak": attn_tflops / peak,
            "attn_passes": attn.attn_passes,
            "dense_ms": dense_ms, "dense_tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
            "dense_frac_of_peak": dense_flops / (dense_ms * 1e-3) / 1e12 / peak,
            "speedup_vs_dense": dense_ms / attn_ms, "density": density,
            "kept_tflop_per_attention": kflops / 1e12, "kept_tflop_per_step": cycle_flops / 1e12,
            "graph": ({"ms_per_step": graph_ms, "value": ws * cycle_flops / (graph_ms * 1e-3) / 1e12}
                      if graph_ms is not None else ({"unavailable": graph_err} if graph_err else None)),
            "phase_ms": {p: statistics.mean(times[p]) for p in phases},
            "reorder_gbs": reorder_bytes / (reorder_ms * 1e-3) / 1e9,
            "inverse_gbs": inverse_bytes / (inverse_ms * 1e-3) / 1e9,
            "pool": {"ms": pool_ms, "gbs": pool_bytes / (pool_ms * 1e-3) / 1e9,
                     "frac_of_hbm": pool_bytes / (pool_ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                     "what": f"svsa_pool of Q and K ({size}-token groups), read bf16 + write fp32 means"},
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": attn_tflops / peak, "traffic": _attn_traffic(w.name),
                         "kernel": "svsa attention (kept-block FLOPs / launch time)",
                         "peak_source": f"{peak_src} " + ("bf16_tflops_sustained (step >= 100 ms)" if sustained
                                                           else "bf16_tflops (burst)")},
            "e2e": {"value": ws * cycle_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "path": (f"svsa_layer_forward_host (C entry point, pinned host buffers, {e2e_groups} row "
                             "groups; the token order built once at svsa_layer_create)") if not attn.cocluster else
                            f"SparseVideoAttention.forward_host (pinned host buffers, {e2e_groups} row groups)"},
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------- schedule mode
def run_schedule(args):
    """One bench step = one whole denoising run of the layer under the step
    schedule: every step reorders, builds its mask only on the schedule's
    rebuild steps, attends and reorders back (same inputs every step)."""
    rank, ws, local = _dist()
    import block_sparse_attention_hilbert_b200 as svsa
    assert torch.cuda.is_available(), "bench.py needs a GPU"
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    svsa.lib()
    w = _workload(args)
    n, dense, start, end, every = args.schedule.split(",")
    sched = (int(n), int(dense), float(start), float(end), int(every))
    n = sched[0]
    stream = torch.cuda.current_stream()
    q, k, v = workloads.make_qkv(w, seed=rank, device=dev)
    attn = svsa.SparseVideoAttention(w.B, w.heads, w.T, w.H, w.W, w.d, order=w.order, select=w.select,
                                     tau=w.tau, keep_frac=w.keep_frac, sub_block=w.sub_block,
                                     routing=w.routing, compensate=w.compensate, schedule=sched, device=dev,
                                     **_LAYER_OPTS)
    out = torch.empty_like(q)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    nvalid = np.minimum(64, w.N - 64 * np.arange(w.nb)).astype(np.int64)
    # untimed pass: the kept FLOPs of every step's mask
    kf, builds = [], 0
    for st in range(n):
        _, rebuilt = attn.step(q, k, v, st, out=out)
        if rebuilt:
            builds += 1
            torch.cuda.synchronize()
            cur = kept_flops_from_lists(attn.buf.kv_idx.cpu().numpy(), attn.buf.kv_cnt.cpu().numpy(), nvalid, w.d)
        kf.append(cur)
    kflops = float(sum(kf))
    dense_flops = 4.0 * w.d * float(w.N) ** 2 * w.heads * w.B * n

    def run():
        for st in range(n):
            attn.step(q, k, v, st, out=out)

    for _ in range(max(args.warmup, 3)):
        run()
    torch.cuda.synchronize()
    launches0 = svsa.svsa_launch_count()
    times = []
    _barrier(ws)
    with ClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            flush.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
    _barrier(ws)
    launches = svsa.svsa_launch_count() - launches0
    run_ms = _max_over_ranks(statistics.mean(times), ws)
    # the same run with dense attention on every step: the denominator of the speedup
    dtimes = []
    for i in range(2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for st in range(n):
            attn.reorder(q, k, v)
            attn.attend_dense()
            attn.inverse(out)
        e1.record(stream)
        torch.cuda.synchronize()
        dtimes.append(e0.elapsed_time(e1))
    dense_run_ms = _max_over_ranks(min(dtimes), ws)
    if rank == 0:
        line = {
            "metric": "block-sparse attn fwd, whole denoising run under the step schedule: kept TFLOP/s",
            "value": ws * kflops / (run_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": run_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "heads": w.heads, "d": w.d, "grid": [w.T, w.H, w.W], "select": w.select,
                       "schedule": {"n_steps": sched[0], "dense_steps": sched[1], "start": sched[2],
                                    "end": sched[3], "refresh_every": sched[4]},
                       "l2": "flushed (512 MiB write) between timed runs",
                       "step": "one bench step = one whole denoising run of the layer"},
            "ms_per_denoising_step": run_ms / n, "mask_builds_per_run": builds,
            "density_per_run": kflops / dense_flops, "dense_run_ms": dense_run_ms,
            "speedup_vs_dense": dense_run_ms / run_ms, "gpu_launches": launches,
            "clocks": clk.summary(),
            "e2e": None, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    elif args.schedule is not None:
        run_schedule(args)
    else:
        run_svsa(args)


if __name__ == "__main__":
    main()
