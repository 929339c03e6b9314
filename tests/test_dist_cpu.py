"""bench.py's multi-rank plumbing on CPU: two gloo ranks, barrier and the
max-over-ranks reduction of the step time (no GPU)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    r, ws, _ = bench._dist()
    assert (r, ws) == (rank, world)
    bench._barrier(ws)
    out[rank] = bench._max_over_ranks(1.5 + rank, ws)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_max_reduction():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_needs_no_process_group():
    os.environ.pop("WORLD_SIZE", None)
    assert bench._dist() == (0, 1, 0)
    assert bench._max_over_ranks(3.25, 1) == 3.25


def test_kept_flops_from_lists():
    # 3 blocks (last has 8 valid tokens), cap 3; rows keep {0}, {0,2}, {1,2}
    idx = np.array([[[0, 9, 9], [0, 2, 9], [1, 2, 9]]], dtype=np.int32)
    cnt = np.array([[1, 2, 2]], dtype=np.int32)
    n = np.array([64, 64, 8])
    expect = 4 * 128 * (64 * 64 + 64 * (64 + 8) + 8 * (64 + 8))
    assert bench.kept_flops_from_lists(idx, cnt, n, 128) == expect


def test_traffic_is_reported_only_for_the_profiled_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from a committed ncu figure only while the
    attention sources still hash to the value recorded with it; any edit of
    them turns it into null (the counters no longer describe the kernel)."""
    import hashlib
    srcs = []
    for name, body in (("attn_tc.cu", b"kernel v1\n"), ("tcgen05.cuh", b"helpers\n")):
        p = tmp_path / name
        p.write_bytes(body)
        srcs.append(str(p))
    h = hashlib.sha256()
    for p in srcs:
        h.update(open(p, "rb").read())
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "attn_demo.traffic.txt").write_text(
        f"# comment: 1\ndram_bytes_per_launch: 12345\nkernel_sha256_16: {h.hexdigest()[:16]}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "ATTN_KERNEL_SRCS", srcs)
    assert bench._attn_traffic("demo") == 12345.0
    assert bench._attn_traffic("missing") is None
    (tmp_path / "attn_tc.cu").write_bytes(b"kernel v2\n")
    assert bench._attn_traffic("demo") is None


def test_committed_traffic_file_is_well_formed():
    """The committed wan13b figure parses and is at least the algorithmic
    Q, K, V, O bytes of a launch within 5% (DRAM bytes below the algorithmic
    ones would mean a capture of some other launch)."""
    path = os.path.join(bench.ROOT, "profiles", "attn_wan13b.traffic.txt")
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            a, b = line.split(":", 1)
            kv[a.strip()] = b.strip()
    assert len(kv["kernel_sha256_16"]) == 16
    algorithmic = 4 * 12 * 32768 * 128 * 2
    assert 0.95 * algorithmic <= float(kv["dram_bytes_per_launch"]) <= 1.25 * algorithmic
