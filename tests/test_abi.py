"""C ABI checks that need no GPU: the library loads, exports every entry point
that include/svsa.h declares, and rejects bad arguments before launching."""
import ctypes
import os
import re

import numpy as np

import pytest

import block_sparse_attention_hilbert_b200 as svsa
from block_sparse_attention_hilbert_b200 import Shape, MaskParams, Mask

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(svsa_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    lib = svsa.lib()
    declared = _declared()
    assert {"svsa_reorder", "svsa_build_mask", "svsa_attn_fwd", "svsa_inverse_reorder"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    # the binding wraps every declared entry point
    assert declared <= set(svsa.exported_symbols())


def test_struct_sizes_match_header():
    assert ctypes.sizeof(Shape) == 24
    assert ctypes.sizeof(MaskParams) == 48
    assert ctypes.sizeof(Mask) == 80


def test_struct_layouts_match_the_c_compiler(tmp_path):
    # every field offset of the binding's structures equals the C compiler's
    # for include/svsa.h (a C probe built with gcc)
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    structs = {"svsa_shape": Shape, "svsa_mask_params": MaskParams, "svsa_mask": Mask,
               "svsa_layer_config": svsa.LayerConfig}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "svsa.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    seen = 0
    for line in out:
        if not line:
            continue
        cname, field, val = line.split()
        cls = structs[cname]
        want = ctypes.sizeof(cls) if field == "size" else getattr(cls, field).offset
        assert int(val) == want, (cname, field, val, want)
        seen += 1
    assert seen == sum(len(c._fields_) + 1 for c in structs.values())


def test_anchor_offset_entry_point_matches_the_oracle():
    # the library's host-side Philox4x32-10 draw against the oracle's, bit for bit
    import oracle
    rng = np.random.default_rng(2024)
    for i in range(1000):
        seed = int(rng.integers(0, 2**63)) * (2 if i % 3 else 1) % 2**64
        step = int(rng.integers(0, 2**31)) if i % 2 else i
        nb = int(rng.integers(1, 16385))
        n = int(rng.integers(0, min(nb, 16) + 1))
        assert svsa.svsa_anchor_offset(seed, step, nb, n) == oracle.anchor_offset(seed, step, nb, n), (seed, step, nb, n)
    # rejections
    lib = svsa.lib()
    out = ctypes.c_int32(0)
    assert lib.svsa_anchor_offset(0, -1, 512, 4, ctypes.byref(out)) == 1
    assert lib.svsa_anchor_offset(0, 0, 0, 0, ctypes.byref(out)) == 1
    assert lib.svsa_anchor_offset(0, 0, 4, 5, ctypes.byref(out)) == 1
    assert lib.svsa_anchor_offset(0, 0, 4, 1, None) == 1


def test_version():
    assert "sm_100a" in svsa.version()


def test_workspace_queries():
    s = svsa.shape(1, 12, 21, 30, 52, 128)
    assert svsa.svsa_perm_workspace_bytes(s, svsa.ORDER_RASTER) == 0
    # 64^3 cube -> 2^18 bits
    assert svsa.svsa_perm_workspace_bytes(s, svsa.ORDER_HILBERT) >= 2 * (1 << 18) // 8
    nb = 512
    p = svsa.mask_params(svsa.SEL_TOPK)
    assert svsa.svsa_mask_workspace_bytes(s, p) >= 12 * nb * nb * 4
    # the structured rule needs workspace only for the query-block pairing table ([BH, nb, 32] int16)
    assert svsa.svsa_mask_workspace_bytes(s, svsa.mask_params(svsa.SEL_STRUCTURED)) >= 12 * nb * 32 * 2
    p16 = svsa.mask_params(svsa.SEL_THRESHOLD, sub_block=16)
    assert svsa.svsa_mask_workspace_bytes(s, p16) > svsa.svsa_mask_workspace_bytes(s, p)
    assert svsa.svsa_mask_workspace_bytes(s, svsa.mask_params(sub_block=32)) == 0
    # attention: one plain pass needs none; the paired-block split needs at
    # least its fp32 partial output [BH, Npad, d] and lse, the exclusive lists
    # [BH, nb, nb] and counts; key-range passes add their lists and outputs
    rows, npad = 12 * nb, nb * 64
    assert svsa.svsa_attn_split_workspace_bytes(s, 1) == 0
    need1 = 12 * npad * 128 * 4 + 12 * npad * 4 + rows * nb * 4 + rows * 4
    assert svsa.svsa_attn_paired_workspace_bytes(s, 1) >= need1
    for P in (2, 3, 8):
        R = -(-nb // P)
        split = svsa.svsa_attn_split_workspace_bytes(s, P)
        # range lists and counts, fp32 outputs and lse, the item schedule
        assert split >= P * (rows * R * 4 + rows * 4 + 12 * npad * 128 * 4 + 12 * npad * 4 + rows * 4)
        assert svsa.svsa_attn_paired_workspace_bytes(s, P) >= split + 12 * npad * 128 * 4 + rows * R * 4
    for P in (0, 9):
        assert svsa.svsa_attn_split_workspace_bytes(s, P) == 0
        assert svsa.svsa_attn_paired_workspace_bytes(s, P) == 0


def _raw():
    return svsa.lib()


def _err():
    return _raw().svsa_last_error().decode()


def test_build_perm_rejects_before_launch():
    lib = _raw()
    s = svsa.shape(1, 1, 4, 8, 8, 64)
    assert lib.svsa_build_perm(s, 1, None, None, None, 0, None) == 1
    assert "perm" in _err()
    assert lib.svsa_build_perm(s, 7, 16, 32, None, 0, None) == 1
    assert lib.svsa_build_perm(svsa.shape(1, 1, 0, 8, 8, 64), 0, 16, 32, None, 0, None) == 1
    assert lib.svsa_build_perm(s, 0, 17, 32, None, 0, None) == 1          # misaligned
    assert "aligned" in _err()
    assert lib.svsa_build_perm(s, 1, 16, 32, 48, 8, None) == 3            # workspace too small
    assert lib.svsa_build_perm(svsa.shape(1, 1, 2000, 2, 2, 64), 1, 16, 32, 48, 1 << 30, None) == 2


def test_reorder_and_attention_reject_before_launch():
    lib = _raw()
    s = svsa.shape(1, 2, 4, 8, 8, 96)                                     # d = 96 unsupported
    assert lib.svsa_reorder(16, 32, 48, s, None) == 2
    s = svsa.shape(1, 2, 4, 8, 8, 128)
    assert lib.svsa_reorder(16, 16, 48, s, None) == 1                     # aliasing
    assert lib.svsa_inverse_reorder(None, 32, 48, s, None) == 1
    m = Mask(None, None, 4, None, None, None, None, None)
    assert lib.svsa_attn_fwd(16, 32, 48, ctypes.byref(m), 0, 64, None, s, None) == 1
    m = Mask(16, 32, 4, None, None, None, None, None, None, 0)
    assert lib.svsa_attn_fwd(16, 32, 48, ctypes.byref(m), 1, 64, None, s, None) == 1   # comp w/o means
    assert "kbar" in _err()
    kb = 80
    m = Mask(16, 32, 4, None, kb, kb + 16, None, None)
    assert lib.svsa_attn_fwd(16, 32, 48, ctypes.byref(m), 1, 64, None, s, None) == 1   # comp w/o bits
    assert "bits" in _err()
    m = Mask(16, 32, 4, 96, kb, kb + 16, None, None)
    assert lib.svsa_attn_fwd(16, 32, 48, ctypes.byref(m), 1, 64, None, s, None) == 1   # comp w/o scratch
    assert "cbar" in _err()
    assert lib.svsa_attn_dense_fwd(16, 32, 48, 16, None, s, None) == 1    # output aliases input
    assert lib.svsa_attn_fwd(16, 32, 48, None, 0, 64, None, s, None) == 1


def test_split_and_paired_attention_reject_before_launch():
    lib = _raw()
    s = svsa.shape(1, 2, 4, 8, 8, 128)                                    # nb = 4
    m = Mask(16, 32, 4, None, None, None, None, None, None, 0)
    ws_need = svsa.svsa_attn_split_workspace_bytes(s, 2)
    assert ws_need > 0
    # passes outside [1, 8]
    for P in (0, 9):
        assert lib.svsa_attn_fwd_split(16, 32, 48, ctypes.byref(m), 0, 64, None, s, P, 80, 1 << 30, None) == 1
        assert lib.svsa_attn_fwd_paired(16, 32, 48, ctypes.byref(m), 0, 64, None, s, P, 80, 1 << 30, None) == 1
    # a workspace smaller than the query
    assert lib.svsa_attn_fwd_split(16, 32, 48, ctypes.byref(m), 0, 64, None, s, 2, 80, ws_need - 1, None) == 3
    assert lib.svsa_attn_fwd_split(16, 32, 48, ctypes.byref(m), 0, 64, None, s, 2, None, ws_need, None) == 1
    # the paired split needs the kept-block bitmap, and its own (larger) workspace
    assert lib.svsa_attn_fwd_paired(16, 32, 48, ctypes.byref(m), 0, 64, None, s, 1, 80, 1 << 30, None) == 1
    assert "bits" in _err()
    mb = Mask(16, 32, 4, 96, None, None, None, None, None, 0)
    need_p = svsa.svsa_attn_paired_workspace_bytes(s, 1)
    assert lib.svsa_attn_fwd_paired(16, 32, 48, ctypes.byref(mb), 0, 64, None, s, 1, 80, need_p - 1, None) == 3
    # the output may not alias an input
    assert lib.svsa_attn_fwd_paired(16, 32, 48, ctypes.byref(mb), 0, 16, None, s, 1, 80, need_p, None) == 1


def test_build_mask_rejects_before_launch():
    lib = _raw()
    s = svsa.shape(1, 2, 4, 8, 8, 128)                                    # nb = 4
    m = Mask(16, 32, 4, None, None, None, None, None, None, 0)
    ok = svsa.mask_params(svsa.SEL_THRESHOLD)
    # capacity below nb for a threshold rule
    small = Mask(16, 32, 3, None, None, None, None, None, None, 0)
    assert lib.svsa_build_mask(16, 32, None, None, s, ctypes.byref(ok), ctypes.byref(small), 64, 1 << 20, None) == 1
    # routing without V / means
    r = svsa.mask_params(svsa.SEL_THRESHOLD, routing=True)
    assert lib.svsa_build_mask(16, 32, None, None, s, ctypes.byref(r), ctypes.byref(m), 64, 1 << 20, None) == 1
    # routing with a non-threshold rule
    r2 = svsa.mask_params(svsa.SEL_TOPK, routing=True)
    assert lib.svsa_build_mask(16, 32, 48, None, s, ctypes.byref(r2), ctypes.byref(m), 64, 1 << 20, None) == 1
    # structured without perm
    st = svsa.mask_params(svsa.SEL_STRUCTURED, n_anchors=2, step=0)
    assert lib.svsa_build_mask(None, None, None, None, s, ctypes.byref(st), ctypes.byref(m), None, 0, None) == 1
    # a negative step index
    st2 = svsa.mask_params(svsa.SEL_STRUCTURED, n_anchors=2, step=-3)
    assert lib.svsa_build_mask(None, None, None, 16, s, ctypes.byref(st2), ctypes.byref(m), None, 0, None) == 1
    # more anchors than blocks
    st3 = svsa.mask_params(svsa.SEL_STRUCTURED, n_anchors=5)
    assert lib.svsa_build_mask(None, None, None, 16, s, ctypes.byref(st3), ctypes.byref(m), None, 0, None) == 1
    # the SICS scorer: not for the structured rule, only 64-token blocks, no routing, unknown scorer
    sx = svsa.mask_params(svsa.SEL_STRUCTURED, scorer=svsa.SCORE_SICS)
    assert lib.svsa_build_mask(None, 32, None, 16, s, ctypes.byref(sx), ctypes.byref(m), 64, 1 << 20, None) == 1
    sx = svsa.mask_params(svsa.SEL_TOPK, sub_block=16, scorer=svsa.SCORE_SICS)
    assert lib.svsa_build_mask(None, 32, None, None, s, ctypes.byref(sx), ctypes.byref(m), 64, 1 << 20, None) == 2
    sx = svsa.mask_params(svsa.SEL_THRESHOLD, routing=True, scorer=svsa.SCORE_SICS)
    assert lib.svsa_build_mask(16, 32, 48, None, s, ctypes.byref(sx), ctypes.byref(m), 64, 1 << 20, None) == 2
    sx = svsa.mask_params(svsa.SEL_TOPK, scorer=7)
    assert lib.svsa_build_mask(16, 32, None, None, s, ctypes.byref(sx), ctypes.byref(m), 64, 1 << 20, None) == 1
    # the SICS scorer needs no queries but its workspace
    sx = svsa.mask_params(svsa.SEL_TOPK, scorer=svsa.SCORE_SICS)
    need = svsa.svsa_mask_workspace_bytes(s, sx)
    assert need > 0
    assert lib.svsa_build_mask(None, 32, None, None, s, ctypes.byref(sx), ctypes.byref(m), 64, need - 1, None) == 3
    # workspace too small
    assert lib.svsa_build_mask(16, 32, None, None, s, ctypes.byref(ok), ctypes.byref(m), 64, 16, None) == 3
    # unknown selection rule / sub-block size
    bad = svsa.mask_params(5)
    assert lib.svsa_build_mask(16, 32, None, None, s, ctypes.byref(bad), ctypes.byref(m), 64, 1 << 20, None) == 1
    bad = svsa.mask_params(svsa.SEL_THRESHOLD, sub_block=32)
    assert lib.svsa_build_mask(16, 32, None, None, s, ctypes.byref(bad), ctypes.byref(m), 64, 1 << 20, None) == 2


def test_status_codes_are_stable():
    # values are part of the ABI
    text = open(os.path.join(ROOT, "include", "svsa.h")).read()
    for name, val in [("SVSA_OK", 0), ("SVSA_ERR_INVALID_ARG", 1), ("SVSA_ERR_UNSUPPORTED", 2),
                      ("SVSA_ERR_WORKSPACE", 3), ("SVSA_ERR_CUDA", 4), ("SVSA_ERR_TIMEOUT", 5),
                      ("SVSA_ERR_RANGE", 6), ("SVSA_ERR_MASK", 7)]:
        assert re.search(rf"{name}\s*=\s*{val}\b", text)


@pytest.mark.parametrize("n,dense,start,end,every", [
    (50, 5, 0.97, 0.85, 5), (12, 0, 0.5, 0.2, 3), (7, 7, 0.9, 0.1, 2), (3, 2, 0.9, 0.1, 1), (1, 0, 0.3, 0.3, 4)])
@pytest.mark.parametrize("select", [svsa.SEL_THRESHOLD, svsa.SEL_TOPK])
def test_schedule_step_matches_the_oracle(n, dense, start, end, every, select):
    """Host-only entry point: the step's rule parameter is the oracle's float32
    value bit for bit, and the rebuild flags are the oracle's pattern."""
    import oracle
    sch = svsa.schedule(n, dense, start, end, every)
    base = svsa.mask_params(select, tau=0.5, keep_frac=0.5)
    flags = oracle.rebuilds(n, dense, every)
    for s in range(n):
        p, rebuild = svsa.svsa_schedule_step(sch, s, base)
        got = p.tau if select == svsa.SEL_THRESHOLD else p.keep_frac
        other = p.keep_frac if select == svsa.SEL_THRESHOLD else p.tau
        assert got == oracle.step_param(n, dense, start, end, s)
        assert other == np.float32(0.5)                       # the other field is untouched
        assert rebuild == flags[s]


def test_schedule_step_rejects():
    lib = _raw()
    sch = svsa.schedule(10, 2, 0.9, 0.5, 3)
    out = svsa.MaskParams()
    r = ctypes.c_int32(0)
    base = svsa.mask_params(svsa.SEL_STRUCTURED)
    assert lib.svsa_schedule_step(ctypes.byref(sch), 0, ctypes.byref(base), ctypes.byref(out), ctypes.byref(r)) == 2
    base = svsa.mask_params(svsa.SEL_THRESHOLD)
    assert lib.svsa_schedule_step(ctypes.byref(sch), 10, ctypes.byref(base), ctypes.byref(out), ctypes.byref(r)) == 1
    bad = svsa.schedule(10, 11, 0.9, 0.5, 3)
    assert lib.svsa_schedule_step(ctypes.byref(bad), 0, ctypes.byref(base), ctypes.byref(out), ctypes.byref(r)) == 1
    bad = svsa.schedule(10, 2, 0.9, 0.5, 0)
    assert lib.svsa_schedule_step(ctypes.byref(bad), 0, ctypes.byref(base), ctypes.byref(out), ctypes.byref(r)) == 1


def test_default_attention_passes():
    """Key-range passes by rule and head size: one while K and V of a head
    fit in 48 MB (and always for the structured rule), else 32 MB each."""
    from block_sparse_attention_hilbert_b200.pipeline import default_attn_passes
    mb = 2**20
    rows = lambda nbytes, d=128: nbytes // (d * 4)          # Npad giving that many K+V bytes
    assert default_attn_passes(svsa.SEL_TOPK, 512 * 64, 128) == 1          # the wan13b layer, 16.8 MB
    assert default_attn_passes(svsa.SEL_THRESHOLD, rows(48 * mb), 128) == 1
    assert default_attn_passes(svsa.SEL_THRESHOLD, rows(48 * mb) + 64, 128) == 2
    assert default_attn_passes(svsa.SEL_THRESHOLD, 3488 * 64, 128) == 4     # HunyuanVideo, 114 MB
    assert default_attn_passes(svsa.SEL_STRUCTURED, 3072 * 64, 128) == 1    # the 6x Wan layer, 101 MB
    assert default_attn_passes(svsa.SEL_TOPK, rows(1024 * mb), 128) == 8    # capped


def test_layer_configuration_checks_need_no_gpu():
    # the host-buffer layer validates its configuration before any CUDA call
    lib = svsa.lib()
    s = svsa.shape(1, 12, 21, 30, 52, 128)
    mp = svsa.mask_params(svsa.SEL_THRESHOLD)
    good = svsa.layer_config(svsa.ORDER_HILBERT, mp, groups=12)
    nb, npad, N = 512, 512 * 64, 21 * 30 * 52
    # at least: four reordered and four raster token tensors, the lists at cap = nb
    need = 12 * (4 * npad + 4 * N) * 128 * 2 + 12 * nb * nb * 4
    assert svsa.svsa_layer_device_bytes(s, good) >= need
    comp = svsa.layer_config(svsa.ORDER_HILBERT, mp, compensate=True, attn_passes=2, groups=3)
    assert svsa.svsa_layer_device_bytes(s, comp) > svsa.svsa_layer_device_bytes(s, good)
    h = ctypes.c_void_p(1)
    bad = [(svsa.layer_config(2, mp), 2),                          # the co-clustering order: unsupported
           (svsa.layer_config(svsa.ORDER_RASTER, mp, groups=0), 1),
           (svsa.layer_config(svsa.ORDER_RASTER, mp, groups=13), 1),
           (svsa.layer_config(svsa.ORDER_RASTER, mp, attn_passes=9), 1)]
    for cfg, status in bad:
        assert svsa.svsa_layer_device_bytes(s, cfg) == 0
        assert lib.svsa_layer_create(s, ctypes.byref(cfg), ctypes.byref(h)) == status
        assert h.value is None
        assert lib.svsa_last_error()
    assert lib.svsa_layer_create(svsa.shape(1, 12, 21, 30, 52, 96), ctypes.byref(good), ctypes.byref(h)) == 2
    assert lib.svsa_layer_create(s, None, ctypes.byref(h)) == 1
    assert lib.svsa_layer_create(s, ctypes.byref(good), None) == 1
    assert lib.svsa_layer_forward_host(None, 16, 16, 16, 16, 0, 0, None) == 1
    assert lib.svsa_layer_destroy(None) == 0
