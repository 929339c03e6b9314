"""Python binding of libsvsa, the B200 block-sparse video attention library.

Argument marshalling only: each function passes raw device pointers, sizes and
the current CUDA stream to the C entry point of the same name (see
include/svsa.h) and raises SvsaError on a non-zero status.  Every step of the
computation runs in the library's CUDA kernels; torch supplies device memory
and streams.  If the shared library is missing, importing works but every
call raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libsvsa.so")

ORDER_RASTER, ORDER_HILBERT = 0, 1
SEL_THRESHOLD, SEL_TOPK, SEL_STRUCTURED = 0, 1, 2
SCORE_POOLED, SCORE_SICS = 0, 1
BLOCK = 64

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA", 5: "TIMEOUT", 6: "RANGE",
          7: "MASK"}


class SvsaError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("heads", ctypes.c_int32), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("W", ctypes.c_int32), ("d", ctypes.c_int32)]


class MaskParams(ctypes.Structure):
    _fields_ = [("select", ctypes.c_int32), ("tau", ctypes.c_float), ("keep_frac", ctypes.c_float),
                ("sub_block", ctypes.c_int32), ("win_t", ctypes.c_int32), ("win_rows", ctypes.c_int32),
                ("n_anchors", ctypes.c_int32), ("step", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("routing", ctypes.c_int32), ("scorer", ctypes.c_int32)]


class Mask(ctypes.Structure):
    _fields_ = [("kv_idx", ctypes.c_void_p), ("kv_cnt", ctypes.c_void_p), ("cap", ctypes.c_int32),
                ("bits", ctypes.c_void_p), ("kbar", ctypes.c_void_p), ("vbar", ctypes.c_void_p),
                ("nvalid", ctypes.c_void_p), ("cbar", ctypes.c_void_p), ("pairs", ctypes.c_void_p),
                ("check", ctypes.c_int32)]


class LayerConfig(ctypes.Structure):
    _fields_ = [("order", ctypes.c_int32), ("mask", MaskParams), ("compensate", ctypes.c_int32),
                ("attn_passes", ctypes.c_int32), ("paired", ctypes.c_int32), ("groups", ctypes.c_int32)]


LAYER_REUSE_MASK = 1
LAYER_INPUTS_READY = 2


class Schedule(ctypes.Structure):
    _fields_ = [("n_steps", ctypes.c_int32), ("dense_steps", ctypes.c_int32), ("start", ctypes.c_float),
                ("end", ctypes.c_float), ("refresh_every", ctypes.c_int32)]


_lib = None

_SIGS = {
    "svsa_perm_workspace_bytes": (ctypes.c_size_t, [Shape, ctypes.c_int32]),
    "svsa_build_perm": (ctypes.c_int, [Shape, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "svsa_build_perm_noalloc": (ctypes.c_int, [Shape, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p]),
    "svsa_reorder": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, Shape,
                                    ctypes.c_void_p]),
    "svsa_reorder_values": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, Shape,
                                           ctypes.c_void_p]),
    "svsa_pool": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_int32, ctypes.c_void_p]),
    "svsa_mask_workspace_bytes": (ctypes.c_size_t, [Shape, ctypes.POINTER(MaskParams)]),
    "svsa_build_mask": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, Shape, ctypes.POINTER(MaskParams),
                                       ctypes.POINTER(Mask), ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]),
    "svsa_attn_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.POINTER(Mask), ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_void_p, Shape, ctypes.c_void_p]),
    "svsa_attn_split_workspace_bytes": (ctypes.c_size_t, [Shape, ctypes.c_int32]),
    "svsa_attn_fwd_split": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.POINTER(Mask), ctypes.c_int32, ctypes.c_void_p,
                                           ctypes.c_void_p, Shape, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p]),
    "svsa_layer_device_bytes": (ctypes.c_size_t, [Shape, ctypes.POINTER(LayerConfig)]),
    "svsa_layer_create": (ctypes.c_int, [Shape, ctypes.POINTER(LayerConfig), ctypes.POINTER(ctypes.c_void_p)]),
    "svsa_layer_forward_host": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]),
    "svsa_layer_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "svsa_attn_paired_workspace_bytes": (ctypes.c_size_t, [Shape, ctypes.c_int32]),
    "svsa_attn_fwd_paired": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.POINTER(Mask), ctypes.c_int32, ctypes.c_void_p,
                                            ctypes.c_void_p, Shape, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t,
                                            ctypes.c_void_p]),
    "svsa_attn_dense_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_void_p]),
    "svsa_inverse_reorder": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, Shape,
                                            ctypes.c_void_p]),
    "svsa_cocluster_workspace_bytes": (ctypes.c_size_t, [Shape]),
    "svsa_build_perm_cocluster": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, Shape, ctypes.c_int32,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "svsa_reorder_heads": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, Shape,
                                          ctypes.c_void_p]),
    "svsa_reorder_values_heads": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, Shape,
                                                 ctypes.c_void_p]),
    "svsa_inverse_reorder_heads": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, Shape,
                                                  ctypes.c_void_p]),
    "svsa_schedule_step": (ctypes.c_int, [ctypes.POINTER(Schedule), ctypes.c_int32, ctypes.POINTER(MaskParams),
                                          ctypes.POINTER(MaskParams), ctypes.POINTER(ctypes.c_int32)]),
    "svsa_anchor_offset": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.POINTER(ctypes.c_int32)]),
    "svsa_selftest_timeout": (ctypes.c_int, [ctypes.c_int32, ctypes.c_void_p]),
    "svsa_sync_status": (ctypes.c_int, [ctypes.c_void_p]),
    "svsa_last_error": (ctypes.c_char_p, []),
    "svsa_version": (ctypes.c_char_p, []),
    "svsa_launch_count": (ctypes.c_ulonglong, []),
}


def lib() -> ctypes.CDLL:
    """The loaded libsvsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_attention_hilbert_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def exported_symbols():
    return list(_SIGS)


def _check(status: int, fn: str) -> None:
    if status != 0:
        raise SvsaError(status, fn, lib().svsa_last_error().decode())


def _p(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def shape(B: int, heads: int, T: int, H: int, W: int, d: int) -> Shape:
    return Shape(B, heads, T, H, W, d)


def mask_params(select: int = SEL_THRESHOLD, tau: float = 0.9, keep_frac: float = 0.25,
                sub_block: int = 64, win_t: int = 2, win_rows: int = 1, n_anchors: int = 0,
                step: int = 0, seed: int = 0, routing: bool = False, scorer: int = SCORE_POOLED) -> MaskParams:
    return MaskParams(select, tau, keep_frac, sub_block, win_t, win_rows, n_anchors, step,
                      seed & 0xFFFFFFFFFFFFFFFF, int(routing), scorer)


def make_mask(kv_idx, kv_cnt, cap: int, bits=None, kbar=None, vbar=None, nvalid=None, cbar=None,
              check: bool = False, pairs=None) -> Mask:
    return Mask(_p(kv_idx), _p(kv_cnt), cap, _p(bits), _p(kbar), _p(vbar), _p(nvalid), _p(cbar), _p(pairs),
                int(check))


def svsa_anchor_offset(seed: int, step: int, nb: int, n_anchors: int) -> int:
    """The anchor rotation of step `step` for a run seeded `seed` (host-only)."""
    out = ctypes.c_int32(0)
    _check(lib().svsa_anchor_offset(seed & 0xFFFFFFFFFFFFFFFF, step, nb, n_anchors, ctypes.byref(out)),
           "svsa_anchor_offset")
    return int(out.value)


def version() -> str:
    return lib().svsa_version().decode()


def svsa_perm_workspace_bytes(s: Shape, order: int) -> int:
    return int(lib().svsa_perm_workspace_bytes(s, order))


def svsa_build_perm(s: Shape, order: int, perm, iperm, ws=None, ws_bytes: int = 0, stream=None) -> None:
    _check(lib().svsa_build_perm(s, order, _p(perm), _p(iperm), _p(ws), ws_bytes, _stream(stream)),
           "svsa_build_perm")


def svsa_build_perm_noalloc(s: Shape, order: int, perm, iperm, stream=None) -> None:
    """svsa_build_perm with the library's fixed scratch (no allocation; max side 128 for Hilbert)."""
    _check(lib().svsa_build_perm_noalloc(s, order, _p(perm), _p(iperm), _stream(stream)),
           "svsa_build_perm_noalloc")


def schedule(n_steps: int, dense_steps: int, start: float, end: float, refresh_every: int) -> Schedule:
    return Schedule(n_steps, dense_steps, start, end, refresh_every)


def svsa_schedule_step(sch: Schedule, step: int, base: MaskParams):
    """(mask params of `step`, True if the step builds its mask)."""
    out = MaskParams()
    rebuild = ctypes.c_int32(0)
    _check(lib().svsa_schedule_step(ctypes.byref(sch), step, ctypes.byref(base), ctypes.byref(out),
                                    ctypes.byref(rebuild)), "svsa_schedule_step")
    return out, bool(rebuild.value)


def svsa_cocluster_workspace_bytes(s: Shape) -> int:
    return int(lib().svsa_cocluster_workspace_bytes(s))


def svsa_build_perm_cocluster(q, k, s: Shape, rounds: int, perm_q, iperm_q, perm_k, iperm_k, ws, ws_bytes: int,
                              stream=None) -> None:
    _check(lib().svsa_build_perm_cocluster(_p(q), _p(k), s, rounds, _p(perm_q), _p(iperm_q), _p(perm_k),
                                           _p(iperm_k), _p(ws), ws_bytes, _stream(stream)),
           "svsa_build_perm_cocluster")


def svsa_reorder_heads(x, xp, perm, s: Shape, stream=None) -> None:
    _check(lib().svsa_reorder_heads(_p(x), _p(xp), _p(perm), s, _stream(stream)), "svsa_reorder_heads")


def svsa_reorder_values_heads(v, vp, perm, s: Shape, stream=None) -> None:
    _check(lib().svsa_reorder_values_heads(_p(v), _p(vp), _p(perm), s, _stream(stream)), "svsa_reorder_values_heads")


def svsa_inverse_reorder_heads(op, o, iperm, s: Shape, stream=None) -> None:
    _check(lib().svsa_inverse_reorder_heads(_p(op), _p(o), _p(iperm), s, _stream(stream)),
           "svsa_inverse_reorder_heads")


def svsa_reorder(x, xp, perm, s: Shape, stream=None) -> None:
    _check(lib().svsa_reorder(_p(x), _p(xp), _p(perm), s, _stream(stream)), "svsa_reorder")


def svsa_reorder_values(v, vp, perm, s: Shape, stream=None) -> None:
    _check(lib().svsa_reorder_values(_p(v), _p(vp), _p(perm), s, _stream(stream)), "svsa_reorder_values")


def svsa_pool(xp, out, s: Shape, size: int, stream=None) -> None:
    _check(lib().svsa_pool(_p(xp), _p(out), s, size, _stream(stream)), "svsa_pool")


def svsa_mask_workspace_bytes(s: Shape, p: MaskParams) -> int:
    return int(lib().svsa_mask_workspace_bytes(s, ctypes.byref(p)))


def svsa_build_mask(qp, kp, vp, perm, s: Shape, p: MaskParams, m: Mask, ws=None, ws_bytes: int = 0,
                    stream=None) -> None:
    _check(lib().svsa_build_mask(_p(qp), _p(kp), _p(vp), _p(perm), s, ctypes.byref(p), ctypes.byref(m),
                                 _p(ws), ws_bytes, _stream(stream)), "svsa_build_mask")


def svsa_attn_fwd(qp, kp, vp, m: Mask, compensate: bool, op, lse, s: Shape, stream=None) -> None:
    _check(lib().svsa_attn_fwd(_p(qp), _p(kp), _p(vp), ctypes.byref(m), int(compensate), _p(op), _p(lse),
                               s, _stream(stream)), "svsa_attn_fwd")


def svsa_attn_split_workspace_bytes(s: Shape, passes: int) -> int:
    return int(lib().svsa_attn_split_workspace_bytes(s, passes))


def svsa_attn_fwd_split(qp, kp, vp, m: Mask, compensate: bool, op, lse, s: Shape, passes: int, ws, ws_bytes: int,
                        stream=None) -> None:
    _check(lib().svsa_attn_fwd_split(_p(qp), _p(kp), _p(vp), ctypes.byref(m), int(compensate), _p(op), _p(lse), s,
                                     passes, _p(ws), ws_bytes, _stream(stream)), "svsa_attn_fwd_split")


def layer_config(order: int, mask: MaskParams, compensate: bool = False, attn_passes: int = 1,
                 paired: bool = False, groups: int = 1) -> LayerConfig:
    return LayerConfig(order, mask, int(compensate), attn_passes, int(paired), groups)


def svsa_layer_device_bytes(s: Shape, cfg: LayerConfig) -> int:
    return int(lib().svsa_layer_device_bytes(s, ctypes.byref(cfg)))


def svsa_layer_create(s: Shape, cfg: LayerConfig) -> int:
    """A host-buffer layer (an opaque handle; free it with svsa_layer_destroy)."""
    h = ctypes.c_void_p(0)
    _check(lib().svsa_layer_create(s, ctypes.byref(cfg), ctypes.byref(h)), "svsa_layer_create")
    return int(h.value)


def svsa_layer_forward_host(layer: int, q, k, v, o, step: int = 0, flags: int = 0, stream=None) -> None:
    """q, k, v, o: host bf16 [B, heads, N, d] (pinned for overlap)."""
    _check(lib().svsa_layer_forward_host(layer, _p(q), _p(k), _p(v), _p(o), step, flags, _stream(stream)),
           "svsa_layer_forward_host")


def svsa_layer_destroy(layer: int) -> None:
    _check(lib().svsa_layer_destroy(layer), "svsa_layer_destroy")


def svsa_attn_paired_workspace_bytes(s: Shape, passes: int) -> int:
    return int(lib().svsa_attn_paired_workspace_bytes(s, passes))


def svsa_attn_fwd_paired(qp, kp, vp, m: Mask, compensate: bool, op, lse, s: Shape, passes: int, ws, ws_bytes: int,
                         stream=None) -> None:
    _check(lib().svsa_attn_fwd_paired(_p(qp), _p(kp), _p(vp), ctypes.byref(m), int(compensate), _p(op), _p(lse), s,
                                      passes, _p(ws), ws_bytes, _stream(stream)), "svsa_attn_fwd_paired")


def svsa_attn_dense_fwd(qp, kp, vp, op, lse, s: Shape, stream=None) -> None:
    _check(lib().svsa_attn_dense_fwd(_p(qp), _p(kp), _p(vp), _p(op), _p(lse), s, _stream(stream)),
           "svsa_attn_dense_fwd")


def svsa_inverse_reorder(op, o, iperm, s: Shape, stream=None) -> None:
    _check(lib().svsa_inverse_reorder(_p(op), _p(o), _p(iperm), s, _stream(stream)), "svsa_inverse_reorder")


def svsa_launch_count() -> int:
    return int(lib().svsa_launch_count())


def svsa_sync_status(stream=None) -> None:
    _check(lib().svsa_sync_status(_stream(stream)), "svsa_sync_status")


from .pipeline import CapturedLayer, SparseVideoAttention, LayerBuffers  # noqa: E402,F401
