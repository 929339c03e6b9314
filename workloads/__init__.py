"""Seeded synthetic workloads for block-sparse video attention.

This module only draws inputs: it holds none of the method's arithmetic (no
ordering, pooling, scoring, selection or attention).  Both the fp64 oracle
(`oracle/`) and the CUDA path consume the arrays it returns, so the two sides
always see the same bf16 bits.

Input recipe (stands in for DiT activations of Wan 2.1 / HunyuanVideo, whose
weights and prompts are not available here):

    X[b, eta, n, c] = 0.8 * sum_{f<8} cos(2*pi * omega_f . xhat_n + phi_f) + 0.5 * eps

with xhat_n = (t/(T-1), h/(H-1), w/(W-1)) the normalised latent coordinate of
raster token n = (t*H + h)*W + w, omega_f ~ U[0,3]^3 and phi_f ~ U[0, 2*pi)
drawn per (tensor, batch, head, channel, f), eps ~ N(0, 1) per element, and the
sum rounded to bf16 (round-to-nearest-even).  Every draw comes from a torch
generator seeded with (seed, tensor id); the field is evaluated in fp32.

The method's own random draw (the per-step rotation of the anchor blocks of
the structured rule) is not made here: the library and the oracle each
implement the counter-based generator it is defined by.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

# tensor ids used to derive independent streams
TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2

BLOCK = 64


@dataclass(frozen=True)
class Workload:
    """One attention layer of a video DiT, with its mask rule."""
    name: str
    B: int
    heads: int
    d: int
    T: int
    H: int
    W: int
    order: str = "hilbert"            # "raster" | "hilbert"
    select: str = "threshold"         # "threshold" | "topk" | "structured"
    tau: float = 0.9
    keep_frac: float = 0.25
    sub_block: int = 64               # 64 or 16 (sub-block scoring)
    win_t: int = 2                    # structured: temporal half-width (latent frames)
    win_rows: int = 1                 # structured: spatial half-width (block rows)
    n_anchors: int = 4
    routing: bool = False
    compensate: bool = False
    scorer: str = "pooled"            # "pooled" | "sics" (per-head block coherence)
    reuse_steps: int = 1              # mask reused over this many denoising steps
    sigma: float = 0.05               # Q/K perturbation between reused steps
    notes: str = ""

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def nb(self) -> int:
        return (self.N + BLOCK - 1) // BLOCK

    @property
    def Npad(self) -> int:
        return self.nb * BLOCK

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five layer shapes: a tiny correctness case, Wan 2.1 1.3B (12 heads),
# the same at a 6x temporal horizon with a structured mask, Wan 2.1 14B
# (40 heads) with compensation and error-aware routing, HunyuanVideo (24
# heads) at a 2x horizon with 16-token sub-block scoring and mask reuse.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 64, 4, 8, 8, order="hilbert", select="threshold", tau=0.9),
    "wan13b": Workload("wan13b", 1, 12, 128, 21, 30, 52, order="hilbert", select="topk", keep_frac=0.25),
    "wan13b_6x": Workload("wan13b_6x", 1, 12, 128, 126, 30, 52, order="raster", select="structured",
                          win_t=2, win_rows=1, n_anchors=4),
    "wan14b": Workload("wan14b", 1, 40, 128, 21, 30, 52, order="hilbert", select="threshold", tau=0.95,
                       routing=True, compensate=True),
    "hunyuan_2x": Workload("hunyuan_2x", 1, 24, 128, 62, 45, 80, order="hilbert", select="threshold",
                           tau=0.9, sub_block=16, reuse_steps=4, sigma=0.05),
}


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    # distinct, reproducible stream per (seed, stream id)
    g.manual_seed((seed * 1_000_003 + stream * 7919 + 12345) & 0x7FFFFFFFFFFFFFFF)
    return g


def smooth_field(B: int, heads: int, T: int, H: int, W: int, d: int, *, seed: int = 0,
                 tensor: int = 0, device="cpu", n_freq: int = 8, amp: float = 0.8,
                 noise: float = 0.5, chunk_tokens: int = 1 << 15) -> torch.Tensor:
    """bf16 [B, heads, T*H*W, d]: smooth random-Fourier field plus white noise."""
    device = torch.device(device)
    N = T * H * W
    g = _gen(seed, 100 + tensor, device)
    omega = torch.rand(B, heads, d, n_freq, 3, generator=g, device=device, dtype=torch.float32) * 3.0
    phi = torch.rand(B, heads, d, n_freq, generator=g, device=device, dtype=torch.float32) * (2 * math.pi)
    out = torch.empty(B, heads, N, d, dtype=torch.bfloat16, device=device)
    tt = torch.arange(T, device=device, dtype=torch.float32) / max(T - 1, 1)
    hh = torch.arange(H, device=device, dtype=torch.float32) / max(H - 1, 1)
    ww = torch.arange(W, device=device, dtype=torch.float32) / max(W - 1, 1)
    coords = torch.stack(torch.meshgrid(tt, hh, ww, indexing="ij"), dim=-1).reshape(N, 3)
    gn = _gen(seed, 200 + tensor, device)
    two_pi = 2 * math.pi
    for b in range(B):
        for eta in range(heads):
            om = omega[b, eta]                     # [d, F, 3]
            ph = phi[b, eta]                       # [d, F]
            for s in range(0, N, chunk_tokens):
                e = min(N, s + chunk_tokens)
                x = coords[s:e]                    # [n, 3]
                arg = torch.einsum("nk,cfk->ncf", x, om) * two_pi + ph  # [n, d, F]
                val = amp * torch.cos(arg).sum(-1)
                val += noise * torch.randn(e - s, d, generator=gn, device=device, dtype=torch.float32)
                out[b, eta, s:e] = val.to(torch.bfloat16)
    return out


def make_qkv(w: Workload, *, seed: int = 0, device="cpu"):
    """Q, K, V bf16 [B, heads, N, d] in raster token order."""
    return tuple(smooth_field(w.B, w.heads, w.T, w.H, w.W, w.d, seed=seed, tensor=t, device=device)
                 for t in (TENSOR_Q, TENSOR_K, TENSOR_V))


def perturb(x: torch.Tensor, *, sigma: float, seed: int, step: int, tensor: int) -> torch.Tensor:
    """bf16(x + sigma * eps): the drift of Q or K between two denoising steps."""
    g = _gen(seed, 1000 + 16 * step + tensor, x.device)
    eps = torch.randn(x.shape, generator=g, device=x.device, dtype=torch.float32)
    return (x.float() + sigma * eps).to(torch.bfloat16)


def qk_at_step(q0: torch.Tensor, k0: torch.Tensor, *, sigma: float, seed: int, step: int):
    """Q_s, K_s after `step` cumulative perturbations (V does not drift)."""
    q, k = q0, k0
    for s in range(1, step + 1):
        q = perturb(q, sigma=sigma, seed=seed, step=s, tensor=TENSOR_Q)
        k = perturb(k, sigma=sigma, seed=seed, step=s, tensor=TENSOR_K)
    return q, k


def random_mask_lists(nb: int, rows: int, *, density: float, seed: int):
    """Random kept-block sets (bool [rows, nb]) for attention-only tests."""
    rng = np.random.default_rng(seed)
    m = rng.random((rows, nb)) < density
    m[np.arange(rows), rng.integers(0, nb, rows)] = True   # at least one block per row
    return m
