"""Timestep-adaptive sparsity with a cached mask -- oracle (test infrastructure only).

Source (page title, section): "DFSAttn: Dynamic Fine-grained Sparse Attention
for Efficient Video Generation", trick 3 ("smart cache", adaptive time): the
first denoising steps look at (nearly) everything because the latent is still
noise, later steps skip more and more of the work as the video clears, and
the mask decided at one step is remembered and reused for the following ones
instead of being re-evaluated at once.  "SVOO", 2.B, also reuses its block
structure over a fixed number of diffusion steps (e.g. every 20).

The pages give the shape of the schedule, not its numbers; the plainest
reading, used here and by the library:
  * steps 0 .. dense_steps-1 keep every block (threshold tau = 1, top-k
    keep_frac = 1);
  * from step dense_steps to the last step n_steps-1 the rule's parameter
    (tau for the threshold rule, keep_frac for top-k) moves linearly from
    `start` to `end`: p(s) = start + (end - start) * u, with
    u = (s - dense_steps) / (n_steps - 1 - dense_steps) (u = 0 when that
    span is empty), with start and end taken as float32 values, evaluated in
    fp64 and rounded to float32 (the rule's parameter type);
  * a mask is built at step 0, at step dense_steps, and every refresh_every
    steps after it; every other step reuses the last mask built (with that
    step's parameter and inputs).
The structured rule has no density parameter and is not scheduled.
"""
from __future__ import annotations

import numpy as np


def step_param(n_steps: int, dense_steps: int, start: float, end: float, step: int) -> float:
    """The rule parameter of `step` (a float32 value, returned as a Python float)."""
    if step < dense_steps:
        return 1.0
    start, end = float(np.float32(start)), float(np.float32(end))
    span = n_steps - 1 - dense_steps
    u = (step - dense_steps) / span if span > 0 else 0.0
    return float(np.float32(start + (end - start) * u))


def rebuilds(n_steps: int, dense_steps: int, refresh_every: int) -> list:
    """Per step: True when that step builds a new mask."""
    out = []
    for s in range(n_steps):
        if s == 0 or s == dense_steps:
            out.append(True)
        elif s > dense_steps:
            out.append((s - dense_steps) % refresh_every == 0)
        else:
            out.append(False)
    return out


def mask_steps(n_steps: int, dense_steps: int, refresh_every: int) -> list:
    """Per step: the step whose mask it uses (the last rebuild at or before it)."""
    src, last = [], 0
    for s, r in enumerate(rebuilds(n_steps, dense_steps, refresh_every)):
        if r:
            last = s
        src.append(last)
    return src
