"""fp64 CPU oracle for block-sparse video attention — TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct definition of what the CUDA
path computes.  Only `tests/`, `__graft_entry__.smoke()` and the `cpu_baseline`
/ `--impl reference` legs of `bench.py` may import it; the library and its
Python binding never do, and it imports nothing from them (the only module the
two sides share is `workloads`, the seeded input generator).

Everything runs in float64 on the exact bf16 inputs (bf16 -> fp64 is exact).

Sources (page title, section):
  * "DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
    Generation" -- trick 1 (3D Hilbert reordering of the tokens so that
    blocks are space-time coherent), trick 2 (sub-block scores summed into
    block scores), trick 3 (reuse of the previous step's mask).
  * "SVG-EAR: Parameter-Free Linear Compensation for Sparse Video Generation
    via Error-aware Routing" -- technical summary 2.A (skipped blocks replaced
    by their centroid key/value), 2.B (error-aware routing with query
    centroids as proxies; greedy pick by error / block size), problem
    statement (sparse attention computes a subset of blocks).
  * "Training-Free Sparse Attention for Fast Video Generation via Offline
    Layer-Wise Sparsity Profiling and Online Bidirectional Co-Clustering"
    (SVOO) -- technical summary 2.A (density needed to cover a cumulative
    attention mass such as 95%).
  * "LVSA: Training-Free Sparse Attention for Long Video Diffusion" --
    abstract (structured window pattern with rotating global anchors; the
    rotation by step index is a Philox4x32-10 draw, Salmon et al., SC'11).
  * "SPADE: An Input-Adaptive Sparse Attention Engine for Fast Video
    Diffusion Models Inference", part 2 -- the SICS coherence scorer (sum of
    intra-block cosine similarities).
  * DFSAttn trick 3 and SVOO 2.B -- a step schedule: dense early steps, a
    sparser rule as the video clears, the mask rebuilt every few steps
    (`schedule.py`).
  * SVOO 2.B and SVG-EAR 2.A -- bidirectional query-key co-clustering and the
    semantic token order it gives (`cluster.py`).

Pins: every function here is checked in `tests/test_oracle_*.py` against
something other than itself (brute force, closed forms, invariants, library
routines); functions without such a pin say "parity unpinned" in their
docstring.  At the time of writing every function is pinned.
"""
from .order import (hilbert_key_3d, perm_raster, perm_hilbert, build_perm, reorder, inverse_reorder,
                    locality_stats)
from .mask import (pool, block_scores, subblock_scores, select_threshold, select_topk, topk_count,
                   select_rows, structured_mask, anchor_blocks, anchor_offset, philox4x32_10, route_ratios,
                   select_routing, mask_from_rows, sics_coherence, sics_scores)
from .attention import (masked_attention, compensated_attention, dense_attention,
                        online_block_attention, kept_flops)
from .schedule import step_param, rebuilds, mask_steps
from .cluster import cocluster, perm_from_clusters, initial_centroids

__all__ = [
    "hilbert_key_3d", "perm_raster", "perm_hilbert", "build_perm", "reorder", "inverse_reorder",
    "locality_stats", "pool", "block_scores", "subblock_scores", "select_threshold", "select_topk",
    "topk_count", "select_rows", "structured_mask", "anchor_blocks", "anchor_offset", "philox4x32_10",
    "route_ratios",
    "select_routing", "mask_from_rows", "masked_attention", "compensated_attention",
    "dense_attention", "online_block_attention", "kept_flops", "step_param", "rebuilds", "mask_steps",
    "cocluster", "perm_from_clusters", "initial_centroids", "sics_coherence", "sics_scores",
]
