/*
 * svsa.h -- C ABI of the B200 block-sparse video attention library (libsvsa.so).
 *
 * The library computes training-free block-sparse self-attention for video
 * diffusion transformers in four steps, each an entry point below:
 *
 *   1. svsa_build_perm / svsa_reorder -- put the (T, H, W) latent tokens in
 *      raster or 3D Hilbert order ("DFSAttn: Dynamic Fine-grained Sparse
 *      Attention for Efficient Video Generation", trick 1: a Hilbert curve
 *      threads the tokens so that sequence neighbours are space-time
 *      neighbours and every block is coherent).
 *   2. svsa_build_mask -- choose, for every 64-token query block, the key
 *      blocks computed exactly (DFSAttn trick 2: block scores from block
 *      averages, optionally from 16-token sub-blocks summed per block; SVOO
 *      "Training-Free Sparse Attention for Fast Video Generation via Offline
 *      Layer-Wise Sparsity Profiling and Online Bidirectional Co-Clustering",
 *      technical summary 2.A: keep the blocks that cover a cumulative
 *      attention mass; "LVSA: Training-Free Sparse Attention for Long Video
 *      Diffusion", abstract: structured window pattern with rotating global
 *      anchors; "SVG-EAR: Parameter-Free Linear Compensation for Sparse Video
 *      Generation via Error-aware Routing", 2.B: error-aware routing).
 *   3. svsa_attn_fwd -- exact softmax attention over the kept block pairs only
 *      (SVG-EAR, problem statement: sparse attention computes a subset of the
 *      attention blocks), optionally with centroid compensation of the skipped
 *      blocks (SVG-EAR 2.A: skipped keys and values are replaced by their
 *      block centroid).
 *   4. svsa_inverse_reorder -- put the output back in raster order.
 *
 * svsa_layer_create / svsa_layer_forward_host run the four steps on host
 * buffers (a layer object that owns its device memory and streams the rows
 * through the entry points above).
 *
 * Conventions shared by every entry point
 *   - Tensors are row-major and contiguous.  Q, K, V and O in raster order are
 *     bf16 [B, heads, N, d] with N = T*H*W; the reordered ("p") tensors are
 *     bf16 [B, heads, Npad, d] with Npad = 64 * nb, nb = ceil(N / 64).  Rows
 *     N..Npad-1 of a reordered tensor are zero pads; they never count in a
 *     mean, a softmax or an output.
 *   - Every pointer is a device pointer owned by the caller, and must be
 *     16-byte aligned.  The library allocates no memory and keeps no state
 *     (the svsa_layer_* object excepted: it owns its arena, and its
 *     forward call takes host pointers).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns after enqueueing its kernels.
 *   - Arguments are validated before anything is launched.  A failed
 *     validation returns SVSA_ERR_INVALID_ARG (or SVSA_ERR_UNSUPPORTED /
 *     SVSA_ERR_WORKSPACE) and launches nothing; a launch failure returns
 *     SVSA_ERR_CUDA.  svsa_last_error() gives a message for the last failure
 *     on the calling thread.  No entry point throws or aborts.
 *   - Supported: d in {64, 128}; B*heads*Npad*d < 2^31; nb <= 16384;
 *     Hilbert order needs max(T, H, W) <= 1024.
 */
#ifndef SVSA_H_
#define SVSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVSA_OK = 0,
  SVSA_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or parameter */
  SVSA_ERR_UNSUPPORTED = 2,   /* valid request outside the supported range */
  SVSA_ERR_WORKSPACE = 3,     /* workspace smaller than the *_workspace_bytes query */
  SVSA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  SVSA_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up (svsa_sync_status) */
  SVSA_ERR_RANGE = 6,         /* an input left the range the fp16 paths hold: a value
                                 given to svsa_reorder_values, or a block / sub-block mean
                                 of the scores, beyond +-65504 or not finite; the result
                                 saturated (svsa_sync_status) */
  SVSA_ERR_MASK = 7           /* svsa_attn_fwd with mask.check set found a malformed list:
                                 kv_cnt outside [0, cap], an index outside [0, nb) or a
                                 row not strictly ascending (svsa_sync_status) */
} svsa_status;

typedef enum { SVSA_ORDER_RASTER = 0, SVSA_ORDER_HILBERT = 1 } svsa_order;

typedef enum {
  SVSA_SEL_THRESHOLD = 0,     /* cumulative score mass >= tau */
  SVSA_SEL_TOPK = 1,          /* k = ceil(keep_frac * nb) highest scores */
  SVSA_SEL_STRUCTURED = 2     /* temporal/spatial window OR rotating anchors */
} svsa_select;

/* What the THRESHOLD / TOPK rules rank. */
typedef enum {
  SVSA_SCORE_POOLED = 0,      /* pooled block scores P_IJ (per query block) */
  SVSA_SCORE_SICS = 1         /* block coherence from the sum of intra-block cosine
                                 similarities of the keys (per head; see svsa_build_mask) */
} svsa_scorer;

/* One attention layer: batch, heads, latent grid (frames T, rows H, columns W)
 * and head dimension d.  N = T*H*W tokens. */
typedef struct {
  int32_t B, heads, T, H, W, d;
} svsa_shape;

/* Mask rule.  Fields a rule does not use are ignored. */
typedef struct {
  int32_t select;         /* svsa_select */
  float tau;              /* THRESHOLD: mass to reach; >= 1 keeps every block */
  float keep_frac;        /* TOPK: k = ceil(keep_frac * nb) clamped to [1, nb] */
  int32_t sub_block;      /* THRESHOLD/TOPK: 64 = block means, 16 = sub-block
                             scores summed per block (DFSAttn trick 2) */
  int32_t win_t;          /* STRUCTURED: keep |t_I - t_J| <= win_t (frames) */
  int32_t win_rows;       /* STRUCTURED: or |h_I - h_J| <= win_rows * ceil(64 / W) */
  int32_t n_anchors;      /* STRUCTURED: anchor key-block columns kept for all rows */
  int32_t step;           /* STRUCTURED: denoising step index s >= 0; the anchors
                             rotate with it (see svsa_anchor_offset) */
  uint64_t seed;          /* STRUCTURED: seed of the run's anchor rotation */
  int32_t routing;        /* THRESHOLD only: 1 = keep, per row, as many blocks as the
                             threshold rule would, chosen by largest estimated
                             compensation error per token (SVG-EAR 2.B); needs vp,
                             mask.kbar, mask.vbar and mask.nvalid */
  int32_t scorer;         /* THRESHOLD / TOPK: svsa_scorer (0 = pooled scores) */
} svsa_mask_params;

/* Block mask, written by svsa_build_mask and read by svsa_attn_fwd.  All
 * buffers are caller-owned device memory. */
typedef struct {
  int32_t* kv_idx;        /* [B, heads, nb, cap] kept key blocks of each query
                             block, strictly ascending (required: the attention
                             checks only a row's last pair for the ragged block
                             nb - 1); entries past kv_cnt are unspecified */
  int32_t* kv_cnt;        /* [B, heads, nb] number of kept key blocks */
  int32_t cap;            /* row capacity: >= nb (>= k for TOPK) */
  uint32_t* bits;         /* nullable [B, heads, nb, ceil(nb/32)]: bit J%32 of word
                             J/32 set iff block J is kept */
  float* kbar;            /* nullable [B, heads, nb, d] fp32 key block means */
  float* vbar;            /* nullable [B, heads, nb, d] fp32 value block means */
  int32_t* nvalid;        /* nullable [nb] valid (non-pad) tokens per block */
  void* cbar;             /* nullable [B, heads, nb, 2*d] 16-bit scratch, required by
                             svsa_attn_fwd(compensate = 1), which first writes each
                             block's kbar (bf16, first d) and vbar (fp16, last d)
                             there; 16-byte aligned; not read by svsa_build_mask */
  int32_t* pairs;         /* nullable [B, heads, nb]: the query blocks of each head in
                             the order svsa_attn_fwd_paired takes them, two at a time
                             (partners that share kept blocks leave more of the work
                             to its 128-row pass).  When non-NULL, svsa_build_mask
                             fills it (a greedy pairing by kept-list overlap; needs
                             bits) and svsa_attn_fwd_paired reads it; it must be a
                             permutation of 0..nb-1 per head (a caller that writes
                             kv_idx itself passes NULL or its own table).  NULL: blocks
                             2p and 2p + 1 go together.  svsa_attn_fwd and
                             svsa_attn_fwd_split do not read it (beyond the check). */
  int32_t check;          /* svsa_attn_fwd only: nonzero = first validate every list
                             (kv_cnt in [0, cap], indices in [0, nb), strictly
                             ascending) and the pairing table when given (a
                             permutation per head) in kernels of their own and record
                             a malformed one for svsa_sync_status (SVSA_ERR_MASK).  The attention
                             still runs, and clamps counts and indices to the tensors,
                             so a bad list gives a wrong output but no stray access. */
} svsa_mask;

/* ---- step 1: token order ------------------------------------------------ */

/* Workspace bytes svsa_build_perm needs (0 for raster order). */
size_t svsa_perm_workspace_bytes(svsa_shape s, int32_t order);

/* Build the permutation of the latent grid.
 *   perm  [Npad] int32 out: position i -> raster token id (t*H + h)*W + w, or
 *         -1 for the pad positions N..Npad-1.
 *   iperm [N]    int32 out: raster token id -> position.
 * Raster order is the identity.  Hilbert order (DFSAttn trick 1) sorts the
 * cells by their index on the Hilbert curve of the enclosing 2^k cube,
 * k = ceil(log2(max(T, H, W))), computed with Skilling's transpose method
 * (axes t, h, w); the sort is a rank by bitmap and prefix count, so the result
 * is deterministic.  ws: svsa_perm_workspace_bytes(s, order) bytes of device
 * scratch (may be NULL when that is 0).  B, heads and d are ignored. */
svsa_status svsa_build_perm(svsa_shape s, int32_t order, int32_t* perm, int32_t* iperm,
                            void* ws, size_t ws_bytes, void* stream);

/* Permutation build for callers that cannot allocate device memory.
 * (An addition of this library: the method descriptions have no counterpart.)  Some
 * callers have no way to provide the scratch svsa_build_perm needs: code that
 * runs where cudaMalloc is not allowed or not reachable -- a plain-C host
 * that owns no allocator, or a component whose device memory is entirely
 * managed by a framework pool it cannot call into.  This variant computes
 * exactly what svsa_build_perm computes, but its scratch (the Hilbert
 * bitmap and prefix counts) is a fixed array inside the library, so it
 * allocates nothing and calls no allocating routine.
 *   - Limit: Hilbert order needs max(T, H, W) <= 128 (the array holds
 *     524,800 bytes; every GPU that loads the library keeps it until the
 *     process exits).  Larger grids return SVSA_ERR_UNSUPPORTED with a
 *     message; use svsa_build_perm with a workspace for them.  Raster order
 *     needs no scratch and has no limit.
 *   - Every call looks up the array's device address in the current
 *     context (a host-side query, nothing is cached across contexts); the
 *     first call on a device also loads the library's device code, so make
 *     that first call before any stream capture.
 *   - Every call shares the one array: two calls whose kernels overlap on
 *     the GPU (different streams, no ordering between them) race and may both
 *     produce wrong permutations.  Order them on one stream or with events.
 *     The array keeps the last call's contents; each call clears what must
 *     start at zero itself.
 * perm, iperm, order, shape and errors are as for svsa_build_perm. */
svsa_status svsa_build_perm_noalloc(svsa_shape s, int32_t order, int32_t* perm, int32_t* iperm, void* stream);

/* Gather the queries or the keys into the reordered layout:
 *   xp[b, h, i, :] = x[b, h, perm[i], :] for i < Npad (zeros where perm[i] = -1).
 * x: bf16 [B, heads, N, d]; xp: bf16 [B, heads, Npad, d]; perm from
 * svsa_build_perm.  Call once for Q and once for K. */
svsa_status svsa_reorder(const void* x, void* xp, const int32_t* perm, svsa_shape s, void* stream);

/* The same gather for the values, converting bf16 to fp16:
 *   vp[b, h, i, :] = fp16(v[b, h, perm[i], :]) (zeros where perm[i] = -1).
 * v: bf16 [B, heads, N, d]; vp: fp16 [B, heads, Npad, d].  The conversion is
 * exact for every bf16 value of magnitude in [2^-14, 65504] (smaller ones keep
 * fp16's 2^-24 absolute resolution, larger ones saturate to +-65504).  The
 * attention's P.V product runs in fp16 so that the softmax weights keep an
 * 11-bit significand. */
svsa_status svsa_reorder_values(const void* v, void* vp, const int32_t* perm, svsa_shape s, void* stream);

/* ---- step 2: block mask ------------------------------------------------- */

/* Block (or sub-block) means of a reordered tensor -- the pooling that
 * svsa_build_mask starts with, as a call of its own ("DFSAttn", trick 2: a
 * block is represented by its average; "SVG-EAR" 2.A: a centroid is the mean
 * of its tokens):
 *   out[b, h, g, :] = mean of the valid rows (position < N) of group g, the
 *   rows [g * size, (g + 1) * size); 0 for a group with no valid row.
 * xp: bf16 [B, heads, Npad, d] (from svsa_reorder); out: fp32
 * [B, heads, Npad / size, d]; size in {64, 16}.  The sums are fp32 in a fixed
 * order, so the result is deterministic. */
svsa_status svsa_pool(const void* xp, float* out, svsa_shape s, int32_t size, void* stream);

/* Workspace bytes svsa_build_mask needs for this shape and rule. */
size_t svsa_mask_workspace_bytes(svsa_shape s, const svsa_mask_params* p);

/* Build the block mask from reordered Q and K (bf16) and V (fp16, from
 * svsa_reorder_values; needed for routing and for mask.vbar).
 * THRESHOLD / TOPK: pooled block scores P_IJ = softmax_J(qbar_I . kbar_J /
 *   sqrt(d)) over all key blocks (means over valid tokens; with sub_block = 16
 *   the per-sub-block softmax probabilities are summed over the 16 sub-pairs
 *   of (I, J) and averaged over the non-empty query sub-blocks of I); each row
 *   is ordered by (score desc, block index asc) and keeps the shortest prefix
 *   whose fp64 cumulative sum reaches tau, or the first k.
 * STRUCTURED: keep (I, J) iff |t_I - t_J| <= win_t or |h_I - h_J| <=
 *   win_rows * ceil(64 / W) or J is an anchor column, where (t, h) is the
 *   coordinate of the block's first token (perm required).  The anchor
 *   columns of step p->step are (o + m * floor(nb / n_anchors)) mod nb,
 *   m < n_anchors, with o = svsa_anchor_offset(p->seed, p->step, ...): the
 *   anchors rotate with the step index ("LVSA", abstract: rotating global
 *   anchors remove the fixed-grid bias).
 * scorer = SVSA_SCORE_SICS ("SPADE: An Input-Adaptive Sparse Attention Engine
 *   for Fast Video Diffusion Models Inference", part 2: the sum of intra-block
 *   cosine similarities decides, per head and per step, which blocks attention
 *   focuses on; a block whose tokens agree is kept, one whose tokens disagree
 *   is skipped).  Reading: for key block J of a head, with n_J valid keys,
 *   SICS_J = sum_{i, j in J} cos(k_i, k_j) (a zero key has cosine 0 with
 *   everything), the coherence c_J = SICS_J / n_J^2 in [0, 1], and the score
 *   S_J = c_J / sum_J' c_J' is the same for every query block of the head;
 *   THRESHOLD / TOPK then keep blocks as above, so every query block of a
 *   head gets the same list.  No pooled scores are computed (qp unused);
 *   sub_block and routing must be 64 and 0.
 * routing = 1: with the threshold rule's count m_I as the budget, keep the
 *   m_I blocks with the largest r_IJ = e_IJ / Z_I * 64 / n_J, where e_IJ is the
 *   l2 norm of the change of the un-normalised output of the proxy query
 *   qbar_I when block J's keys/values are replaced by their means (SVG-EAR 2.B).
 * Outputs: m->kv_idx, m->kv_cnt, and m->bits / kbar / vbar / nvalid when those
 * are non-NULL (kbar, vbar, nvalid required for routing).  perm may be NULL
 * unless select = STRUCTURED.  vp may be NULL unless routing = 1.
 * THRESHOLD / TOPK / routing stage each mask row's keys in shared memory
 * (within the nb <= 16384 limit above). */
svsa_status svsa_build_mask(const void* qp, const void* kp, const void* vp, const int32_t* perm,
                            svsa_shape s, const svsa_mask_params* p, const svsa_mask* m,
                            void* ws, size_t ws_bytes, void* stream);

/* The rotation of the anchor columns at denoising step `step` of a run seeded
 * `seed`: with stride = max(floor(nb / n_anchors), 1),
 *   *offset = Philox4x32-10(counter = (step, 0, 0, 0),
 *                           key = (seed mod 2^32, floor(seed / 2^32)))[0] mod stride,
 * the first output word of the counter-based generator of J. K. Salmon et al.,
 * "Parallel random numbers: as easy as 1, 2, 3" (SC'11); 0 when n_anchors is
 * 0.  The same (seed, step) always gives the same anchors, and consecutive
 * steps give independent rotations ("LVSA", abstract).  Host-only, no device
 * work.  step >= 0, nb >= 1, n_anchors in [0, nb]. */
svsa_status svsa_anchor_offset(uint64_t seed, int32_t step, int32_t nb, int32_t n_anchors, int32_t* offset);

/* ---- step 3: attention -------------------------------------------------- */

/* Block-sparse attention over the reordered tensors (qp, kp bf16 from
 * svsa_reorder, vp fp16 from svsa_reorder_values):
 *   O_i = sum_{J kept for block(i)} sum_{j in J, j < N} softmax(q_i . k_j / sqrt(d)) v_j
 * computed with an online softmax on the tensor cores (Q.K^T in bf16, P.V in
 * fp16, fp32 statistics and accumulators, P rounded to fp16).  compensate = 1 adds, for every
 * skipped block J, n_J copies of (kbar_J, vbar_J) to the same softmax
 * (SVG-EAR 2.A), n_J = the valid tokens of block J.  That needs m->kbar and
 * m->vbar (fp32 means, as svsa_build_mask writes them), m->bits (the kept
 * set; it must agree with kv_idx / kv_cnt) and m->cbar (scratch, overwritten:
 * the means rounded to bf16 keys / fp16 values for the tensor cores).
 * op: bf16 [B, heads, Npad, d] (pad rows are written as zeros).
 * lse: nullable fp32 [B, heads, Npad]: natural-log sum-exp of each row's
 * scaled scores (0 for pad rows). */
svsa_status svsa_attn_fwd(const void* qp, const void* kp, const void* vp, const svsa_mask* m,
                          int32_t compensate, void* op, float* lse, svsa_shape s, void* stream);

/* svsa_attn_fwd in `passes` key-range passes, for layers whose keys and
 * values outgrow L2: pass p attends over the kept key blocks in
 * [p * R, (p + 1) * R), R = ceil(nb / passes), and yields an fp32 output
 * normalised within the pass with its log-sum-exp; the passes are merged as
 * O = sum_p exp(lse_p - lse) O_p, lse = log sum_p exp(lse_p) (the softmax over
 * the union of disjoint key sets), so the result is svsa_attn_fwd's up to
 * rounding.  Compensation terms go with the last pass.  kv_idx rows must be
 * ascending (as svsa_build_mask writes them).  With passes > 1, every pass's
 * work items (query blocks) are assigned to the kernel's persistent CTAs by
 * a schedule computed on the device from the kept counts: wave by wave, the
 * costliest item of a wave to the least loaded CTA; the result is the same
 * bit for bit as without it, only the load is balanced.  passes in [1, 8]
 * (1 = a plain svsa_attn_fwd call, no workspace needed); ws: device memory of
 * svsa_attn_split_workspace_bytes(s, passes) bytes. */
size_t svsa_attn_split_workspace_bytes(svsa_shape s, int32_t passes);
svsa_status svsa_attn_fwd_split(const void* qp, const void* kp, const void* vp, const svsa_mask* m,
                                int32_t compensate, void* op, float* lse, svsa_shape s, int32_t passes, void* ws,
                                size_t ws_bytes, void* stream);

/* svsa_attn_fwd as the paired-block split, same result up to rounding.  The
 * query blocks go in pairs (m->pairs entries 2p, 2p + 1 when given, else
 * blocks 2p, 2p + 1; an odd last block alone).  The key blocks that both
 * blocks of a pair keep are attended by 128 query rows at once (both blocks
 * share every key tile, so no tensor work is spent on a masked quarter); the
 * key blocks that only one of them keeps, and the compensation terms, are
 * attended by 64 query rows into an fp32 partial output with its
 * log-sum-exp, which the 128-row pass then merges into its rows by the same
 * rule as svsa_attn_fwd_split's passes.  Needs m->bits (the kept set; it
 * must agree with kv_idx / kv_cnt).  passes in [1, 8] as for
 * svsa_attn_fwd_split (each key-range pass is split this way); ws: device
 * memory of svsa_attn_paired_workspace_bytes(s, passes) bytes. */
size_t svsa_attn_paired_workspace_bytes(svsa_shape s, int32_t passes);
svsa_status svsa_attn_fwd_paired(const void* qp, const void* kp, const void* vp, const svsa_mask* m,
                                 int32_t compensate, void* op, float* lse, svsa_shape s, int32_t passes, void* ws,
                                 size_t ws_bytes, void* stream);

/* Dense attention over all N keys, same arithmetic and layouts as
 * svsa_attn_fwd; the denominator of the speedup the benchmark reports. */
svsa_status svsa_attn_dense_fwd(const void* qp, const void* kp, const void* vp, void* op,
                                float* lse, svsa_shape s, void* stream);

/* ---- step 4: back to raster order --------------------------------------- */

/* o[b, h, r, :] = op[b, h, iperm[r], :] for r < N.
 * op: bf16 [B, heads, Npad, d]; o: bf16 [B, heads, N, d]. */
svsa_status svsa_inverse_reorder(const void* op, void* o, const int32_t* iperm, svsa_shape s,
                                 void* stream);

/* ---- step 1, data-dependent alternative: co-clustering order ------------- */

/* Semantic token order by bidirectional query-key co-clustering ("Training-
 * Free Sparse Attention for Fast Video Generation via Offline Layer-Wise
 * Sparsity Profiling and Online Bidirectional Co-Clustering" (SVOO), 2.B:
 * alternately group the keys by affinity to the query centroids and the
 * queries by affinity to the updated key centroids; "SVG-EAR" 2.A: permute so
 * that a cluster is contiguous).  Reading: per (batch, head), C = nb
 * clusters; initial query centroids = means of the raster 64-token blocks;
 * affinity = q . k, decided exactly (bf16 tokens, float32 centroids, fp64
 * value; ties to the lower cluster index); a centroid is the float32 mean of
 * its tokens, an empty cluster takes the centroid it was matched against;
 * one round = key assignment, key centroids, query assignment, query
 * centroids; tokens sorted by (cluster, raster index).
 * q, k: raster bf16 [B, heads, N, d].  Writes the query order
 * perm_q [B, heads, Npad] (raster id or -1 for a pad) / iperm_q [B, heads, N]
 * and the key order perm_k / iperm_k (same shapes), for the *_heads gathers:
 * Q with perm_q, K and V with perm_k, O back with iperm_q.  rounds in [1, 64];
 * ws: svsa_cocluster_workspace_bytes(s) bytes of device memory. */
size_t svsa_cocluster_workspace_bytes(svsa_shape s);
svsa_status svsa_build_perm_cocluster(const void* q, const void* k, svsa_shape s, int32_t rounds,
                                      int32_t* perm_q, int32_t* iperm_q, int32_t* perm_k, int32_t* iperm_k,
                                      void* ws, size_t ws_bytes, void* stream);

/* svsa_reorder / svsa_reorder_values / svsa_inverse_reorder with one map per
 * (batch, head) row: perm [B, heads, Npad], iperm [B, heads, N]. */
svsa_status svsa_reorder_heads(const void* x, void* xp, const int32_t* perm, svsa_shape s, void* stream);
svsa_status svsa_reorder_values_heads(const void* v, void* vp, const int32_t* perm, svsa_shape s, void* stream);
svsa_status svsa_inverse_reorder_heads(const void* op, void* o, const int32_t* iperm, svsa_shape s,
                                       void* stream);

/* ---- step schedule -------------------------------------------------------- */

/* Timestep-adaptive sparsity with a cached mask ("DFSAttn: Dynamic Fine-grained
 * Sparse Attention for Efficient Video Generation", trick 3: look at nearly
 * everything while the latent is noise, skip more as the video clears, and
 * reuse a decided mask for the following steps; "SVOO" 2.B reuses its block
 * structure every N diffusion steps).  The pages give the shape, not the
 * numbers; this reading:
 *   steps [0, dense_steps) keep every block (tau = 1 or keep_frac = 1);
 *   from step dense_steps to n_steps - 1 the rule parameter (tau for
 *   THRESHOLD, keep_frac for TOPK) moves linearly from start to end:
 *   p = start + (end - start) * (step - dense_steps) / (n_steps - 1 - dense_steps)
 *   in double, rounded to float (p = start when that span is empty);
 *   a mask is built at step 0, at step dense_steps and every refresh_every
 *   steps after it; the steps in between reuse the last one. */
typedef struct {
  int32_t n_steps;        /* denoising steps of the run, >= 1 */
  int32_t dense_steps;    /* in [0, n_steps] */
  float start, end;       /* rule parameter at step dense_steps and at the last step, >= 0 */
  int32_t refresh_every;  /* >= 1 */
} svsa_schedule;

/* Mask parameters of `step` (in [0, n_steps)): *out = *base with tau
 * (THRESHOLD) or keep_frac (TOPK) replaced by the step's value; *rebuild = 1
 * when this step builds its mask, 0 when it reuses the last one.  Host-only,
 * no device work.  STRUCTURED has no density parameter: SVSA_ERR_UNSUPPORTED.
 * out may alias base. */
svsa_status svsa_schedule_step(const svsa_schedule* sch, int32_t step, const svsa_mask_params* base,
                               svsa_mask_params* out, int32_t* rebuild);

/* ---- the whole layer on host buffers ------------------------------------ */

/* A layer object that owns every device buffer of the four steps, for
 * callers whose q, k, v and output live in host memory.  Configuration: */
typedef struct {
  int32_t order;          /* svsa_order (RASTER or HILBERT) */
  svsa_mask_params mask;  /* the selection rule; mask.step is set by each call */
  int32_t compensate;     /* 1: centroid compensation of the skipped blocks */
  int32_t attn_passes;    /* key-range passes of the attention, [1, 8] */
  int32_t paired;         /* 1: the attention as svsa_attn_fwd_paired */
  int32_t groups;         /* row groups the host path streams, [1, B * heads] */
} svsa_layer_config;

typedef struct svsa_layer svsa_layer;

/* Allocate the layer's device memory on the current device (about
 * B * heads * Npad * d * 22 bytes plus the mask and workspaces) and build its
 * token order.  Synchronous.  *out is NULL on failure. */
svsa_status svsa_layer_create(svsa_shape s, const svsa_layer_config* cfg, svsa_layer** out);

/* Device bytes a layer of this shape and configuration holds (0 for an
 * invalid request). */
size_t svsa_layer_device_bytes(svsa_shape s, const svsa_layer_config* cfg);

/* One layer call on host buffers: q, k, v, o are bf16 [B, heads, N, d] in
 * raster order (host memory; pinned memory lets the copies overlap the
 * work).  The rows (batch, head) go in cfg->groups groups: each group's
 * inputs are copied in on one stream, each group's reorder, block mask,
 * attention and inverse reorder run on `stream` once its inputs have
 * arrived, and its output is copied out on a third stream, so the copies of
 * one group overlap the work of another.  Asynchronous with respect to the
 * host: o is complete when `stream` reaches the point of this call, and the
 * inputs must stay unchanged until then.  step: the denoising step (the
 * structured rule's anchor rotation).  flags: SVSA_LAYER_REUSE_MASK keeps the
 * mask of the previous call (built if there is none); SVSA_LAYER_INPUTS_READY
 * declares that q, k, v are not produced by work still pending on `stream`
 * (for instance not the o of a call not yet complete), so their copies may
 * start at once and overlap the previous call's work (the calls alternate
 * between two input staging sets).  Calls on one layer must be made from one
 * stream.  The result equals the device-side sequence of svsa_reorder /
 * svsa_reorder_values, svsa_build_mask, the attention entry point and
 * svsa_inverse_reorder on the whole layer. */
enum { SVSA_LAYER_REUSE_MASK = 1, SVSA_LAYER_INPUTS_READY = 2 };
svsa_status svsa_layer_forward_host(svsa_layer* layer, const void* q, const void* k, const void* v, void* o,
                                    int32_t step, int32_t flags, void* stream);

/* Free the layer (after the work queued on it has completed).  NULL is a no-op. */
svsa_status svsa_layer_destroy(svsa_layer* layer);

/* ---- status ------------------------------------------------------------- */

/* Synchronise `stream` and report device-side failures recorded by the
 * kernels since the last call (a bounded wait that gave up -> SVSA_ERR_TIMEOUT;
 * an asynchronous CUDA error -> SVSA_ERR_CUDA).  Clears the recorded flags. */
svsa_status svsa_sync_status(void* stream);

/* Self-test of the failure path: launches a one-thread kernel whose bounded
 * wait on a barrier that nothing arrives at gives up after wait_us
 * microseconds (in [1, 1e6]) and records the failure the way every bounded
 * wait of the library does; the next svsa_sync_status then reports
 * SVSA_ERR_TIMEOUT (and clears it).  Nothing faults, traps or hangs. */
svsa_status svsa_selftest_timeout(int32_t wait_us, void* stream);

/* Message for the last failure on the calling thread ("" if none). */
const char* svsa_last_error(void);

/* Library version string. */
const char* svsa_version(void);

/* Number of kernels this process has launched through the library (all
 * threads, all devices); a diagnostic for benchmarks and tests. */
unsigned long long svsa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SVSA_H_ */
