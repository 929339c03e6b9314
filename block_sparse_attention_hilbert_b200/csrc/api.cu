// C ABI of libsvsa: argument validation, workspace layout, kernel launches.
// Every entry point validates before launching anything, returns a status
// and never throws across the boundary.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "svsa.h"

namespace svsa {
// kernels (one translation unit each)
cudaError_t launch_build_perm(int T, int H, int W, int hilbert, int32_t* perm, int32_t* iperm,
                              void* ws, cudaStream_t st);
size_t perm_workspace_bytes(int T, int H, int W);
int hilbert_order_bits(int T, int H, int W);
int perm_noalloc_max_bits();
size_t perm_noalloc_scratch_bytes();
cudaError_t perm_noalloc_scratch(void** out);
cudaError_t launch_gather_rows(const void* src, void* dst, const int32_t* map, long long map_stride, long long BH,
                               long long rows_dst, long long rows_src, int d, cudaStream_t st);
cudaError_t launch_gather_rows_f16(const void* src, void* dst, const int32_t* map, long long map_stride,
                                   long long BH, long long rows_dst, long long rows_src, int d, cudaStream_t st);
size_t cocluster_workspace_bytes(long long BH, long long N, int nb, int d);
cudaError_t launch_cocluster(const void* q, const void* k, long long BH, long long N, int nb, int d, int rounds,
                             int32_t* perm_q, int32_t* iperm_q, int32_t* perm_k, int32_t* iperm_k, void* ws,
                             cudaStream_t st, int* launches);
cudaError_t cocluster_tc_error(unsigned int* code, cudaStream_t st);
cudaError_t launch_pool(const void* xp, float* out, void* split, void* split_bf, int32_t* nvalid, long long BH,
                        long long N, long long Npad, int d, int size, cudaStream_t st);
cudaError_t launch_pool_f16(const void* xp, float* out, int32_t* nvalid, long long BH, long long N,
                            long long Npad, int d, int size, cudaStream_t st);
cudaError_t launch_nvalid(int32_t* nvalid, long long N, int nb, cudaStream_t st);
cudaError_t launch_scores(const void* qsplit, const void* ksplit, float* S, float* L, long long BH, long long N,
                          int ng, int nb, int d, int size, cudaStream_t st);
cudaError_t launch_select(const float* S, const float* R, long long rows, int nb, int mode, float tau,
                          int k, int cap, int32_t* kv_idx, int32_t* kv_cnt, uint32_t* bits,
                          cudaStream_t st);
cudaError_t launch_structured(const int32_t* perm, long long rows, int nb, int H, int W, int win_t,
                              int R, int n_anchors, int anchor_offset, int cap, int32_t* kv_idx,
                              int32_t* kv_cnt, uint32_t* bits, cudaStream_t st);
int route_nsplit(int nb);
cudaError_t launch_route(const void* qsplit_bf, const void* kp, const void* vp, const float* L, const float* vbar,
                         float* R, float* Rm, float* Mp, float* Zp, int nsplit, long long BH, long long N, int nb,
                         int d, cudaStream_t st);
cudaError_t route_tc_error(unsigned int* code, cudaStream_t st);
cudaError_t launch_centroid16(const float* kbar, const float* vbar, void* cbar, long long rows, int d,
                              cudaStream_t st);
cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, const int32_t* kv_idx,
                           const int32_t* kv_cnt, int cap, const uint32_t* bits, const void* cbar, void* o,
                           float* lse, long long BH, long long N, int nb, int d, bool dense, cudaStream_t st,
                           float* o32 = nullptr, float lse_empty = 0.f, const int32_t* sched = nullptr,
                           long long nwaves = 0);
long long attn_tc_grid(long long items);
cudaError_t launch_sched(const int32_t* cnt_p, long long items, int cap, int P, int G, long long nwaves,
                         int32_t* sched, cudaStream_t st);
cudaError_t launch_attn_fa(const void* q, const void* k, const void* v, const int32_t* kv_idx,
                           const int32_t* kv_cnt, int cap, const uint32_t* bits, const void* cbar, void* o,
                           float* lse, long long BH, long long N, int nb, int d, bool dense, cudaStream_t st,
                           float* o32 = nullptr, float lse_empty = 0.f, const int32_t* pairs = nullptr,
                           int inter_only = 0, const float* m_in = nullptr, const float* lse_in = nullptr);
cudaError_t launch_exclusive(const int32_t* kv_idx, const int32_t* kv_cnt, int cap, const uint32_t* bits,
                             const int32_t* pairs, long long BH, int nb, int32_t* x_idx, int xcap, int32_t* x_cnt,
                             cudaStream_t st);
cudaError_t attn_fa_error(unsigned int* code, cudaStream_t st);
size_t pair_table_bytes(long long BH, int nb);
cudaError_t launch_pair(const uint32_t* bits, long long BH, int nb, int16_t* tab, int32_t* pairs,
                        cudaStream_t st);
cudaError_t launch_split_mask(const int32_t* kv_idx, const int32_t* kv_cnt, int cap, long long rows, int nb, int P,
                              int R, int32_t* idx_p, int32_t* cnt_p, cudaStream_t st);
cudaError_t launch_combine(const float* o_p, const float* lse_p, long long rows, int P, int d, void* out,
                           float* lse_out, cudaStream_t st);
cudaError_t attn_tc_error(unsigned int* code, cudaStream_t st);
cudaError_t launch_selftest_timeout(unsigned long long budget_ns, cudaStream_t st);
cudaError_t scores_tc_error(unsigned int* code, cudaStream_t st);
cudaError_t launch_sics(const void* kp, float* coh, float* S, long long BH, long long N, int nb, int d,
                        cudaStream_t st);
cudaError_t launch_broadcast(const int32_t* hidx, const int32_t* hcnt, int hcap, long long BH, int nb, int cap,
                             int32_t* kv_idx, int32_t* kv_cnt, uint32_t* bits, cudaStream_t st);
cudaError_t launch_check_mask(const int32_t* kv_idx, const int32_t* kv_cnt, long long rows, int cap, int nb,
                              cudaStream_t st);
cudaError_t launch_check_pairs(const int32_t* pairs, long long BH, int nb, cudaStream_t st);
cudaError_t sics_flags(unsigned int* v, cudaStream_t st);
cudaError_t reorder_flags(unsigned int* v, cudaStream_t st);
cudaError_t pool_flags(unsigned int* v, cudaStream_t st);
svsa_status record_error(svsa_status st, const char* msg);
}  // namespace svsa

using namespace svsa;

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_launches{0};

// Count `n` kernel launches once a launch helper reported success.
cudaError_t counted(cudaError_t e, int n) {
  if (e == cudaSuccess) g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed);
  return e;
}

svsa_status fail(svsa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

}  // namespace

// For the library's other host-side files: record a failure message.
svsa_status svsa::record_error(svsa_status st, const char* msg) { return fail(st, "%s", msg); }

namespace {

svsa_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SVSA_OK;
  return fail(SVSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxBlocks = 16384;

svsa_status check_shape(const svsa_shape& s, bool need_heads) {
  if (s.T < 1 || s.H < 1 || s.W < 1)
    return fail(SVSA_ERR_INVALID_ARG, "grid dims must be >= 1 (T=%d H=%d W=%d)", s.T, s.H, s.W);
  const long long N = (long long)s.T * s.H * s.W;
  if (N >= (1LL << 31)) return fail(SVSA_ERR_UNSUPPORTED, "N = T*H*W = %lld exceeds int32", N);
  if (need_heads) {
    if (s.B < 1 || s.heads < 1)
      return fail(SVSA_ERR_INVALID_ARG, "B and heads must be >= 1 (B=%d heads=%d)", s.B, s.heads);
    if (s.d != 64 && s.d != 128) return fail(SVSA_ERR_UNSUPPORTED, "head dim d=%d (supported: 64, 128)", s.d);
    const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
    if (g.BH * g.Npad * s.d >= (1LL << 31))
      return fail(SVSA_ERR_UNSUPPORTED, "B*heads*Npad*d = %lld exceeds int32", g.BH * g.Npad * s.d);
  }
  return SVSA_OK;
}

#define SVSA_TRY(expr)                   \
  do {                                   \
    svsa_status _s = (expr);             \
    if (_s != SVSA_OK) return _s;        \
  } while (0)

#define SVSA_PTR(p, name)                                                                      \
  do {                                                                                         \
    if ((p) == nullptr) return fail(SVSA_ERR_INVALID_ARG, "%s is NULL", name);                 \
    if (!aligned16(p)) return fail(SVSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);   \
  } while (0)

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace layout of svsa_build_mask.
struct MaskWs {
  size_t qsplit, ksplit, S, R, Rm, qbf, L, Mp, Zp, q64, k64, coh, hidx, hcnt, ptab, total;
};

MaskWs mask_ws_layout(const Dims& g, const svsa_mask_params& p, bool have_kbar) {
  MaskWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
  const size_t f = sizeof(float);
  // the query-block pairing's intersection table (used when mask.pairs is given)
  w.ptab = take(pair_table_bytes(g.BH, g.nb));
  if (p.select == SVSA_SEL_STRUCTURED) {
    w.qsplit = w.ksplit = w.S = w.R = w.Rm = w.qbf = w.L = w.Mp = w.Zp = w.q64 = w.k64 = SIZE_MAX;
    w.coh = w.hidx = w.hcnt = SIZE_MAX;
    w.total = off;
    return w;
  }
  if (p.scorer == SVSA_SCORE_SICS) {
    // per-head coherences, their normalised scores, and one selected list per head
    w.qsplit = w.ksplit = w.R = w.Rm = w.qbf = w.L = w.Mp = w.Zp = w.q64 = w.k64 = SIZE_MAX;
    w.coh = take((size_t)g.BH * g.nb * f);
    w.S = take((size_t)g.BH * g.nb * f);
    w.hidx = take((size_t)g.BH * g.nb * 4);
    w.hcnt = take((size_t)g.BH * 4);
    w.total = off;
    return w;
  }
  w.coh = w.hidx = w.hcnt = SIZE_MAX;
  const int sub = p.sub_block;
  const long long ng = g.Npad / sub;
  (void)have_kbar;
  // pooled Q and K as fp16 hi | lo pairs for the tensor-core scores
  w.qsplit = take((size_t)g.BH * ng * 2 * g.d * 2);
  w.ksplit = take((size_t)g.BH * ng * 2 * g.d * 2);
  w.S = take((size_t)g.BH * g.nb * g.nb * f);
  w.R = w.Rm = w.qbf = w.L = w.Mp = w.Zp = w.q64 = w.k64 = SIZE_MAX;
  if (p.routing) {
    const size_t nn = (size_t)g.BH * g.nb * g.nb * f;
    const size_t part = (size_t)g.BH * g.nb * route_nsplit(g.nb) * f;
    w.R = take(nn);
    w.Rm = take(nn);
    w.L = take(nn);                                        // centroid logits
    w.Mp = take(part);
    w.Zp = take(part);
    w.qbf = take((size_t)g.BH * g.nb * 2 * g.d * 2);       // query block means, bf16 hi | lo
    if (sub != kBlock) {                                   // block-level splits for the centroid logits
      w.q64 = take((size_t)g.BH * g.nb * 2 * g.d * 2);
      w.k64 = take((size_t)g.BH * g.nb * 2 * g.d * 2);
    }
  }
  w.total = off;
  return w;
}

svsa_status check_params(const svsa_mask_params* p, const Dims& g) {
  if (p == nullptr) return fail(SVSA_ERR_INVALID_ARG, "params is NULL");
  if (p->select < 0 || p->select > 2) return fail(SVSA_ERR_INVALID_ARG, "select=%d unknown", p->select);
  if (p->select != SVSA_SEL_STRUCTURED && p->sub_block != 64 && p->sub_block != 16)
    return fail(SVSA_ERR_UNSUPPORTED, "sub_block=%d (supported: 64, 16)", p->sub_block);
  if (p->select == SVSA_SEL_THRESHOLD && !(p->tau >= 0.f))
    return fail(SVSA_ERR_INVALID_ARG, "tau=%g must be >= 0", (double)p->tau);
  if (p->select == SVSA_SEL_TOPK && !(p->keep_frac >= 0.f))
    return fail(SVSA_ERR_INVALID_ARG, "keep_frac=%g must be >= 0", (double)p->keep_frac);
  if (p->routing && p->select != SVSA_SEL_THRESHOLD)
    return fail(SVSA_ERR_INVALID_ARG, "routing needs select = THRESHOLD (its budget)");
  if (p->scorer != SVSA_SCORE_POOLED && p->scorer != SVSA_SCORE_SICS)
    return fail(SVSA_ERR_INVALID_ARG, "scorer=%d unknown", p->scorer);
  if (p->scorer == SVSA_SCORE_SICS) {
    if (p->select == SVSA_SEL_STRUCTURED)
      return fail(SVSA_ERR_INVALID_ARG, "the SICS scorer ranks blocks for THRESHOLD / TOPK, not STRUCTURED");
    if (p->sub_block != 64 || p->routing)
      return fail(SVSA_ERR_UNSUPPORTED, "the SICS scorer works on 64-token blocks without routing");
  }
  if (p->select == SVSA_SEL_STRUCTURED) {
    if (p->win_t < 0 || p->win_rows < 0 || p->n_anchors < 0 || p->n_anchors > g.nb)
      return fail(SVSA_ERR_INVALID_ARG, "structured window/anchors out of range");
    if (p->step < 0) return fail(SVSA_ERR_INVALID_ARG, "step=%d must be >= 0", p->step);
  }
  if (g.nb > kMaxBlocks) return fail(SVSA_ERR_UNSUPPORTED, "nb=%d blocks exceeds %d", g.nb, kMaxBlocks);
  return SVSA_OK;
}

// Philox4x32-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC'11): ten rounds, each two
// 32x32 -> 64-bit products of counter words with the round multipliers, the
// high halves XORed with the other counter words and the key; the key is
// bumped by the two Weyl increments before every round after the first.
void philox4x32_10(const uint32_t in[4], uint32_t k0, uint32_t k1, uint32_t out[4]) {
  uint32_t c0 = in[0], c1 = in[1], c2 = in[2], c3 = in[3];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    c0 = n0;
    c1 = (uint32_t)p1;
    c2 = n2;
    c3 = (uint32_t)p0;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

// Rotation of the anchor columns at step `step` (>= 0): the first Philox word
// of counter (step, 0, 0, 0) under key (seed low, seed high), mod the stride.
int anchor_rotation(uint64_t seed, int32_t step, int nb, int n_anchors) {
  if (n_anchors <= 0 || nb <= 0) return 0;
  const uint32_t stride = (uint32_t)std::max(nb / n_anchors, 1);
  const uint32_t ctr[4] = {(uint32_t)step, 0u, 0u, 0u};
  uint32_t out[4];
  philox4x32_10(ctr, (uint32_t)seed, (uint32_t)(seed >> 32), out);
  return (int)(out[0] % stride);
}

int topk_count(float keep_frac, int nb) {
  double k = std::ceil((double)keep_frac * (double)nb);
  if (k < 1.0) k = 1.0;
  if (k > nb) k = nb;
  return (int)k;
}

}  // namespace

namespace {
// NVTX range around a public call: the calls appear by name in a timeline
// profiler; without one attached the push / pop cost nothing measurable.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// The row gathers of steps 2 and 4; per_head: the map holds one row per (batch, head).
svsa_status gather(const void* src, void* dst, const int32_t* map, svsa_shape s, bool forward, bool to_f16,
                   bool per_head, void* stream, const char* what) {
  NvtxRange nvtx_(what);
  g_last_error.clear();
  SVSA_TRY(check_shape(s, true));
  SVSA_PTR(src, "input");
  SVSA_PTR(dst, "output");
  SVSA_PTR(map, forward ? "perm" : "iperm");
  if (src == dst) return fail(SVSA_ERR_INVALID_ARG, "input and output must not alias");
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  const long long rows_dst = forward ? g.Npad : g.N, rows_src = forward ? g.N : g.Npad;
  const long long stride = per_head ? rows_dst : 0;
  cudaError_t e = to_f16 ? launch_gather_rows_f16(src, dst, map, stride, g.BH, rows_dst, rows_src, g.d,
                                                  (cudaStream_t)stream)
                         : launch_gather_rows(src, dst, map, stride, g.BH, rows_dst, rows_src, g.d,
                                              (cudaStream_t)stream);
  return cuda_status(counted(e, 1), what);
}
}  // namespace

extern "C" {

const char* svsa_last_error(void) { return g_last_error.c_str(); }

const char* svsa_version(void) { return "svsa 0.1.0 (sm_100a)"; }

unsigned long long svsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t svsa_perm_workspace_bytes(svsa_shape s, int32_t order) {
  if (order != SVSA_ORDER_HILBERT || s.T < 1 || s.H < 1 || s.W < 1) return 0;
  if (hilbert_order_bits(s.T, s.H, s.W) > 10) return 0;
  return perm_workspace_bytes(s.T, s.H, s.W);
}

svsa_status svsa_build_perm(svsa_shape s, int32_t order, int32_t* perm, int32_t* iperm, void* ws,
                            size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("svsa_build_perm");
  g_last_error.clear();
  SVSA_TRY(check_shape(s, false));
  if (order != SVSA_ORDER_RASTER && order != SVSA_ORDER_HILBERT)
    return fail(SVSA_ERR_INVALID_ARG, "order=%d unknown", order);
  SVSA_PTR(perm, "perm");
  SVSA_PTR(iperm, "iperm");
  if (order == SVSA_ORDER_HILBERT) {
    if (hilbert_order_bits(s.T, s.H, s.W) > 10)
      return fail(SVSA_ERR_UNSUPPORTED, "Hilbert order needs max(T,H,W) <= 1024");
    const size_t need = perm_workspace_bytes(s.T, s.H, s.W);
    SVSA_PTR(ws, "ws");
    if (ws_bytes < need) return fail(SVSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  }
  return cuda_status(counted(launch_build_perm(s.T, s.H, s.W, order == SVSA_ORDER_HILBERT, perm, iperm, ws,
                                               (cudaStream_t)stream),
                             order == SVSA_ORDER_HILBERT ? 5 : 1),
                     "build_perm launch");
}

svsa_status svsa_build_perm_noalloc(svsa_shape s, int32_t order, int32_t* perm, int32_t* iperm, void* stream) {
  NvtxRange nvtx_("svsa_build_perm_noalloc");
  g_last_error.clear();
  SVSA_TRY(check_shape(s, false));
  if (order != SVSA_ORDER_RASTER && order != SVSA_ORDER_HILBERT)
    return fail(SVSA_ERR_INVALID_ARG, "order=%d unknown", order);
  SVSA_PTR(perm, "perm");
  SVSA_PTR(iperm, "iperm");
  void* scratch = nullptr;
  if (order == SVSA_ORDER_HILBERT) {
    if (hilbert_order_bits(s.T, s.H, s.W) > perm_noalloc_max_bits())
      return fail(SVSA_ERR_UNSUPPORTED,
                  "no-allocation permutation build supports max(T,H,W) <= %d (got T=%d H=%d W=%d); "
                  "use svsa_build_perm with a workspace",
                  1 << perm_noalloc_max_bits(), s.T, s.H, s.W);
    SVSA_TRY(cuda_status(perm_noalloc_scratch(&scratch), "resolving the static scratch address"));
  }
  return cuda_status(counted(launch_build_perm(s.T, s.H, s.W, order == SVSA_ORDER_HILBERT, perm, iperm, scratch,
                                               (cudaStream_t)stream),
                             order == SVSA_ORDER_HILBERT ? 5 : 1),
                     "build_perm_noalloc launch");
}

svsa_status svsa_reorder(const void* x, void* xp, const int32_t* perm, svsa_shape s, void* stream) {
  return gather(x, xp, perm, s, true, false, false, stream, "reorder launch");
}

svsa_status svsa_reorder_values(const void* v, void* vp, const int32_t* perm, svsa_shape s, void* stream) {
  return gather(v, vp, perm, s, true, true, false, stream, "reorder_values launch");
}

svsa_status svsa_inverse_reorder(const void* op, void* o, const int32_t* iperm, svsa_shape s, void* stream) {
  return gather(op, o, iperm, s, false, false, false, stream, "inverse_reorder launch");
}

svsa_status svsa_reorder_heads(const void* x, void* xp, const int32_t* perm, svsa_shape s, void* stream) {
  return gather(x, xp, perm, s, true, false, true, stream, "reorder_heads launch");
}

svsa_status svsa_reorder_values_heads(const void* v, void* vp, const int32_t* perm, svsa_shape s, void* stream) {
  return gather(v, vp, perm, s, true, true, true, stream, "reorder_values_heads launch");
}

svsa_status svsa_inverse_reorder_heads(const void* op, void* o, const int32_t* iperm, svsa_shape s, void* stream) {
  return gather(op, o, iperm, s, false, false, true, stream, "inverse_reorder_heads launch");
}

size_t svsa_cocluster_workspace_bytes(svsa_shape s) {
  if (s.T < 1 || s.H < 1 || s.W < 1 || s.B < 1 || s.heads < 1 || (s.d != 64 && s.d != 128)) return 0;
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  return cocluster_workspace_bytes(g.BH, g.N, g.nb, g.d);
}

svsa_status svsa_build_perm_cocluster(const void* q, const void* k, svsa_shape s, int32_t rounds, int32_t* perm_q,
                                      int32_t* iperm_q, int32_t* perm_k, int32_t* iperm_k, void* ws, size_t ws_bytes,
                                      void* stream) {
  NvtxRange nvtx_("svsa_build_perm_cocluster");
  g_last_error.clear();
  SVSA_TRY(check_shape(s, true));
  SVSA_PTR(q, "q");
  SVSA_PTR(k, "k");
  SVSA_PTR(perm_q, "perm_q");
  SVSA_PTR(iperm_q, "iperm_q");
  SVSA_PTR(perm_k, "perm_k");
  SVSA_PTR(iperm_k, "iperm_k");
  SVSA_PTR(ws, "ws");
  if (rounds < 1 || rounds > 64) return fail(SVSA_ERR_INVALID_ARG, "rounds=%d outside [1, 64]", rounds);
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  if (g.nb > kMaxBlocks) return fail(SVSA_ERR_UNSUPPORTED, "nb=%d exceeds %d", g.nb, kMaxBlocks);
  const size_t need = cocluster_workspace_bytes(g.BH, g.N, g.nb, g.d);
  if (ws_bytes < need) return fail(SVSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  int launches = 0;
  cudaError_t e = launch_cocluster(q, k, g.BH, g.N, g.nb, g.d, rounds, perm_q, iperm_q, perm_k, iperm_k, ws,
                                   (cudaStream_t)stream, &launches);
  return cuda_status(counted(e, launches), "cocluster launch");
}

svsa_status svsa_pool(const void* xp, float* out, svsa_shape s, int32_t size, void* stream) {
  NvtxRange nvtx_("svsa_pool");
  g_last_error.clear();
  SVSA_TRY(check_shape(s, true));
  SVSA_PTR(xp, "xp");
  SVSA_PTR(out, "out");
  if (size != 64 && size != 16) return fail(SVSA_ERR_UNSUPPORTED, "size=%d (supported: 64, 16)", size);
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  return cuda_status(counted(launch_pool(xp, out, nullptr, nullptr, nullptr, g.BH, g.N, g.Npad, g.d, size,
                                         (cudaStream_t)stream), 1),
                     "pool launch");
}

size_t svsa_mask_workspace_bytes(svsa_shape s, const svsa_mask_params* p) {
  if (p == nullptr || s.T < 1 || s.H < 1 || s.W < 1 || s.B < 1 || s.heads < 1) return 0;
  if (p->select != SVSA_SEL_STRUCTURED && p->sub_block != 64 && p->sub_block != 16) return 0;
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  // sized for the worst case (caller's kbar/vbar absent)
  return mask_ws_layout(g, *p, false).total;
}

// The kept lists of svsa_build_mask (everything but the pairing).
static svsa_status build_mask_lists(const void* qp, const void* kp, const void* vp, const int32_t* perm,
                                    svsa_shape s, const svsa_mask_params* p, const svsa_mask* m, void* ws,
                                    size_t ws_bytes, void* stream) {
  SVSA_TRY(check_shape(s, true));
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  SVSA_TRY(check_params(p, g));
  if (m == nullptr) return fail(SVSA_ERR_INVALID_ARG, "mask is NULL");
  SVSA_PTR(m->kv_idx, "mask.kv_idx");
  SVSA_PTR(m->kv_cnt, "mask.kv_cnt");
  if (m->bits != nullptr && !aligned16(m->bits)) return fail(SVSA_ERR_INVALID_ARG, "mask.bits misaligned");
  if (m->pairs != nullptr) {
    if (!aligned16(m->pairs)) return fail(SVSA_ERR_INVALID_ARG, "mask.pairs misaligned");
    if (m->bits == nullptr) return fail(SVSA_ERR_INVALID_ARG, "mask.pairs needs mask.bits (the pairing reads it)");
  }
  if (m->kbar != nullptr && !aligned16(m->kbar)) return fail(SVSA_ERR_INVALID_ARG, "mask.kbar misaligned");
  if (m->vbar != nullptr && !aligned16(m->vbar)) return fail(SVSA_ERR_INVALID_ARG, "mask.vbar misaligned");
  if (m->nvalid != nullptr && !aligned16(m->nvalid)) return fail(SVSA_ERR_INVALID_ARG, "mask.nvalid misaligned");
  const int k = topk_count(p->keep_frac, g.nb);
  const int need_cap = p->select == SVSA_SEL_TOPK ? k : g.nb;
  if (m->cap < need_cap) return fail(SVSA_ERR_INVALID_ARG, "mask.cap=%d < %d", m->cap, need_cap);
  const bool structured = p->select == SVSA_SEL_STRUCTURED;
  if (!structured) {
    if (p->scorer != SVSA_SCORE_SICS) SVSA_PTR(qp, "qp");
    SVSA_PTR(kp, "kp");
  }
  if (structured) SVSA_PTR(perm, "perm");
  if (p->routing) {
    SVSA_PTR(vp, "vp");
    SVSA_PTR(m->kbar, "mask.kbar (routing)");
    SVSA_PTR(m->vbar, "mask.vbar (routing)");
    SVSA_PTR(m->nvalid, "mask.nvalid (routing)");
  }
  if (m->vbar != nullptr) SVSA_PTR(vp, "vp (mask.vbar requested)");
  if (m->kbar != nullptr) SVSA_PTR(kp, "kp (mask.kbar requested)");
  const MaskWs w = mask_ws_layout(g, *p, m->kbar != nullptr);
  // (the structured rule uses the workspace only for the pairing table)
  if (w.total > 0 && !(structured && m->pairs == nullptr)) {
    SVSA_PTR(ws, "ws");
    if (ws_bytes < w.total) return fail(SVSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, w.total);
  }
  cudaStream_t st = (cudaStream_t)stream;
  char* base = reinterpret_cast<char*>(ws);
  auto at = [&](size_t off) { return off == SIZE_MAX ? nullptr : reinterpret_cast<float*>(base + off); };
  const long long rows = g.BH * g.nb;
  int32_t* nvalid = m->nvalid;

  // block-level outputs the caller asked for (compensation / routing inputs)
  if (nvalid != nullptr) SVSA_TRY(cuda_status(counted(launch_nvalid(nvalid, g.N, g.nb, st), 1), "nvalid"));
  if (m->kbar != nullptr && (structured || p->sub_block != kBlock || p->scorer == SVSA_SCORE_SICS))
    SVSA_TRY(cuda_status(counted(launch_pool(kp, m->kbar, nullptr, nullptr, nullptr, g.BH, g.N, g.Npad, g.d, kBlock, st), 1),
                         "pool K"));
  if (m->vbar != nullptr)
    SVSA_TRY(cuda_status(counted(launch_pool_f16(vp, m->vbar, nullptr, g.BH, g.N, g.Npad, g.d, kBlock, st), 1),
                         "pool V"));

  if (structured) {
    const int R = p->win_rows * ((kBlock + g.W - 1) / g.W);
    const int offset = anchor_rotation(p->seed, p->step, g.nb, p->n_anchors);
    return cuda_status(counted(launch_structured(perm, rows, g.nb, g.H, g.W, p->win_t, R, p->n_anchors, offset,
                                                 m->cap, m->kv_idx, m->kv_cnt, m->bits, st), 1),
                       "structured mask");
  }

  if (p->scorer == SVSA_SCORE_SICS) {
    // per-head coherence scores -> one selected list per head -> every row of the head
    float* coh = at(w.coh);
    float* S1 = at(w.S);
    int32_t* hidx = reinterpret_cast<int32_t*>(base + w.hidx);
    int32_t* hcnt = reinterpret_cast<int32_t*>(base + w.hcnt);
    SVSA_TRY(cuda_status(counted(launch_sics(kp, coh, S1, g.BH, g.N, g.nb, g.d, st), 2), "SICS scores"));
    SVSA_TRY(cuda_status(counted(launch_select(S1, nullptr, g.BH, g.nb, p->select == SVSA_SEL_TOPK ? 1 : 0, p->tau,
                                               k, g.nb, hidx, hcnt, nullptr, st), 1),
                         "SICS select"));
    return cuda_status(counted(launch_broadcast(hidx, hcnt, g.nb, g.BH, g.nb, m->cap, m->kv_idx, m->kv_cnt, m->bits,
                                                st), 1),
                       "SICS lists");
  }

  const int sub = p->sub_block;
  const int ng = (int)(g.Npad / sub);
  void* qsplit = base + w.qsplit;
  void* ksplit = base + w.ksplit;
  float* S = at(w.S);
  // the routing proxies (bf16 split of the query block means) ride along when the rule works on blocks
  void* qbf = p->routing ? base + w.qbf : nullptr;
  float* L = p->routing ? at(w.L) : nullptr;
  SVSA_TRY(cuda_status(counted(launch_pool(qp, nullptr, qsplit, sub == kBlock ? qbf : nullptr, nullptr, g.BH, g.N,
                                           g.Npad, g.d, sub, st), 1),
                       "pool Q"));
  SVSA_TRY(cuda_status(counted(launch_pool(kp, sub == kBlock ? m->kbar : nullptr, ksplit, nullptr, nullptr, g.BH,
                                           g.N, g.Npad, g.d, sub, st), 1),
                       "pool K"));
  SVSA_TRY(cuda_status(counted(launch_scores(qsplit, ksplit, S, sub == kBlock ? L : nullptr, g.BH, g.N, ng, g.nb,
                                             g.d, sub, st), 1),
                       "scores"));
  const float* Rr = nullptr;
  int mode = p->select == SVSA_SEL_TOPK ? 1 : 0;
  if (p->routing) {
    if (sub != kBlock) {
      // block-level means for the proxies and the centroid logits
      SVSA_TRY(cuda_status(counted(launch_pool(qp, nullptr, base + w.q64, qbf, nullptr, g.BH, g.N, g.Npad, g.d,
                                               kBlock, st), 1),
                           "pool Q (blocks)"));
      SVSA_TRY(cuda_status(counted(launch_pool(kp, nullptr, base + w.k64, nullptr, nullptr, g.BH, g.N, g.Npad, g.d,
                                               kBlock, st), 1),
                           "pool K (blocks)"));
      SVSA_TRY(cuda_status(counted(launch_scores(base + w.q64, base + w.k64, nullptr, L, g.BH, g.N, g.nb, g.nb, g.d,
                                                 kBlock, st), 1),
                           "centroid logits"));
    }
    SVSA_TRY(cuda_status(counted(launch_route(qbf, kp, vp, L, m->vbar, at(w.R), at(w.Rm), at(w.Mp), at(w.Zp),
                                              route_nsplit(g.nb), g.BH, g.N, g.nb, g.d, st), 2),
                         "route"));
    Rr = at(w.R);
    mode = 3;
  }
  return cuda_status(counted(launch_select(S, Rr, rows, g.nb, mode, p->tau, k, m->cap, m->kv_idx,
                                           m->kv_cnt, m->bits, st), 1), "select");
}

svsa_status svsa_build_mask(const void* qp, const void* kp, const void* vp, const int32_t* perm,
                            svsa_shape s, const svsa_mask_params* p, const svsa_mask* m, void* ws,
                            size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("svsa_build_mask");
  g_last_error.clear();
  SVSA_TRY(build_mask_lists(qp, kp, vp, perm, s, p, m, ws, ws_bytes, stream));
  if (m->pairs == nullptr) return SVSA_OK;
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  int16_t* tab = reinterpret_cast<int16_t*>(reinterpret_cast<char*>(ws) + mask_ws_layout(g, *p, false).ptab);
  return cuda_status(counted(launch_pair(m->bits, g.BH, g.nb, tab, m->pairs, (cudaStream_t)stream), 2),
                     "query-block pairing");
}

svsa_status svsa_attn_fwd(const void* qp, const void* kp, const void* vp, const svsa_mask* m,
                          int32_t compensate, void* op, float* lse, svsa_shape s, void* stream) {
  NvtxRange nvtx_("svsa_attn_fwd");
  g_last_error.clear();
  SVSA_TRY(check_shape(s, true));
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  SVSA_PTR(qp, "qp");
  SVSA_PTR(kp, "kp");
  SVSA_PTR(vp, "vp");
  SVSA_PTR(op, "op");
  if (m == nullptr) return fail(SVSA_ERR_INVALID_ARG, "mask is NULL");
  SVSA_PTR(m->kv_idx, "mask.kv_idx");
  SVSA_PTR(m->kv_cnt, "mask.kv_cnt");
  if (m->cap < 1) return fail(SVSA_ERR_INVALID_ARG, "mask.cap=%d", m->cap);
  if (m->pairs != nullptr && !aligned16(m->pairs)) return fail(SVSA_ERR_INVALID_ARG, "mask.pairs misaligned");
  if (lse != nullptr && !aligned16(lse)) return fail(SVSA_ERR_INVALID_ARG, "lse misaligned");
  if (g.nb > kMaxBlocks) return fail(SVSA_ERR_UNSUPPORTED, "nb=%d exceeds %d", g.nb, kMaxBlocks);
  if (compensate) {
    SVSA_PTR(m->kbar, "mask.kbar (compensation)");
    SVSA_PTR(m->vbar, "mask.vbar (compensation)");
    SVSA_PTR(m->bits, "mask.bits (compensation)");
    SVSA_PTR(m->cbar, "mask.cbar (compensation)");
  }
  if (op == qp || op == kp || op == vp) return fail(SVSA_ERR_INVALID_ARG, "op must not alias an input");
  if (m->check) {
    SVSA_TRY(cuda_status(counted(launch_check_mask(m->kv_idx, m->kv_cnt, g.BH * g.nb, m->cap, g.nb,
                                                   (cudaStream_t)stream), 1),
                         "mask check"));
    if (m->pairs != nullptr)
      SVSA_TRY(cuda_status(counted(launch_check_pairs(m->pairs, g.BH, g.nb, (cudaStream_t)stream), 1),
                           "pairing check"));
  }
  if (compensate)
    SVSA_TRY(cuda_status(counted(launch_centroid16(m->kbar, m->vbar, m->cbar, g.BH * g.nb, g.d,
                                                   (cudaStream_t)stream), 1),
                         "centroid copies"));
  return cuda_status(counted(launch_attn_tc(qp, kp, vp, m->kv_idx, m->kv_cnt, m->cap, compensate ? m->bits : nullptr,
                                            compensate ? m->cbar : nullptr, op, lse, g.BH, g.N, g.nb, g.d, false,
                                            (cudaStream_t)stream), 1),
                     "attn_fwd launch");
}

namespace {
struct SplitWs {
  size_t idx, cnt, o, lse, sched, xidx, xcnt, part, plse, total;
};
constexpr int kSchedMaxCtas = 256;   // the item schedule serves grids of up to this many CTAs
// Workspace of svsa_attn_fwd_split / svsa_attn_fwd_paired: the P range lists,
// per-pass outputs and the item schedule of every pass (P > 1, split), then
// (paired) the exclusive lists and the fp32 partial of the paired-block split.
SplitWs split_layout(const Dims& g, int P, bool paired) {
  SplitWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~(size_t)255; return o; };
  const long long rows = g.BH * g.nb;
  const int R = (g.nb + P - 1) / P;
  w.idx = w.cnt = w.o = w.lse = w.sched = w.xidx = w.xcnt = w.part = w.plse = SIZE_MAX;
  if (P > 1) {
    w.idx = take((size_t)P * rows * R * 4);
    w.cnt = take((size_t)P * rows * 4);
    w.o = take((size_t)P * g.BH * g.Npad * g.d * 4);
    w.lse = take((size_t)P * g.BH * g.Npad * 4);
  }
  if (!paired && P > 1) w.sched = take((size_t)P * (rows + kSchedMaxCtas) * 4);   // [P][waves][grid]
  if (paired) {
    w.xidx = take((size_t)rows * std::min(R, g.nb) * 4);
    w.xcnt = take((size_t)rows * 4);
    w.part = take((size_t)g.BH * g.Npad * g.d * 4);
    w.plse = take((size_t)g.BH * g.Npad * 4);
  }
  w.total = off;
  return w;
}
}  // namespace

size_t svsa_attn_split_workspace_bytes(svsa_shape s, int32_t passes) {
  if (passes < 1 || passes > 8 || s.T < 1 || s.H < 1 || s.W < 1 || s.B < 1 || s.heads < 1) return 0;
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  return split_layout(g, passes, false).total;
}

size_t svsa_attn_paired_workspace_bytes(svsa_shape s, int32_t passes) {
  if (passes < 1 || passes > 8 || s.T < 1 || s.H < 1 || s.W < 1 || s.B < 1 || s.heads < 1) return 0;
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  return split_layout(g, passes, true).total;
}

namespace {
svsa_status attn_split(const void* qp, const void* kp, const void* vp, const svsa_mask* m, int32_t compensate,
                       void* op, float* lse, svsa_shape s, int32_t passes, void* ws, size_t ws_bytes, void* stream,
                       bool hybrid) {
  g_last_error.clear();
  if (passes < 1 || passes > 8) return fail(SVSA_ERR_INVALID_ARG, "passes=%d outside [1, 8]", passes);
  SVSA_TRY(check_shape(s, true));
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  SVSA_PTR(qp, "qp");
  SVSA_PTR(kp, "kp");
  SVSA_PTR(vp, "vp");
  SVSA_PTR(op, "op");
  SVSA_PTR(ws, "ws");
  if (m == nullptr) return fail(SVSA_ERR_INVALID_ARG, "mask is NULL");
  SVSA_PTR(m->kv_idx, "mask.kv_idx");
  SVSA_PTR(m->kv_cnt, "mask.kv_cnt");
  if (m->cap < 1) return fail(SVSA_ERR_INVALID_ARG, "mask.cap=%d", m->cap);
  if (m->pairs != nullptr && !aligned16(m->pairs)) return fail(SVSA_ERR_INVALID_ARG, "mask.pairs misaligned");
  if (lse != nullptr && !aligned16(lse)) return fail(SVSA_ERR_INVALID_ARG, "lse misaligned");
  if (g.nb > kMaxBlocks) return fail(SVSA_ERR_UNSUPPORTED, "nb=%d exceeds %d", g.nb, kMaxBlocks);
  if (compensate) {
    SVSA_PTR(m->kbar, "mask.kbar (compensation)");
    SVSA_PTR(m->vbar, "mask.vbar (compensation)");
    SVSA_PTR(m->bits, "mask.bits (compensation)");
    SVSA_PTR(m->cbar, "mask.cbar (compensation)");
  }
  if (hybrid) SVSA_PTR(m->bits, "mask.bits (paired-block split)");
  if (op == qp || op == kp || op == vp) return fail(SVSA_ERR_INVALID_ARG, "op must not alias an input");
  const SplitWs w = split_layout(g, passes, hybrid);
  if (ws_bytes < w.total) return fail(SVSA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, w.total);
  cudaStream_t st = (cudaStream_t)stream;
  char* base = reinterpret_cast<char*>(ws);
  auto at = [&](size_t off) { return off == SIZE_MAX ? nullptr : base + off; };
  int32_t* idx_p = reinterpret_cast<int32_t*>(at(w.idx));
  int32_t* cnt_p = reinterpret_cast<int32_t*>(at(w.cnt));
  float* o_p = reinterpret_cast<float*>(at(w.o));
  float* lse_p = reinterpret_cast<float*>(at(w.lse));
  int32_t* xidx = reinterpret_cast<int32_t*>(at(w.xidx));
  int32_t* xcnt = reinterpret_cast<int32_t*>(at(w.xcnt));
  float* part = reinterpret_cast<float*>(at(w.part));
  float* plse = reinterpret_cast<float*>(at(w.plse));
  int32_t* sched = reinterpret_cast<int32_t*>(at(w.sched));
  const long long rows = g.BH * g.nb;
  const int R = (g.nb + passes - 1) / passes;
  if (m->check) {
    SVSA_TRY(cuda_status(counted(launch_check_mask(m->kv_idx, m->kv_cnt, rows, m->cap, g.nb, st), 1), "mask check"));
    if (m->pairs != nullptr)
      SVSA_TRY(cuda_status(counted(launch_check_pairs(m->pairs, g.BH, g.nb, st), 1), "pairing check"));
  }
  if (compensate)
    SVSA_TRY(cuda_status(counted(launch_centroid16(m->kbar, m->vbar, m->cbar, g.BH * g.nb, g.d, st), 1),
                         "centroid copies"));
  if (passes > 1)
    SVSA_TRY(cuda_status(counted(launch_split_mask(m->kv_idx, m->kv_cnt, m->cap, rows, g.nb, passes, R, idx_p, cnt_p,
                                                   st), 1),
                         "split mask"));
  // every pass's items balanced over the attention's persistent CTAs
  const long long grid = attn_tc_grid(rows);
  const long long nwaves = (rows + grid - 1) / grid;
  const bool use_sched = sched != nullptr && grid <= kSchedMaxCtas;
  if (use_sched)
    SVSA_TRY(cuda_status(counted(launch_sched(passes > 1 ? cnt_p : m->kv_cnt, rows, passes > 1 ? R : m->cap, passes,
                                              (int)grid, nwaves, sched, st), 1),
                         "item schedule"));
  const long long rows_o = g.BH * g.Npad;
  for (int p = 0; p < passes; ++p) {
    // this pass's lists; the centroid tiles of the skipped blocks go with the last pass
    const int32_t* L_idx = passes > 1 ? idx_p + (long long)p * rows * R : m->kv_idx;
    const int32_t* L_cnt = passes > 1 ? cnt_p + (long long)p * rows : m->kv_cnt;
    const int L_cap = passes > 1 ? R : m->cap;
    const bool comp = compensate && p + 1 == passes;
    float* out32 = passes > 1 ? o_p + (long long)p * rows_o * g.d : nullptr;
    float* out_lse = passes > 1 ? lse_p + (long long)p * rows_o : lse;
    if (!hybrid) {
      SVSA_TRY(cuda_status(counted(launch_attn_tc(qp, kp, vp, L_idx, L_cnt, L_cap, comp ? m->bits : nullptr,
                                                   comp ? m->cbar : nullptr, passes > 1 ? nullptr : op, out_lse,
                                                   g.BH, g.N, g.nb, g.d, false, st, out32,
                                                   passes > 1 ? -INFINITY : 0.f,
                                                   use_sched ? sched + (long long)p * nwaves * grid : nullptr,
                                                   nwaves), 1),
                           "attn_fwd pass launch"));
      continue;
    }
    // The paired-block split: every pair of query blocks (the pairing table,
    // else blocks 2p, 2p + 1) shares the key blocks both keep -- the 128-row
    // kernel takes those with no masked quarter -- and each block keeps the
    // ones its partner does not -- the transposed 64-query kernel takes those,
    // with the centroid tiles, into an fp32 partial that the 128-row kernel
    // then merges (log-sum-exp) into its output rows.
    const int xcap = std::min(L_cap, g.nb);
    SVSA_TRY(cuda_status(counted(launch_exclusive(L_idx, L_cnt, L_cap, m->bits, m->pairs, g.BH, g.nb, xidx, xcap,
                                                  xcnt, st), 1),
                         "exclusive lists"));
    SVSA_TRY(cuda_status(counted(launch_attn_tc(qp, kp, vp, xidx, xcnt, xcap, comp ? m->bits : nullptr,
                                                 comp ? m->cbar : nullptr, nullptr, plse, g.BH, g.N, g.nb, g.d, false,
                                                 st, part, -INFINITY), 1),
                         "attn_fwd exclusive launch"));
    SVSA_TRY(cuda_status(counted(launch_attn_fa(qp, kp, vp, L_idx, L_cnt, L_cap, nullptr, nullptr,
                                                 passes > 1 ? nullptr : op, out_lse, g.BH, g.N, g.nb, g.d, false, st,
                                                 out32, passes > 1 ? -INFINITY : 0.f, m->pairs, 1, part, plse), 1),
                         "attn_fwd shared launch"));
  }
  if (passes == 1) return SVSA_OK;
  return cuda_status(counted(launch_combine(o_p, lse_p, g.BH * g.Npad, passes, g.d, op, lse, st), 1),
                     "combine launch");
}
}  // namespace

svsa_status svsa_attn_fwd_split(const void* qp, const void* kp, const void* vp, const svsa_mask* m,
                                int32_t compensate, void* op, float* lse, svsa_shape s, int32_t passes, void* ws,
                                size_t ws_bytes, void* stream) {
  // one pass: the plain call (measured, the item schedule does not pay for itself there)
  if (passes == 1) return svsa_attn_fwd(qp, kp, vp, m, compensate, op, lse, s, stream);
  NvtxRange nvtx_("svsa_attn_fwd_split");
  return attn_split(qp, kp, vp, m, compensate, op, lse, s, passes, ws, ws_bytes, stream, false);
}

svsa_status svsa_attn_fwd_paired(const void* qp, const void* kp, const void* vp, const svsa_mask* m,
                                 int32_t compensate, void* op, float* lse, svsa_shape s, int32_t passes, void* ws,
                                 size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("svsa_attn_fwd_paired");
  return attn_split(qp, kp, vp, m, compensate, op, lse, s, passes, ws, ws_bytes, stream, true);
}

svsa_status svsa_attn_dense_fwd(const void* qp, const void* kp, const void* vp, void* op, float* lse,
                                svsa_shape s, void* stream) {
  NvtxRange nvtx_("svsa_attn_dense_fwd");
  g_last_error.clear();
  SVSA_TRY(check_shape(s, true));
  const Dims g = make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  SVSA_PTR(qp, "qp");
  SVSA_PTR(kp, "kp");
  SVSA_PTR(vp, "vp");
  SVSA_PTR(op, "op");
  if (lse != nullptr && !aligned16(lse)) return fail(SVSA_ERR_INVALID_ARG, "lse misaligned");
  if (op == qp || op == kp || op == vp) return fail(SVSA_ERR_INVALID_ARG, "op must not alias an input");
  return cuda_status(counted(launch_attn_fa(qp, kp, vp, nullptr, nullptr, 1, nullptr, nullptr, op, lse, g.BH, g.N,
                                            g.nb, g.d, true, (cudaStream_t)stream), 1),
                     "attn_dense_fwd launch");
}

svsa_status svsa_schedule_step(const svsa_schedule* sch, int32_t step, const svsa_mask_params* base,
                               svsa_mask_params* out, int32_t* rebuild) {
  g_last_error.clear();
  if (sch == nullptr || base == nullptr || out == nullptr || rebuild == nullptr)
    return fail(SVSA_ERR_INVALID_ARG, "schedule, base, out and rebuild must not be NULL");
  if (sch->n_steps < 1 || sch->dense_steps < 0 || sch->dense_steps > sch->n_steps || sch->refresh_every < 1)
    return fail(SVSA_ERR_INVALID_ARG, "schedule n_steps=%d dense_steps=%d refresh_every=%d out of range",
                sch->n_steps, sch->dense_steps, sch->refresh_every);
  if (!(sch->start >= 0.f) || !(sch->end >= 0.f) || !std::isfinite(sch->start) || !std::isfinite(sch->end))
    return fail(SVSA_ERR_INVALID_ARG, "schedule start/end must be finite and >= 0");
  if (step < 0 || step >= sch->n_steps)
    return fail(SVSA_ERR_INVALID_ARG, "step=%d outside [0, %d)", step, sch->n_steps);
  if (base->select != SVSA_SEL_THRESHOLD && base->select != SVSA_SEL_TOPK)
    return fail(SVSA_ERR_UNSUPPORTED, "only THRESHOLD and TOPK rules have a density to schedule");
  float p = 1.0f;
  if (step >= sch->dense_steps) {
    const int span = sch->n_steps - 1 - sch->dense_steps;
    const double u = span > 0 ? (double)(step - sch->dense_steps) / (double)span : 0.0;
    p = (float)((double)sch->start + ((double)sch->end - (double)sch->start) * u);
  }
  const int32_t r = (step == 0 || step == sch->dense_steps ||
                     (step > sch->dense_steps && (step - sch->dense_steps) % sch->refresh_every == 0))
                        ? 1 : 0;
  svsa_mask_params o = *base;
  if (o.select == SVSA_SEL_THRESHOLD) o.tau = p;
  else o.keep_frac = p;
  *out = o;
  *rebuild = r;
  return SVSA_OK;
}

svsa_status svsa_anchor_offset(uint64_t seed, int32_t step, int32_t nb, int32_t n_anchors, int32_t* offset) {
  g_last_error.clear();
  if (offset == nullptr) return fail(SVSA_ERR_INVALID_ARG, "offset is NULL");
  if (step < 0) return fail(SVSA_ERR_INVALID_ARG, "step=%d must be >= 0", step);
  if (nb < 1 || n_anchors < 0 || n_anchors > nb)
    return fail(SVSA_ERR_INVALID_ARG, "nb=%d, n_anchors=%d: need nb >= 1 and n_anchors in [0, nb]", nb, n_anchors);
  *offset = anchor_rotation(seed, step, nb, n_anchors);
  return SVSA_OK;
}

svsa_status svsa_selftest_timeout(int32_t wait_us, void* stream) {
  NvtxRange nvtx_("svsa_selftest_timeout");
  g_last_error.clear();
  if (wait_us < 1 || wait_us > 1000000) return fail(SVSA_ERR_INVALID_ARG, "wait_us=%d outside [1, 1e6]", wait_us);
  return cuda_status(counted(launch_selftest_timeout((unsigned long long)wait_us * 1000ull, (cudaStream_t)stream), 1),
                     "selftest launch");
}

svsa_status svsa_sync_status(void* stream) {
  NvtxRange nvtx_("svsa_sync_status");
  g_last_error.clear();
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "stream synchronize");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "asynchronous error");
  // every tensor-core translation unit keeps its own error word; read (and clear) all of them
  cudaError_t (*readers[5])(unsigned int*, cudaStream_t) = {attn_fa_error, attn_tc_error, scores_tc_error,
                                                           route_tc_error, cocluster_tc_error};
  const char* names[5] = {"attention", "self-test", "scores", "routing", "co-clustering"};
  unsigned int first_code = 0u;
  const char* first_name = nullptr;
  for (int i = 0; i < 5; ++i) {
    unsigned int code = 0u;
    e = readers[i](&code, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e, "reading the device error word");
    if (code != 0u && first_name == nullptr) {
      first_code = code;
      first_name = names[i];
    }
  }
  // status bits of the data checks (reading clears them)
  unsigned int fl[3] = {0u, 0u, 0u};
  cudaError_t (*flag_readers[3])(unsigned int*, cudaStream_t) = {reorder_flags, pool_flags, sics_flags};
  for (int i = 0; i < 3; ++i) {
    e = flag_readers[i](&fl[i], (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e, "reading a status word");
  }
  const unsigned int bits = fl[0] | fl[1] | fl[2];
  if (first_name != nullptr)
    return fail(SVSA_ERR_TIMEOUT, "%s kernel: a bounded wait gave up (site %u)", first_name, first_code);
  if (bits & kFlagMask)
    return fail(SVSA_ERR_MASK, "a mask list checked before the attention was malformed "
                               "(kv_cnt outside [0, cap], an index outside [0, nb), not strictly ascending, "
                               "or a pairing table that is not a permutation)");
  if (bits & (kFlagRangeValue | kFlagRangeMean))
    return fail(SVSA_ERR_RANGE, "%s beyond the fp16 range (+-65504) or not finite; the result saturated",
                (bits & kFlagRangeValue) ? "a value given to svsa_reorder_values" : "a block mean of the scores");
  return SVSA_OK;
}

}  // extern "C"
