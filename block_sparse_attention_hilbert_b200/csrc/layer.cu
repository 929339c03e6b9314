// The whole layer on host buffers (svsa_layer_*): a layer object owns one
// device arena holding every buffer of the four steps (with two sets of input
// staging, used in turn), plus two copy streams and the events that chain
// them to the caller's stream.  A call streams the
// (batch, head) rows in groups -- inputs in on one stream, the four steps on
// the caller's stream, the output out on another -- through the library's
// own entry points, one group's copies overlapping another group's work.
#include <algorithm>
#include <cstdio>
#include <numeric>
#include <vector>

#include "common.cuh"
#include "svsa.h"

namespace svsa {
svsa_status record_error(svsa_status st, const char* msg);
}

struct svsa_layer {
  svsa_shape s;
  svsa_layer_config cfg;
  svsa::Dims g;
  int device = 0;
  char* arena = nullptr;
  int32_t *perm = nullptr, *iperm = nullptr;
  void *perm_ws = nullptr, *mask_ws = nullptr, *attn_ws = nullptr;
  size_t perm_ws_bytes = 0, mask_ws_bytes = 0, attn_ws_bytes = 0;
  void *qp = nullptr, *kp = nullptr, *vp = nullptr, *op = nullptr;
  void *sq[2] = {}, *sk[2] = {}, *sv[2] = {};   // raster input staging, two sets used in turn
  void* so = nullptr;                           // raster output staging
  int32_t *kv_idx = nullptr, *kv_cnt = nullptr, *nvalid = nullptr;
  uint32_t* bits = nullptr;
  float *kbar = nullptr, *vbar = nullptr;
  void* cbar = nullptr;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev_start = nullptr, ev_done = nullptr;
  cudaEvent_t ev_free[2] = {};                  // the caller's stream has read input set i
  std::vector<cudaEvent_t> ev_in[2], ev_out;    // per group: inputs of set i arrived / output ready
  unsigned long long calls = 0;
  std::vector<long long> bounds;   // row group bounds
  bool mask_ready = false;
};

namespace {

using svsa::record_error;

svsa_status err(svsa_status st, const char* fmt, long long a = 0, long long b = 0) {
  char buf[256];
  snprintf(buf, sizeof(buf), fmt, a, b);
  return record_error(st, buf);
}

svsa_status cuda_err(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SVSA_OK;
  char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", what, cudaGetErrorString(e));
  return record_error(SVSA_ERR_CUDA, buf);
}

#define LTRY(expr)                    \
  do {                                \
    svsa_status _s = (expr);          \
    if (_s != SVSA_OK) return _s;     \
  } while (0)

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

bool needs_means(const svsa_layer_config& c) { return c.compensate != 0 || c.mask.routing != 0; }
bool needs_bits(const svsa_layer_config& c) { return c.compensate != 0 || c.paired != 0; }

// Offsets of every buffer in the arena (256-byte aligned).
struct Arena {
  size_t perm, iperm, perm_ws, qp, kp, vp, op, sq[2], sk[2], sv[2], so, kv_idx, kv_cnt, nvalid, bits, kbar, vbar,
      cbar, mask_ws, attn_ws, total;
};

svsa_status layout(const svsa_shape& s, const svsa_layer_config& c, Arena& A, size_t& perm_ws_bytes,
                   size_t& mask_ws_bytes, size_t& attn_ws_bytes) {
  if (c.order != SVSA_ORDER_RASTER && c.order != SVSA_ORDER_HILBERT)
    return err(SVSA_ERR_UNSUPPORTED, "layer order %lld: raster or hilbert (the co-clustering order is built "
                                     "from the device tensors of the whole layer)", c.order);
  if (c.attn_passes < 1 || c.attn_passes > 8)
    return err(SVSA_ERR_INVALID_ARG, "attn_passes=%lld outside [1, 8]", c.attn_passes);
  if (s.B < 1 || s.heads < 1 || s.T < 1 || s.H < 1 || s.W < 1)
    return err(SVSA_ERR_INVALID_ARG, "shape dims must be >= 1");
  if (s.d != 64 && s.d != 128) return err(SVSA_ERR_UNSUPPORTED, "head dim d=%lld (supported: 64, 128)", s.d);
  const svsa::Dims g = svsa::make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  if (c.groups < 1 || c.groups > g.BH)
    return err(SVSA_ERR_INVALID_ARG, "groups=%lld outside [1, B*heads=%lld]", c.groups, g.BH);
  if (g.BH * g.Npad * s.d >= (1LL << 31) || g.N >= (1LL << 31))
    return err(SVSA_ERR_UNSUPPORTED, "layer too large for int32 indexing");
  perm_ws_bytes = svsa_perm_workspace_bytes(s, c.order);
  mask_ws_bytes = svsa_mask_workspace_bytes(s, &c.mask);
  attn_ws_bytes = c.paired ? svsa_attn_paired_workspace_bytes(s, c.attn_passes)
                           : svsa_attn_split_workspace_bytes(s, c.attn_passes);
  const size_t words = (size_t)(g.nb + 31) / 32, rows = (size_t)g.BH, nb = (size_t)g.nb;
  const size_t tok = rows * (size_t)g.Npad * s.d * 2, raw = rows * (size_t)g.N * s.d * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += a256(bytes); return o; };
  A.perm = take((size_t)g.Npad * 4);
  A.iperm = take((size_t)g.N * 4);
  A.perm_ws = take(perm_ws_bytes);
  A.qp = take(tok); A.kp = take(tok); A.vp = take(tok); A.op = take(tok);
  for (int i = 0; i < 2; ++i) {
    A.sq[i] = take(raw); A.sk[i] = take(raw); A.sv[i] = take(raw);
  }
  A.so = take(raw);
  A.kv_idx = take(rows * nb * nb * 4);            // cap = nb
  A.kv_cnt = take(rows * nb * 4);
  A.nvalid = take(needs_means(c) ? nb * 4 : 0);
  A.bits = take(needs_bits(c) ? rows * nb * words * 4 : 0);
  A.kbar = take(needs_means(c) ? rows * nb * s.d * 4 : 0);
  A.vbar = take(needs_means(c) ? rows * nb * s.d * 4 : 0);
  A.cbar = take(c.compensate ? rows * nb * 2 * s.d * 2 : 0);
  A.mask_ws = take(mask_ws_bytes);
  A.attn_ws = take(attn_ws_bytes);
  A.total = off;
  return SVSA_OK;
}

void release(svsa_layer* L) {
  for (int i = 0; i < 2; ++i) {
    for (cudaEvent_t e : L->ev_in[i]) if (e) cudaEventDestroy(e);
    if (L->ev_free[i]) cudaEventDestroy(L->ev_free[i]);
  }
  for (cudaEvent_t e : L->ev_out) if (e) cudaEventDestroy(e);
  if (L->ev_start) cudaEventDestroy(L->ev_start);
  if (L->ev_done) cudaEventDestroy(L->ev_done);
  if (L->h2d) cudaStreamDestroy(L->h2d);
  if (L->d2h) cudaStreamDestroy(L->d2h);
  if (L->arena) cudaFree(L->arena);
  delete L;
}

// The mask struct of rows [r0, r1) of the layer.
svsa_mask group_mask(const svsa_layer* L, long long r0) {
  const long long nb = L->g.nb, words = (nb + 31) / 32, d = L->s.d;
  svsa_mask m{};
  m.kv_idx = L->kv_idx + r0 * nb * nb;
  m.kv_cnt = L->kv_cnt + r0 * nb;
  m.cap = (int32_t)nb;
  m.bits = L->bits ? L->bits + r0 * nb * words : nullptr;
  m.kbar = L->kbar ? L->kbar + r0 * nb * d : nullptr;
  m.vbar = L->vbar ? L->vbar + r0 * nb * d : nullptr;
  m.nvalid = L->nvalid;
  m.cbar = L->cbar ? static_cast<char*>(L->cbar) + r0 * nb * 2 * d * 2 : nullptr;
  m.pairs = nullptr;                           // the paired split takes blocks 2p and 2p + 1
  m.check = 0;
  return m;
}

}  // namespace

extern "C" {

size_t svsa_layer_device_bytes(svsa_shape s, const svsa_layer_config* cfg) {
  if (cfg == nullptr) return 0;
  Arena A{};
  size_t a = 0, b = 0, c = 0;
  if (layout(s, *cfg, A, a, b, c) != SVSA_OK) return 0;
  return A.total;
}

svsa_status svsa_layer_create(svsa_shape s, const svsa_layer_config* cfg, svsa_layer** out) {
  if (out == nullptr) return err(SVSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (cfg == nullptr) return err(SVSA_ERR_INVALID_ARG, "cfg is NULL");
  Arena A{};
  size_t perm_ws = 0, mask_ws = 0, attn_ws = 0;
  LTRY(layout(s, *cfg, A, perm_ws, mask_ws, attn_ws));
  svsa_layer* L = new svsa_layer();
  L->s = s;
  L->cfg = *cfg;
  L->g = svsa::make_dims(s.B, s.heads, s.T, s.H, s.W, s.d);
  auto fail_free = [&](svsa_status st) { release(L); return st; };
  svsa_status st = cuda_err(cudaGetDevice(&L->device), "cudaGetDevice");
  if (st != SVSA_OK) return fail_free(st);
  st = cuda_err(cudaMalloc(reinterpret_cast<void**>(&L->arena), A.total), "layer arena");
  if (st != SVSA_OK) return fail_free(st);
  auto at = [&](size_t off) { return static_cast<void*>(L->arena + off); };
  L->perm = static_cast<int32_t*>(at(A.perm));
  L->iperm = static_cast<int32_t*>(at(A.iperm));
  L->perm_ws = perm_ws ? at(A.perm_ws) : nullptr;
  L->perm_ws_bytes = perm_ws;
  L->qp = at(A.qp); L->kp = at(A.kp); L->vp = at(A.vp); L->op = at(A.op);
  for (int i = 0; i < 2; ++i) {
    L->sq[i] = at(A.sq[i]); L->sk[i] = at(A.sk[i]); L->sv[i] = at(A.sv[i]);
  }
  L->so = at(A.so);
  L->kv_idx = static_cast<int32_t*>(at(A.kv_idx));
  L->kv_cnt = static_cast<int32_t*>(at(A.kv_cnt));
  L->nvalid = needs_means(*cfg) ? static_cast<int32_t*>(at(A.nvalid)) : nullptr;
  L->bits = needs_bits(*cfg) ? static_cast<uint32_t*>(at(A.bits)) : nullptr;
  L->kbar = needs_means(*cfg) ? static_cast<float*>(at(A.kbar)) : nullptr;
  L->vbar = needs_means(*cfg) ? static_cast<float*>(at(A.vbar)) : nullptr;
  L->cbar = cfg->compensate ? at(A.cbar) : nullptr;
  L->mask_ws = mask_ws ? at(A.mask_ws) : nullptr;
  L->mask_ws_bytes = mask_ws;
  L->attn_ws = attn_ws ? at(A.attn_ws) : nullptr;
  L->attn_ws_bytes = attn_ws;
  // row groups: bounds keep every per-row mask slice 16-byte aligned (a
  // group's first row times nb int32 entries must be a multiple of 4 words)
  const long long rows = L->g.BH;
  const long long unit = 4 / std::gcd((long long)L->g.nb, 4LL);
  for (int k = 0; k <= cfg->groups; ++k) {
    const long long r = k == cfg->groups ? rows : std::min(rows, (rows * k / cfg->groups) / unit * unit);
    if (L->bounds.empty() || r > L->bounds.back()) L->bounds.push_back(r);
  }
  const size_t ng = L->bounds.size() - 1;
  st = cuda_err(cudaStreamCreateWithFlags(&L->h2d, cudaStreamNonBlocking), "copy stream");
  if (st == SVSA_OK) st = cuda_err(cudaStreamCreateWithFlags(&L->d2h, cudaStreamNonBlocking), "copy stream");
  if (st == SVSA_OK) st = cuda_err(cudaEventCreateWithFlags(&L->ev_start, cudaEventDisableTiming), "event");
  if (st == SVSA_OK) st = cuda_err(cudaEventCreateWithFlags(&L->ev_done, cudaEventDisableTiming), "event");
  for (int k = 0; k < 2; ++k) {
    L->ev_in[k].assign(ng, nullptr);
    if (st == SVSA_OK) st = cuda_err(cudaEventCreateWithFlags(&L->ev_free[k], cudaEventDisableTiming), "event");
  }
  L->ev_out.assign(ng, nullptr);
  for (size_t i = 0; i < ng && st == SVSA_OK; ++i) {
    st = cuda_err(cudaEventCreateWithFlags(&L->ev_in[0][i], cudaEventDisableTiming), "event");
    if (st == SVSA_OK) st = cuda_err(cudaEventCreateWithFlags(&L->ev_in[1][i], cudaEventDisableTiming), "event");
    if (st == SVSA_OK) st = cuda_err(cudaEventCreateWithFlags(&L->ev_out[i], cudaEventDisableTiming), "event");
  }
  if (st != SVSA_OK) return fail_free(st);
  // the token order, once
  st = svsa_build_perm(s, cfg->order, L->perm, L->iperm, L->perm_ws, L->perm_ws_bytes, L->h2d);
  if (st == SVSA_OK) st = cuda_err(cudaStreamSynchronize(L->h2d), "token order");
  if (st != SVSA_OK) return fail_free(st);
  *out = L;
  return SVSA_OK;
}

svsa_status svsa_layer_forward_host(svsa_layer* L, const void* q, const void* k, const void* v, void* o,
                                    int32_t step, int32_t flags, void* stream) {
  if (L == nullptr) return err(SVSA_ERR_INVALID_ARG, "layer is NULL");
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
    return err(SVSA_ERR_INVALID_ARG, "a host buffer is NULL");
  if (step < 0) return err(SVSA_ERR_INVALID_ARG, "step=%lld < 0", step);
  if (flags & ~(int32_t)(SVSA_LAYER_REUSE_MASK | SVSA_LAYER_INPUTS_READY))
    return err(SVSA_ERR_INVALID_ARG, "unknown flags %lld", flags);
  int dev = -1;
  LTRY(cuda_err(cudaGetDevice(&dev), "cudaGetDevice"));
  if (dev != L->device) return err(SVSA_ERR_INVALID_ARG, "current device %lld, layer on %lld", dev, L->device);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const bool build = !((flags & SVSA_LAYER_REUSE_MASK) && L->mask_ready);
  svsa_mask_params p = L->cfg.mask;
  p.step = step;
  const long long N = L->g.N, Npad = L->g.Npad, d = L->s.d;
  const size_t row_raw = (size_t)N * d * 2, row_tok = (size_t)Npad * d * 2;
  const size_t ng = L->bounds.size() - 1;
  auto raw = [&](const void* base, long long r) { return static_cast<const char*>(base) + r * row_raw; };
  auto rawm = [&](void* base, long long r) { return static_cast<char*>(base) + r * row_raw; };
  auto tokm = [&](void* base, long long r) { return static_cast<char*>(base) + r * row_tok; };
  // Input set of this call (the two sets alternate).  The output copies start
  // after what the caller's stream has queued (which includes the previous
  // call's last output copy); so do the input copies, unless the caller
  // declares its host inputs ready -- then they wait only until the call two
  // back has read this set, and overlap the previous call's work.
  const int set = (int)(L->calls++ & 1ull);
  LTRY(cuda_err(cudaEventRecord(L->ev_start, cs), "event record"));
  LTRY(cuda_err(cudaStreamWaitEvent(L->h2d, (flags & SVSA_LAYER_INPUTS_READY) ? L->ev_free[set] : L->ev_start, 0),
                "stream wait"));
  LTRY(cuda_err(cudaStreamWaitEvent(L->d2h, L->ev_start, 0), "stream wait"));
  void *sq = L->sq[set], *sk = L->sk[set], *sv = L->sv[set];
  // every group's inputs first, so the link stays busy whatever the host's launch rate
  for (size_t gi = 0; gi < ng; ++gi) {
    const long long r0 = L->bounds[gi], r1 = L->bounds[gi + 1];
    const size_t bytes = (size_t)(r1 - r0) * row_raw;
    LTRY(cuda_err(cudaMemcpyAsync(rawm(sq, r0), raw(q, r0), bytes, cudaMemcpyHostToDevice, L->h2d), "copy in"));
    LTRY(cuda_err(cudaMemcpyAsync(rawm(sk, r0), raw(k, r0), bytes, cudaMemcpyHostToDevice, L->h2d), "copy in"));
    LTRY(cuda_err(cudaMemcpyAsync(rawm(sv, r0), raw(v, r0), bytes, cudaMemcpyHostToDevice, L->h2d), "copy in"));
    LTRY(cuda_err(cudaEventRecord(L->ev_in[set][gi], L->h2d), "event record"));
  }
  for (size_t gi = 0; gi < ng; ++gi) {
    const long long r0 = L->bounds[gi], r1 = L->bounds[gi + 1];
    svsa_shape gs = L->s;
    gs.B = 1;
    gs.heads = (int32_t)(r1 - r0);
    svsa_mask m = group_mask(L, r0);
    void *gq = tokm(L->qp, r0), *gk = tokm(L->kp, r0), *gv = tokm(L->vp, r0), *go = tokm(L->op, r0);
    LTRY(cuda_err(cudaStreamWaitEvent(cs, L->ev_in[set][gi], 0), "stream wait"));
    LTRY(svsa_reorder(rawm(sq, r0), gq, L->perm, gs, cs));
    LTRY(svsa_reorder(rawm(sk, r0), gk, L->perm, gs, cs));
    LTRY(svsa_reorder_values(rawm(sv, r0), gv, L->perm, gs, cs));
    if (build) LTRY(svsa_build_mask(gq, gk, gv, L->perm, gs, &p, &m, L->mask_ws, L->mask_ws_bytes, cs));
    if (L->cfg.paired)
      LTRY(svsa_attn_fwd_paired(gq, gk, gv, &m, L->cfg.compensate, go, nullptr, gs, L->cfg.attn_passes,
                                L->attn_ws, L->attn_ws_bytes, cs));
    else
      LTRY(svsa_attn_fwd_split(gq, gk, gv, &m, L->cfg.compensate, go, nullptr, gs, L->cfg.attn_passes,
                               L->attn_ws, L->attn_ws_bytes, cs));
    LTRY(svsa_inverse_reorder(go, rawm(L->so, r0), L->iperm, gs, cs));
    LTRY(cuda_err(cudaEventRecord(L->ev_out[gi], cs), "event record"));
    LTRY(cuda_err(cudaStreamWaitEvent(L->d2h, L->ev_out[gi], 0), "stream wait"));
    LTRY(cuda_err(cudaMemcpyAsync(static_cast<char*>(o) + r0 * row_raw, rawm(L->so, r0), (size_t)(r1 - r0) * row_raw,
                                  cudaMemcpyDeviceToHost, L->d2h), "copy out"));
  }
  if (build) L->mask_ready = true;
  LTRY(cuda_err(cudaEventRecord(L->ev_free[set], cs), "event record"));   // this call's reads of the set
  LTRY(cuda_err(cudaEventRecord(L->ev_done, L->d2h), "event record"));
  return cuda_err(cudaStreamWaitEvent(cs, L->ev_done, 0), "stream wait");
}

svsa_status svsa_layer_destroy(svsa_layer* L) {
  if (L == nullptr) return SVSA_OK;
  const int dev = L->device;
  int prev = -1;
  cudaGetDevice(&prev);
  if (prev != dev) cudaSetDevice(dev);
  // work queued on the caller's stream may still use the arena
  const cudaError_t e = cudaDeviceSynchronize();
  release(L);
  if (prev >= 0 && prev != dev) cudaSetDevice(prev);
  return cuda_err(e, "layer destroy");
}

}  // extern "C"
