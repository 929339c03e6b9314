// Per-row block selection and compaction into the kept-block lists.
//
// Rules ("SVOO" 2.A and "SVG-EAR" 4: cumulative-mass / top-p; top-k; "LVSA"
// abstract: structured window with rotating anchors; "SVG-EAR" 2.B: routing by
// estimated error under the threshold rule's budget):
//   THRESHOLD  order the row by (score desc, index asc) and keep the shortest
//              prefix whose fp64 cumulative sum reaches tau;
//   TOPK       keep the first k of that order;
//   ROUTING    m = count THRESHOLD keeps on the score row, then the first m of
//              the (ratio desc, index asc) order of the ratio row;
//   STRUCTURED |t_I - t_J| <= win_t or |h_I - h_J| <= R or J an anchor.
//
// The ordered prefix is found without sorting: scores are non-negative
// floats, so their bit patterns order like the values.  A most-significant-
// digit-first radix select over the 32 bits (4 passes of 8 bits) histograms
// the candidates' counts and fp64 masses per digit, and a suffix scan over the
// 256 digits locates the digit holding the crossing element.  After the 4th
// pass the crossing value v* is known exactly; everything above v* is kept,
// and of the elements equal to v* the first t in index order.  One CTA per
// row; the row lives in shared memory; output lists are ascending by
// construction (a block-wide prefix count in index order).
#include "common.cuh"

namespace svsa {

constexpr int kSelThreads = 256;

enum { SEL_THRESHOLD = 0, SEL_TOPK = 1, SEL_STRUCTURED = 2, SEL_ROUTING = 3 };

struct SelShared {
  uint32_t cnt[256];
  double mass[256];
  uint32_t scan_cnt[kSelThreads / 32];
  double scan_mass[kSelThreads / 32];
  uint32_t prefix, above_cnt, eq_cnt, take;
  uint32_t found, min_dg;
  double above_mass, total;
  uint32_t run;                     // running output position (compaction)
};

__device__ __forceinline__ uint32_t score_key(float x) { return x > 0.f ? __float_as_uint(x) : 0u; }

// Block-wide inclusive scan of (count, mass) over threadIdx.x.
__device__ __forceinline__ void block_scan2(uint32_t& c, double& m, SelShared& sh) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t yc = __shfl_up_sync(0xffffffffu, c, o);
    const double ym = __shfl_up_sync(0xffffffffu, m, o);
    if (lane >= o) { c += yc; m += ym; }
  }
  if (lane == 31) { sh.scan_cnt[wid] = c; sh.scan_mass[wid] = m; }
  __syncthreads();
  uint32_t oc = 0; double om = 0.0;
  for (int w = 0; w < wid; ++w) { oc += sh.scan_cnt[w]; om += sh.scan_mass[w]; }
  c += oc; m += om;
  __syncthreads();
}

// Radix select over keys[0..n): on return sh.prefix = v* (bits), sh.above_cnt /
// sh.above_mass = count / mass strictly above v*, sh.eq_cnt = elements equal to
// v*, sh.take = how many of those (first in index order) are kept.
// by_mass: reach `tau` in mass; else reach `k` in count.  Requires a reachable
// target (caller handles "keep all").
__device__ void radix_cut(const uint32_t* keys, int n, bool by_mass, double tau, uint32_t k,
                          SelShared& sh) {
  const int tid = threadIdx.x;
  if (tid == 0) { sh.prefix = 0u; sh.above_cnt = 0u; sh.above_mass = 0.0; }
  uint32_t pmask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    sh.cnt[tid] = 0u;
    sh.mass[tid] = 0.0;
    if (tid == 0) { sh.found = 0u; sh.min_dg = 256u; }
    __syncthreads();
    const uint32_t prefix = sh.prefix;
    for (int j = tid; j < n; j += kSelThreads) {
      const uint32_t key = keys[j];
      if ((key & pmask) == prefix) {
        const uint32_t dg = (key >> shift) & 255u;
        atomicAdd(&sh.cnt[dg], 1u);
        if (by_mass) atomicAdd(&sh.mass[dg], (double)__uint_as_float(key));
      }
    }
    __syncthreads();
    // thread t owns digit 255 - t; inclusive scan = suffix sums over digits
    const uint32_t dg = 255u - (uint32_t)tid;
    uint32_t c = sh.cnt[dg];
    double m = sh.mass[dg];
    const uint32_t own_c = c;
    const double own_m = m;
    block_scan2(c, m, sh);
    const uint32_t above_c = sh.above_cnt;
    const double above_m = sh.above_mass;
    bool hit;
    if (by_mass) hit = (above_m + m >= tau) && (above_m + (m - own_m) < tau);
    else hit = (above_c + c >= k) && (above_c + (c - own_c) < k);
    if (own_c > 0u) atomicMin(&sh.min_dg, dg);
    if (hit) sh.found = 1u;
    __syncthreads();
    // fp64 sums taken in a different order in this pass can miss the target by
    // an ulp when the cumulative mass sits on tau; the crossing is then the
    // last candidate, i.e. the smallest non-empty digit.
    if (!sh.found && dg == sh.min_dg) hit = true;
    if (hit) {
      sh.prefix = prefix | (dg << shift);
      sh.above_cnt = above_c + (c - own_c);
      sh.above_mass = above_m + (m - own_m);
      sh.eq_cnt = own_c;
    }
    pmask |= 255u << shift;
    __syncthreads();
  }
  if (tid == 0) {
    uint32_t t = 1;
    if (by_mass) {
      const double v = (double)__uint_as_float(sh.prefix);
      double acc = sh.above_mass + v;
      while (acc < tau && t < sh.eq_cnt) { acc += v; ++t; }
    } else {
      t = k - sh.above_cnt;
    }
    sh.take = t;
  }
  __syncthreads();
}

// Write the kept list: flag(j) computed by `keep`; returns nothing, writes
// kv_idx (ascending), kv_cnt and the optional bit row.
template <typename KeepFn>
__device__ void compact_row(int n, KeepFn keep, int32_t* idx_out, int32_t* cnt_out,
                            uint32_t* bits_out, SelShared& sh) {
  const int tid = threadIdx.x;
  if (tid == 0) sh.run = 0u;
  __syncthreads();
  for (int base = 0; base < n; base += kSelThreads) {
    const int j = base + tid;
    const bool f = j < n && keep(j);
    const uint32_t ballot = __ballot_sync(0xffffffffu, f);
    if (bits_out != nullptr && (tid & 31) == 0 && base + (tid & ~31) < n)
      bits_out[(base + tid) >> 5] = ballot;
    uint32_t c = f ? 1u : 0u;
    double dummy = 0.0;
    const uint32_t own = c;
    block_scan2(c, dummy, sh);
    if (f) idx_out[sh.run + c - own] = j;
    __syncthreads();
    if (tid == kSelThreads - 1) sh.run += c;
    __syncthreads();
  }
  if (tid == 0) *cnt_out = (int32_t)sh.run;
}

// Prefix rank among the elements equal to v* (in index order) is needed to
// keep only the first `take` of them; computed on the fly during compaction.
__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ S, const float* __restrict__ R, int nb, int mode, float tau, int k,
    int cap, int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt, uint32_t* __restrict__ bits) {
  extern __shared__ uint32_t keys[];                   // [nb]
  __shared__ SelShared sh;
  const long long row = blockIdx.x;
  const int tid = threadIdx.x;
  const int words = (nb + 31) / 32;
  const float* srow = S + row * (long long)nb;

  // --- score row: total mass (fp64), keys
  double part = 0.0;
  for (int j = tid; j < nb; j += kSelThreads) {
    const uint32_t key = score_key(srow[j]);
    keys[j] = key;
    part += (double)__uint_as_float(key);
  }
  {
    uint32_t dc = 0;
    block_scan2(dc, part, sh);
    if (tid == kSelThreads - 1) sh.total = part;
    __syncthreads();
  }
  const double total = sh.total;

  bool keep_all = false;
  uint32_t budget = 0;
  if (mode == SEL_THRESHOLD || mode == SEL_ROUTING) {
    if ((double)tau >= 1.0 || total < (double)tau) {
      keep_all = true;
      budget = (uint32_t)nb;
    } else {
      radix_cut(keys, nb, true, (double)tau, 0u, sh);
      budget = sh.above_cnt + sh.take;
    }
  } else {  // TOPK
    budget = (uint32_t)k;
    if (k >= nb) keep_all = true;
    else radix_cut(keys, nb, false, 0.0, (uint32_t)k, sh);
  }

  if (mode == SEL_ROUTING && !keep_all) {
    // rank by the ratio row instead, same budget
    __syncthreads();
    const float* rrow = R + row * (long long)nb;
    for (int j = tid; j < nb; j += kSelThreads) keys[j] = score_key(rrow[j]);
    __syncthreads();
    if (budget >= (uint32_t)nb) keep_all = true;
    else radix_cut(keys, nb, false, 0.0, budget, sh);
  }

  int32_t* idx_out = kv_idx + row * (long long)cap;
  uint32_t* bits_out = bits ? bits + row * (long long)words : nullptr;
  if (keep_all) {
    compact_row(nb, [](int) { return true; }, idx_out, kv_cnt + row, bits_out, sh);
    return;
  }
  // elements equal to v*: keep the first `take` in index order.  A running
  // count of equal elements seen in earlier chunks plus an in-chunk scan.
  const uint32_t vstar = sh.prefix;
  const uint32_t take = sh.take;
  __shared__ uint32_t eq_run;
  if (tid == 0) { eq_run = 0u; sh.run = 0u; }
  __syncthreads();
  for (int base = 0; base < nb; base += kSelThreads) {
    const int j = base + tid;
    const uint32_t key = j < nb ? keys[j] : 0u;
    const bool eq = j < nb && key == vstar;
    uint32_t ce = eq ? 1u : 0u;
    double dz = 0.0;
    block_scan2(ce, dz, sh);
    const uint32_t eq_rank = eq_run + ce - (eq ? 1u : 0u);
    const bool f = j < nb && (key > vstar || (eq && eq_rank < take));
    const uint32_t ballot = __ballot_sync(0xffffffffu, f);
    if (bits_out != nullptr && (tid & 31) == 0 && base + (tid & ~31) < nb)
      bits_out[(base + tid) >> 5] = ballot;
    uint32_t c = f ? 1u : 0u;
    double dz2 = 0.0;
    block_scan2(c, dz2, sh);
    if (f) idx_out[sh.run + c - 1u] = j;
    __syncthreads();
    if (tid == kSelThreads - 1) { sh.run += c; eq_run += ce; }
    __syncthreads();
  }
  if (tid == 0) kv_cnt[row] = (int32_t)sh.run;
}

// STRUCTURED: block coordinates from the raster id of each block's first token.
__global__ void __launch_bounds__(kSelThreads) structured_kernel(
    const int32_t* __restrict__ perm, int nb, int H, int W, int win_t, int R, int n_anchors,
    int anchor_offset, int heads_rows, int cap, int32_t* __restrict__ kv_idx,
    int32_t* __restrict__ kv_cnt, uint32_t* __restrict__ bits) {
  __shared__ SelShared sh;
  const long long row = blockIdx.x;                    // (bh, I)
  const int I = (int)(row % nb);
  const int words = (nb + 31) / 32;
  const long long HW = (long long)H * W;
  auto coord = [&](int J, int& t, int& h) {
    const long long r = perm[(long long)J * kBlock];
    t = (int)(r / HW);
    h = (int)((r % HW) / W);
  };
  int tI, hI;
  coord(I, tI, hI);
  const int stride = n_anchors > 0 ? (nb / n_anchors > 0 ? nb / n_anchors : 1) : 1;
  auto keep = [&](int J) {
    int tJ, hJ;
    coord(J, tJ, hJ);
    if (abs(tI - tJ) <= win_t || abs(hI - hJ) <= R) return true;
    for (int m = 0; m < n_anchors; ++m)
      if (((long long)anchor_offset + (long long)m * stride) % nb == J) return true;
    return false;
  };
  compact_row(nb, keep, kv_idx + row * (long long)cap, kv_cnt + row,
              bits ? bits + row * (long long)words : nullptr, sh);
  (void)heads_rows;
}

cudaError_t launch_select(const float* S, const float* R, long long rows, int nb, int mode, float tau,
                          int k, int cap, int32_t* kv_idx, int32_t* kv_cnt, uint32_t* bits,
                          cudaStream_t st) {
  const size_t smem = (size_t)nb * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)std::max<size_t>(smem, 1));
  if (e != cudaSuccess) return e;
  select_kernel<<<(unsigned)rows, kSelThreads, smem, st>>>(S, R, nb, mode, tau, k, cap, kv_idx,
                                                            kv_cnt, bits);
  return cudaGetLastError();
}

cudaError_t launch_structured(const int32_t* perm, long long rows, int nb, int H, int W, int win_t,
                              int R, int n_anchors, int anchor_offset, int cap, int32_t* kv_idx,
                              int32_t* kv_cnt, uint32_t* bits, cudaStream_t st) {
  structured_kernel<<<(unsigned)rows, kSelThreads, 0, st>>>(perm, nb, H, W, win_t, R, n_anchors,
                                                            anchor_offset, 0, cap, kv_idx, kv_cnt, bits);
  return cudaGetLastError();
}

}  // namespace svsa
