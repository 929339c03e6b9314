// Per-row block selection and compaction into the kept-block lists.
//
// Rules ("SVOO" 2.A and "SVG-EAR" 4: cumulative-mass / top-p; top-k; "LVSA"
// abstract: structured window with rotating anchors; "SVG-EAR" 2.B: routing by
// estimated error under the threshold rule's budget):
//   THRESHOLD  order the row by (score desc, index asc) and keep the shortest
//              prefix whose cumulative sum reaches tau;
//   TOPK       keep the first k of that order;
//   ROUTING    m = count THRESHOLD keeps on the score row, then the first m of
//              the (ratio desc, index asc) order of the ratio row;
//   STRUCTURED |t_I - t_J| <= win_t or |h_I - h_J| <= R or J an anchor.
//
// The ordered prefix is found without sorting: scores are non-negative
// floats, so their bit patterns order like the values.  A most-significant-
// digit-first radix select over the 31 bits below the sign (4 passes: the
// 8 exponent bits, then 8, 8 and 7 significand bits) histograms
// the candidates' counts and masses per digit, and a suffix scan over the 256
// digits locates the digit holding the crossing element.  After the 4th pass
// the crossing value v* is known exactly; everything above v* is kept, and of
// the elements equal to v* the first t in index order.  Short rows: one warp
// per row, its keys staged in shared memory once for all passes; long rows:
// one CTA per row.  Histogram updates are plain per-lane shared-memory
// atomics (measured faster than aggregating the lanes that share a digit with
// match / reduce).  Output lists are ascending by construction (ballot-based
// compaction in index order).
#include "common.cuh"

namespace svsa {

enum { SEL_THRESHOLD = 0, SEL_TOPK = 1, SEL_STRUCTURED = 2, SEL_ROUTING = 3 };

__device__ __forceinline__ uint32_t score_key(float x) { return x > 0.f ? __float_as_uint(x) : 0u; }

// ---------------------------------------------------------------- one warp per row
// Masses are exact 48-bit fixed-point integers (x * 2^48 truncated; scores are
// probabilities, x <= 1, so a row of up to 16384 sums below 2^62): every
// partial sum is exact and independent of the order it is taken in, so the
// crossing digit found in one pass is consistent with the next, and the sums
// differ from fp64 cumulative sums by < nb * 2^-48.
constexpr double kFix = 281474976710656.0;   // 2^48

__device__ __forceinline__ unsigned long long fix48(uint32_t key) {
  return (unsigned long long)((double)__uint_as_float(key) * kFix);
}

struct WarpHist {
  uint32_t cnt[256];
  unsigned long long mass[256];
};

struct Cut {
  uint32_t vstar;       // the crossing key
  uint32_t take;        // how many keys equal to vstar (first in index order) are kept
};

// Radix select over one row by a single warp: every pass reads the keys
// through `key_of` (the row staged in shared memory).  by_mass: the shortest
// prefix of the (key desc, index asc) order whose mass reaches tau_fx; else
// the first k.  The target must be reachable (the caller handles "keep all").
template <typename KeyOf>
__device__ Cut warp_radix_cut(KeyOf key_of, int n, bool by_mass, unsigned long long tau_fx, uint32_t k,
                              WarpHist& h) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0u, pmask = 0u, above_c = 0u, eq_c = 0u;
  unsigned long long above_m = 0ull;
  // digits below the (always clear) sign bit: bits 30-23 (the exponent, one
  // binade per bin), 22-15, 14-7 and 6-0
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = pass < 3 ? 23 - 8 * pass : 0;
    const uint32_t dmask = pass < 3 ? 255u : 127u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      h.cnt[lane * 8 + i] = 0u;
      h.mass[lane * 8 + i] = 0ull;
    }
    __syncwarp();
    for (int base = 0; base < n; base += 32) {
      const int j = base + lane;
      const uint32_t key = j < n ? key_of(j) : 0u;
      const bool cand = j < n && (key & pmask) == prefix;
      if (cand) {
        const uint32_t dg = (key >> shift) & dmask;
        if (by_mass) atomicAdd(&h.mass[dg], fix48(key));
        atomicAdd(&h.cnt[dg], 1u);
      }
    }
    __syncwarp();
    // lane L owns digits 255 - 8L .. 248 - 8L (descending); exclusive scan over lanes
    uint32_t c8[8];
    unsigned long long m8[8];
    uint32_t lc = 0u;
    unsigned long long lm = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int dg = 255 - (lane * 8 + i);
      c8[i] = h.cnt[dg];
      m8[i] = h.mass[dg];
      lc += c8[i];
      lm += m8[i];
    }
    uint32_t sc = lc;
    unsigned long long sm = lm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t yc = __shfl_up_sync(0xffffffffu, sc, o);
      const unsigned long long ym = __shfl_up_sync(0xffffffffu, sm, o);
      if (lane >= o) { sc += yc; sm += ym; }
    }
    uint32_t acc_c = above_c + sc - lc;           // everything above this lane's first digit
    unsigned long long acc_m = above_m + sm - lm;
    int hit = -1;
    uint32_t hit_above_c = 0u, hit_c = 0u;
    unsigned long long hit_above_m = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool reach = by_mass ? (acc_m + m8[i] >= tau_fx && acc_m < tau_fx) : (acc_c + c8[i] >= k && acc_c < k);
      if (hit < 0 && reach && c8[i] > 0u) {
        hit = 255 - (lane * 8 + i);
        hit_above_c = acc_c;
        hit_above_m = acc_m;
        hit_c = c8[i];
      }
      acc_c += c8[i];
      acc_m += m8[i];
    }
    const uint32_t hb = __ballot_sync(0xffffffffu, hit >= 0);
    const int src = hb ? __ffs(hb) - 1 : 31;     // exact sums: exactly one lane hits
    const int dg = __shfl_sync(0xffffffffu, hit, src);
    above_c = __shfl_sync(0xffffffffu, hit_above_c, src);
    above_m = __shfl_sync(0xffffffffu, hit_above_m, src);
    eq_c = __shfl_sync(0xffffffffu, hit_c, src);
    prefix |= (uint32_t)(dg < 0 ? 0 : dg) << shift;
    pmask |= dmask << shift;
    __syncwarp();
  }
  Cut cut;
  cut.vstar = prefix;
  if (by_mass) {
    const unsigned long long v = fix48(prefix);
    const unsigned long long need = tau_fx - above_m;           // > 0 by construction
    unsigned long long t = v > 0ull ? (need + v - 1ull) / v : (unsigned long long)eq_c;
    if (t < 1ull) t = 1ull;
    if (t > eq_c) t = eq_c;
    cut.take = (uint32_t)t;
  } else {
    cut.take = k - above_c;
  }
  return cut;
}

// One warp per row, blockDim.x / 32 rows per CTA.  The row's keys are copied
// once into this warp's slice of dynamic shared memory and every pass reads
// them there, so the row is read from global memory once, not once per pass.
// Dynamic shared memory: one histogram per warp, then one row of nb keys per
// warp.
constexpr int kSelMaxWarps = 4;
constexpr size_t kSelMaxSmem = 227 * 1024;   // opt-in dynamic shared memory per CTA

__global__ void __launch_bounds__(kSelMaxWarps * 32) select_kernel(
    const float* __restrict__ S, const float* __restrict__ R, long long rows, int nb, int mode, float tau, int k,
    int cap, int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt, uint32_t* __restrict__ bits) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int warps = (int)(blockDim.x >> 5);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * warps + wid;
  if (row >= rows) return;
  WarpHist& h = reinterpret_cast<WarpHist*>(sel_smem)[wid];
  uint32_t* const kbuf = reinterpret_cast<uint32_t*>(sel_smem + warps * sizeof(WarpHist)) + (size_t)wid * nb;
  const uint32_t lt = (1u << lane) - 1u;
  const int words = (nb + 31) / 32;
  const float* srow = S + row * (long long)nb;
  const float* rrow = R != nullptr ? R + row * (long long)nb : nullptr;
  // stage a row's keys; returns the lane's part of the fixed-point mass
  auto stage = [&](const float* src, bool mass) -> unsigned long long {
    unsigned long long part = 0ull;
    for (int j = lane; j < nb; j += 32) {
      const uint32_t key = score_key(__ldg(src + j));
      kbuf[j] = key;
      if (mass) part += fix48(key);
    }
    __syncwarp();
    return part;
  };
  auto key_at = [&](int j) { return kbuf[j]; };

  bool keep_all = false;
  uint32_t budget = 0u;
  Cut cut{0u, 0u};
  if (mode == SEL_THRESHOLD || mode == SEL_ROUTING) {
    unsigned long long part = stage(srow, true);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    const unsigned long long tau_fx = (unsigned long long)((double)tau * kFix);
    if ((double)tau >= 1.0 || part < tau_fx) {
      keep_all = true;
      budget = (uint32_t)nb;
    } else if (tau_fx == 0ull) {
      cut = warp_radix_cut(key_at, nb, false, 0ull, 1u, h);     // the shortest prefix is one block
      budget = 1u;
    } else {
      cut = warp_radix_cut(key_at, nb, true, tau_fx, 0u, h);
      // budget = kept count: keys above vstar plus `take`
      uint32_t above = 0u;
      for (int j = lane; j < nb; j += 32) above += key_at(j) > cut.vstar ? 1u : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
      budget = above + cut.take;
    }
  } else {  // TOPK
    budget = (uint32_t)k;
    if (k >= nb) keep_all = true;
    else {
      stage(srow, false);
      cut = warp_radix_cut(key_at, nb, false, 0ull, (uint32_t)k, h);
    }
  }
  const bool by_ratio = mode == SEL_ROUTING && !keep_all;
  if (by_ratio) {
    if (budget >= (uint32_t)nb) keep_all = true;
    else {
      __syncwarp();                      // every lane is done with the score keys
      stage(rrow, false);                // the cut and the compaction below read the ratios
      cut = warp_radix_cut(key_at, nb, false, 0ull, budget, h);
    }
  }

  int32_t* idx_out = kv_idx + row * (long long)cap;
  uint32_t* bits_out = bits ? bits + row * (long long)words : nullptr;
  uint32_t run = 0u, eq_run = 0u;
  for (int base = 0; base < nb; base += 32) {
    const int j = base + lane;
    bool f = j < nb;
    bool eq = false;
    if (!keep_all && f) {
      const uint32_t key = key_at(j);
      eq = key == cut.vstar;
      f = key > cut.vstar;
    }
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    if (eq) f = eq_run + (uint32_t)__popc(eb & lt) < cut.take;
    eq_run += (uint32_t)__popc(eb);
    const uint32_t fb = __ballot_sync(0xffffffffu, f);
    if (bits_out != nullptr && lane == 0) bits_out[base >> 5] = fb;
    if (f) idx_out[run + (uint32_t)__popc(fb & lt)] = j;
    run += (uint32_t)__popc(fb);
  }
  if (lane == 0) kv_cnt[row] = (int32_t)run;
}

// ---------------------------------------------------------------- one CTA per row
// Long rows (nb > kRowNbMin): a CTA of kRowThreads threads per row, the row's
// keys staged in shared memory once.  Same radix cut as the warp version: a
// 256-bin histogram per digit (one copy per warp, merged per bin, so that the
// shared-memory atomics of different warps never meet on one address), a
// block scan over the bins in descending digit order, and the one bin where
// the cumulative count or mass reaches its target.
constexpr int kRowThreads = 256;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowNbMin = 1024;
static_assert(kRowThreads == 256, "one histogram bin per thread");

struct RowShared {
  uint32_t cnt[kRowWarps][256];                 // one histogram per warp
  unsigned long long mass[kRowWarps][256];
  uint32_t wc[kRowWarps];
  unsigned long long wm[kRowWarps];
  uint32_t eq_w[kRowWarps];
  int hit_digit;
  uint32_t hit_above_c, hit_c;
  unsigned long long hit_above_m;
};

// Inclusive block scan of (c, m) over threadIdx.x (all kRowThreads threads call it).
__device__ __forceinline__ void row_scan(uint32_t& c, unsigned long long& m, RowShared& sh) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t yc = __shfl_up_sync(0xffffffffu, c, o);
    const unsigned long long ym = __shfl_up_sync(0xffffffffu, m, o);
    if (lane >= o) { c += yc; m += ym; }
  }
  if (lane == 31) { sh.wc[wid] = c; sh.wm[wid] = m; }
  __syncthreads();
  uint32_t oc = 0u;
  unsigned long long om = 0ull;
  for (int w = 0; w < wid; ++w) { oc += sh.wc[w]; om += sh.wm[w]; }
  c += oc;
  m += om;
  __syncthreads();
}

struct RowCut {
  uint32_t vstar;       // the crossing key
  uint32_t take;        // keys equal to vstar kept (first in index order)
  uint32_t above;       // keys strictly above vstar
};

// by_mass: the shortest prefix of the (key desc, index asc) order whose mass
// reaches tau_fx (reachable: the caller checked the row's total); else the
// first k (1 <= k < nb).
__device__ RowCut row_radix_cut(const uint32_t* keys, int nb, bool by_mass, unsigned long long tau_fx, uint32_t k,
                                RowShared& sh) {
  const int tid = threadIdx.x, wid = tid >> 5;
  uint32_t prefix = 0u, pmask = 0u, above_c = 0u, eq_c = 0u;
  unsigned long long above_m = 0ull;
  // digits below the (always clear) sign bit: bits 30-23 (the exponent, one
  // binade per bin), 22-15, 14-7 and 6-0
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = pass < 3 ? 23 - 8 * pass : 0;
    const uint32_t dmask = pass < 3 ? 255u : 127u;
#pragma unroll
    for (int w = 0; w < kRowWarps; ++w) {   // bin tid of every warp's histogram
      sh.cnt[w][tid] = 0u;
      sh.mass[w][tid] = 0ull;
    }
    if (tid == 0) {                    // (a reachable target always overwrites these)
      sh.hit_digit = 0;
      sh.hit_above_c = above_c;
      sh.hit_above_m = above_m;
      sh.hit_c = 0u;
    }
    __syncthreads();
    for (int base = 0; base < nb; base += kRowThreads) {
      const int j = base + tid;
      const uint32_t key = j < nb ? keys[j] : 0u;
      const bool cand = j < nb && (key & pmask) == prefix;
      if (cand) {                      // this warp's own histogram
        const uint32_t dg = (key >> shift) & dmask;
        if (by_mass) atomicAdd(&sh.mass[wid][dg], fix48(key));
        atomicAdd(&sh.cnt[wid][dg], 1u);
      }
    }
    __syncthreads();
    // thread t owns digit 255 - t: scan in descending digit order
    uint32_t c = 0u;
    unsigned long long m = 0ull;
#pragma unroll
    for (int w = 0; w < kRowWarps; ++w) {
      c += sh.cnt[w][255 - tid];
      m += sh.mass[w][255 - tid];
    }
    uint32_t sc = c;
    unsigned long long sm = m;
    row_scan(sc, sm, sh);
    const uint32_t ex_c = above_c + sc - c;
    const unsigned long long ex_m = above_m + sm - m;
    const bool reach = by_mass ? (ex_m + m >= tau_fx && ex_m < tau_fx) : (ex_c + c >= k && ex_c < k);
    if (reach && c > 0u) {             // exact sums: exactly one thread
      sh.hit_digit = 255 - tid;
      sh.hit_above_c = ex_c;
      sh.hit_above_m = ex_m;
      sh.hit_c = c;
    }
    __syncthreads();
    const int dg = sh.hit_digit;
    above_c = sh.hit_above_c;
    above_m = sh.hit_above_m;
    eq_c = sh.hit_c;
    prefix |= (uint32_t)dg << shift;
    pmask |= dmask << shift;
    __syncthreads();                   // the hit is read before the next pass clears the bins
  }
  RowCut cut;
  cut.vstar = prefix;
  cut.above = above_c;
  if (by_mass) {
    const unsigned long long v = fix48(prefix);
    const unsigned long long need = tau_fx - above_m;           // > 0 by construction
    unsigned long long t = v > 0ull ? (need + v - 1ull) / v : (unsigned long long)eq_c;
    if (t < 1ull) t = 1ull;
    if (t > eq_c) t = eq_c;
    cut.take = (uint32_t)t;
  } else {
    cut.take = k - above_c;
  }
  return cut;
}

// Stage a row's keys; returns the row's fixed-point mass (every thread).
__device__ unsigned long long row_stage(const float* __restrict__ src, int nb, uint32_t* keys, bool mass,
                                        RowShared& sh) {
  unsigned long long part = 0ull;
  for (int j = threadIdx.x; j < nb; j += kRowThreads) {
    const uint32_t key = score_key(__ldg(src + j));
    keys[j] = key;
    if (mass) part += fix48(key);
  }
  uint32_t c = 0u;
  row_scan(c, part, sh);               // (also orders the staging stores before later reads)
  if (threadIdx.x == kRowThreads - 1) sh.hit_above_m = part;
  __syncthreads();
  const unsigned long long total = sh.hit_above_m;
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kRowThreads, 4) select_row_kernel(
    const float* __restrict__ S, const float* __restrict__ R, int nb, int mode, float tau, int k, int cap,
    int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt, uint32_t* __restrict__ bits) {
  extern __shared__ __align__(16) uint32_t row_keys[];
  __shared__ RowShared sh;
  const long long row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int words = (nb + 31) / 32;
  bool keep_all = false;
  uint32_t budget = 0u;
  RowCut cut{0u, 0u, 0u};
  if (mode == SEL_THRESHOLD || mode == SEL_ROUTING) {
    const unsigned long long total = row_stage(S + row * (long long)nb, nb, row_keys, true, sh);
    const unsigned long long tau_fx = (unsigned long long)((double)tau * kFix);
    if ((double)tau >= 1.0 || total < tau_fx) {
      keep_all = true;
      budget = (uint32_t)nb;
    } else if (tau_fx == 0ull) {
      cut = row_radix_cut(row_keys, nb, false, 0ull, 1u, sh);   // the shortest prefix is one block
      budget = 1u;
    } else {
      cut = row_radix_cut(row_keys, nb, true, tau_fx, 0u, sh);
      budget = cut.above + cut.take;
    }
  } else {  // TOPK
    budget = (uint32_t)k;
    if (k >= nb) keep_all = true;
    else {
      row_stage(S + row * (long long)nb, nb, row_keys, false, sh);
      cut = row_radix_cut(row_keys, nb, false, 0ull, (uint32_t)k, sh);
    }
  }
  if (mode == SEL_ROUTING && !keep_all) {
    if (budget >= (uint32_t)nb) keep_all = true;
    else {
      row_stage(R + row * (long long)nb, nb, row_keys, false, sh);   // the ratios replace the scores
      cut = row_radix_cut(row_keys, nb, false, 0ull, budget, sh);
    }
  }

  // compaction in index order: keys above vstar, then the first `take` equal
  // to it.  Warp w owns the 32-aligned segment [w * seg, (w + 1) * seg): it
  // counts its keys above / equal, one barrier publishes the per-warp counts,
  // and each warp writes its kept indices at its offset.
  int32_t* idx_out = kv_idx + row * (long long)cap;
  uint32_t* bits_out = bits ? bits + row * (long long)words : nullptr;
  const uint32_t lt = (1u << lane) - 1u;
  const int seg = ((nb + kRowThreads - 1) / kRowThreads) * 32;
  const int s0 = wid * seg, s1 = min(nb, s0 + seg);
  auto flags = [&](int j, bool& gt, bool& eq) {
    const uint32_t key = (j < s1 && !keep_all) ? row_keys[j] : 0u;
    gt = j < s1 && (keep_all || key > cut.vstar);
    eq = j < s1 && !keep_all && key == cut.vstar;
  };
  uint32_t n_gt = 0u, n_eq = 0u;
  for (int base = s0; base < s1; base += 32) {
    bool gt, eq;
    flags(base + lane, gt, eq);
    n_gt += (uint32_t)__popc(__ballot_sync(0xffffffffu, gt));
    n_eq += (uint32_t)__popc(__ballot_sync(0xffffffffu, eq));
  }
  if (lane == 0) {
    sh.wc[wid] = n_gt;
    sh.eq_w[wid] = n_eq;
  }
  __syncthreads();
  uint32_t gt_before = 0u, eq_before = 0u, gt_all = 0u, eq_all = 0u;
#pragma unroll
  for (int w = 0; w < kRowWarps; ++w) {
    const uint32_t g = sh.wc[w], e = sh.eq_w[w];
    if (w < wid) { gt_before += g; eq_before += e; }
    gt_all += g;
    eq_all += e;
  }
  uint32_t run = gt_before + min(eq_before, cut.take);     // kept entries before this segment
  uint32_t eq_run = eq_before;                              // equal keys before the current word
  for (int base = s0; base < s1; base += 32) {
    bool gt, eq;
    flags(base + lane, gt, eq);
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    const bool f = gt || (eq && eq_run + (uint32_t)__popc(eb & lt) < cut.take);
    eq_run += (uint32_t)__popc(eb);
    const uint32_t fb = __ballot_sync(0xffffffffu, f);
    if (f) idx_out[run + (uint32_t)__popc(fb & lt)] = base + lane;
    if (bits_out != nullptr && lane == 0) bits_out[base >> 5] = fb;
    run += (uint32_t)__popc(fb);
  }
  if (tid == 0) kv_cnt[row] = (int32_t)(gt_all + min(eq_all, cut.take));
}

// STRUCTURED: block coordinates from the raster id of each block's first
// token.  A CTA takes kStructRows rows (one warp each); it first builds, in
// shared memory, every key block's (t, h) coordinate and a bitmap of the
// anchor columns, then each warp walks its row 32 blocks at a time and
// compacts with ballots (ascending lists, no block barriers).
constexpr int kStructRows = 8;

__global__ void __launch_bounds__(kStructRows * 32) structured_kernel(
    const int32_t* __restrict__ perm, long long rows, int nb, int H, int W, int win_t, int R, int n_anchors,
    int anchor_offset, int cap, int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
    uint32_t* __restrict__ bits) {
  extern __shared__ __align__(16) unsigned char st_smem[];
  int2* const crd = reinterpret_cast<int2*>(st_smem);                         // [nb] (t, h)
  uint32_t* const anchor = reinterpret_cast<uint32_t*>(st_smem + (size_t)nb * sizeof(int2));   // [words]
  const int words = (nb + 31) / 32;
  const long long HW = (long long)H * W;
  for (int J = threadIdx.x; J < nb; J += blockDim.x) {
    const long long r = perm[(long long)J * kBlock];
    crd[J] = make_int2((int)(r / HW), (int)((r % HW) / W));
  }
  for (int w = threadIdx.x; w < words; w += blockDim.x) anchor[w] = 0u;
  __syncthreads();
  const int stride = n_anchors > 0 ? (nb / n_anchors > 0 ? nb / n_anchors : 1) : 1;
  for (int m = threadIdx.x; m < n_anchors; m += blockDim.x) {
    const int J = (int)(((long long)anchor_offset + (long long)m * stride) % nb);
    atomicOr(&anchor[J >> 5], 1u << (J & 31));
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const long long row = (long long)blockIdx.x * kStructRows + (threadIdx.x >> 5);    // (bh, I)
  if (row >= rows) return;
  const int I = (int)(row % nb);
  const int2 cI = crd[I];
  int32_t* idx_out = kv_idx + row * (long long)cap;
  uint32_t* bits_out = bits ? bits + row * (long long)words : nullptr;
  uint32_t run = 0u;
  for (int base = 0; base < nb; base += 32) {
    const int J = base + lane;
    bool f = false;
    if (J < nb) {
      const int2 cJ = crd[J];
      f = abs(cI.x - cJ.x) <= win_t || abs(cI.y - cJ.y) <= R || ((anchor[J >> 5] >> (J & 31)) & 1u);
    }
    const uint32_t fb = __ballot_sync(0xffffffffu, f);
    if (bits_out != nullptr && lane == 0) bits_out[base >> 5] = fb;
    if (f) idx_out[run + (uint32_t)__popc(fb & lt)] = J;
    run += (uint32_t)__popc(fb);
  }
  if (lane == 0) kv_cnt[row] = (int32_t)run;
}

cudaError_t launch_select(const float* S, const float* R, long long rows, int nb, int mode, float tau,
                          int k, int cap, int32_t* kv_idx, int32_t* kv_cnt, uint32_t* bits,
                          cudaStream_t st) {
  if (nb > kRowNbMin) {
    // long rows: one CTA per row, its keys staged in shared memory
    const size_t smem = (size_t)nb * sizeof(uint32_t);
    if (smem + sizeof(RowShared) > kSelMaxSmem) return cudaErrorInvalidValue;
    if (smem > 48 * 1024 - sizeof(RowShared)) {
      const cudaError_t e = cudaFuncSetAttribute(select_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
      if (e != cudaSuccess) return e;
    }
    select_row_kernel<<<(unsigned)rows, kRowThreads, smem, st>>>(S, R, nb, mode, tau, k, cap, kv_idx, kv_cnt, bits);
    return cudaGetLastError();
  }
  // short rows: one warp per row, as many rows per CTA (up to 4) as fit in
  // shared memory with their keys
  const size_t per_warp = sizeof(WarpHist) + (size_t)nb * sizeof(uint32_t);
  const int warps = (int)std::min<size_t>(kSelMaxWarps, kSelMaxSmem / per_warp);
  if (warps < 1) return cudaErrorInvalidValue;
  const size_t smem = (size_t)warps * per_warp;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const long long blocks = (rows + warps - 1) / warps;
  select_kernel<<<(unsigned)blocks, warps * 32, smem, st>>>(S, R, rows, nb, mode, tau, k, cap, kv_idx, kv_cnt, bits);
  return cudaGetLastError();
}

cudaError_t launch_structured(const int32_t* perm, long long rows, int nb, int H, int W, int win_t,
                              int R, int n_anchors, int anchor_offset, int cap, int32_t* kv_idx,
                              int32_t* kv_cnt, uint32_t* bits, cudaStream_t st) {
  const size_t smem = (size_t)nb * sizeof(int2) + (size_t)((nb + 31) / 32) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(structured_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  structured_kernel<<<(unsigned)((rows + kStructRows - 1) / kStructRows), kStructRows * 32, smem, st>>>(
      perm, rows, nb, H, W, win_t, R, n_anchors, anchor_offset, cap, kv_idx, kv_cnt, bits);
  return cudaGetLastError();
}

}  // namespace svsa
