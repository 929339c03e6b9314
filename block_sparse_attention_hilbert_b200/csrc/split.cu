// Key-range passes for layers whose keys and values outgrow L2.
//
// The attention of a query block over its kept key blocks is split into P
// passes over the key-block ranges [p * R, (p + 1) * R), R = ceil(nb / P):
// each pass is an exact attention over the kept blocks of its range and
// yields O_p (fp32, normalised within the pass) and its log-sum-exp lse_p;
// then
//     lse = log sum_p exp(lse_p),    O = sum_p exp(lse_p - lse) O_p
// is the attention over all kept blocks (the softmax over a union of
// disjoint key sets).  A pass touches 1 / P of a head's keys and values, so
// that working set stays in L2 while the query blocks stream.
//
// split_mask_kernel cuts every ascending kept list into its P range lists
// (each at most R long, so the P masks together take the room of one);
// sched_kernel balances each pass's items over the attention's persistent
// CTAs; combine_kernel merges the passes.
#include <climits>

#include <cuda_fp16.h>

#include "common.cuh"

namespace svsa {
namespace {

constexpr int kWarps = 8;

// One warp per (bh, query block) row.  Lists are ascending: the entries of
// range p are a contiguous run starting at the count of entries below p * R.
__global__ void split_mask_kernel(const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt, int cap,
                                  long long rows, int nb, int P, int R, int32_t* __restrict__ idx_p,
                                  int32_t* __restrict__ cnt_p) {
  const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int c0 = kv_cnt[row];
  const int cnt = c0 < 0 ? 0 : (c0 > cap ? cap : c0);
  const int32_t* lst = kv_idx + row * (long long)cap;
  // start[p] = entries with J < p * R (ascending lists)
  int below[9];
#pragma unroll
  for (int p = 0; p <= 8; ++p) below[p] = 0;
  for (int e = lane; e < cnt; e += 32) {
    int J = lst[e];
    J = J < 0 ? 0 : (J >= nb ? nb - 1 : J);
    const int pe = J / R;
#pragma unroll
    for (int p = 1; p <= 8; ++p)
      if (p <= P && pe < p) ++below[p];
  }
#pragma unroll
  for (int p = 1; p <= 8; ++p) below[p] = (int)warp_sum((float)below[p]);
  for (int p = 0; p < P; ++p) {
    const int s = p == 0 ? 0 : below[p];
    const int t = p + 1 == P ? cnt : below[p + 1];
    if (lane == 0) cnt_p[(long long)p * rows + row] = t - s;
    for (int e = s + lane; e < t; e += 32) {
      int J = lst[e];
      J = J < 0 ? 0 : (J >= nb ? nb - 1 : J);
      const int pos = e - s;
      if (pos < R) idx_p[((long long)p * rows + row) * R + pos] = J;
    }
  }
}

// One warp per output row: O = sum_p exp(lse_p - lse) O_p, lse = log sum exp(lse_p).
template <int D>
__global__ void combine_kernel(const float* __restrict__ o_p, const float* __restrict__ lse_p, long long rows, int P,
                               __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out) {
  const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int p = 0; p < P; ++p) m = fmaxf(m, lse_p[(long long)p * rows + row]);
  constexpr int U = D / 32;
  float acc[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc[u] = 0.f;
  float wsum = 0.f;
  if (m > -INFINITY) {
    for (int p = 0; p < P; ++p) {
      const float l = lse_p[(long long)p * rows + row];
      if (l == -INFINITY) continue;
      const float w = __expf(l - m);
      wsum += w;
      const float* src = o_p + ((long long)p * rows + row) * D;
#pragma unroll
      for (int u = 0; u < U; ++u) acc[u] = fmaf(w, src[lane + 32 * u], acc[u]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) out[row * D + lane + 32 * u] = __float2bfloat16_rn(acc[u] * inv);
  if (lse_out != nullptr && lane == 0) lse_out[row] = wsum > 0.f ? m + __logf(wsum) : 0.f;
}

// One warp per pair item p of a head: the query blocks I0 = pairs[2p] and
// I1 = pairs[2p + 1] (2p and 2p + 1 without a table).  Writes the blocks of
// each list that the partner does not keep -- A \ B for I0, B \ A for I1 --
// as ascending lists (ballot compaction in list order); the partner's kept
// set is read from its bitmap row.  A block without a partner (odd nb) keeps
// its whole list.  Entries are clamped to [0, nb), counts to [0, cap]; the
// output rows have xcap = min(cap, nb) entries (more than nb only for a list
// with repeats, whose excess is dropped).
__global__ void exclusive_kernel(const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt, int cap,
                                 const uint32_t* __restrict__ bits, const int32_t* __restrict__ pairs, long long BH,
                                 int nb, int npairs, int32_t* __restrict__ x_idx, int xcap,
                                 int32_t* __restrict__ x_cnt) {
  const long long item = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (item >= BH * npairs) return;
  const long long bh = item / npairs;
  const int p = (int)(item % npairs);
  const int words = (nb + 31) / 32;
  int blk[2] = {2 * p, 2 * p + 1 < nb ? 2 * p + 1 : -1};
  if (pairs != nullptr) {
    for (int h = 0; h < 2; ++h)
      if (blk[h] >= 0) {
        const int x = pairs[bh * nb + blk[h]];
        blk[h] = x < 0 ? 0 : (x >= nb ? nb - 1 : x);
      }
  }
  for (int h = 0; h < 2; ++h) {
    const int I = blk[h], Ip = blk[h ^ 1];
    if (I < 0) continue;
    const long long row = bh * nb + I;
    const int c0 = kv_cnt[row];
    const int cnt = c0 < 0 ? 0 : (c0 > cap ? cap : c0);
    const int32_t* lst = kv_idx + row * (long long)cap;
    const uint32_t* pb = Ip >= 0 ? bits + (bh * nb + Ip) * (long long)words : nullptr;
    int out = 0;
    for (int base = 0; base < cnt; base += 32) {
      const int e = base + lane;
      int J = 0;
      bool keep = false;
      if (e < cnt) {
        J = lst[e];
        J = J < 0 ? 0 : (J >= nb ? nb - 1 : J);
        keep = pb == nullptr || ((pb[J >> 5] >> (J & 31)) & 1u) == 0u;
      }
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      const int at = out + __popc(m & ((1u << lane) - 1u));
      if (keep && at < xcap) x_idx[row * (long long)xcap + at] = J;
      out += __popc(m);
    }
    if (lane == 0) x_cnt[row] = out < xcap ? out : xcap;
  }
}

// Wave-by-wave longest-first assignment of one pass's items to the G
// persistent CTAs of the attention (one CTA of this kernel per pass).  Wave w
// holds items [w G, w G + G) -- neighbouring query blocks, which share their
// keys in L2, so they still run together.  Its items, ranked by estimated
// cost (descending, ties to the lower index), go to the CTAs ranked by the
// cost already given to them (ascending, ties to the lower index), so after
// every wave the CTAs' totals stay within about one item of each other.
// Cost of an item: its pair tiles ((count + 1) / 2) plus 2 for the per-item
// work; an empty item 1.  sched[p][w][b] = item index, or -1 (the last wave
// of a pass whose items are not a multiple of G).
constexpr int kSchedMaxG = 256;

__global__ void __launch_bounds__(2 * kSchedMaxG) sched_kernel(const int32_t* __restrict__ cnt_p, long long items,
                                                               int cap, int G, long long nwaves,
                                                               int32_t* __restrict__ sched) {
  // slots G.. hold values that never rank before a real one (read in 16-byte vectors)
  __shared__ __align__(16) int cost[kSchedMaxG];
  __shared__ __align__(16) long long load[kSchedMaxG];
  __shared__ int16_t item_at[kSchedMaxG], cta_at[kSchedMaxG];
  const int t = threadIdx.x;
  const int32_t* cnt = cnt_p + (long long)blockIdx.x * items;
  int32_t* out = sched + (long long)blockIdx.x * nwaves * G;
  const int G4 = (G + 3) >> 2, G2 = (G + 1) >> 1;
  if (t < kSchedMaxG) {
    load[t] = t < G ? 0 : LLONG_MAX;
    cost[t] = INT_MIN;
  }
  __syncthreads();
  for (long long w = 0; w < nwaves; ++w) {
    const long long base = w * G;
    if (t < G) {
      int c = -1;                                  // no item in this slot
      if (base + t < items) {
        int k = cnt[base + t];
        k = k < 0 ? 0 : (k > cap ? cap : k);
        const int tiles = (k + 1) >> 1;
        c = tiles > 0 ? tiles + 2 : 1;
      }
      cost[t] = c;
    }
    __syncthreads();
    if (t < G) {                                   // rank of item t: cost descending, ties to the lower index
      const int c = cost[t];
      int r0 = 0, r1 = 0;
#pragma unroll 4
      for (int u4 = 0; u4 < G4; ++u4) {
        const int4 v = reinterpret_cast<const int4*>(cost)[u4];
        const int u = 4 * u4;
        r0 += (v.x > c) | ((v.x == c) & (u < t));
        r1 += (v.y > c) | ((v.y == c) & (u + 1 < t));
        r0 += (v.z > c) | ((v.z == c) & (u + 2 < t));
        r1 += (v.w > c) | ((v.w == c) & (u + 3 < t));
      }
      item_at[r0 + r1] = (int16_t)t;
    } else if (t >= kSchedMaxG && t - kSchedMaxG < G) {   // rank of CTA b: load ascending, ties to the lower index
      const int b = t - kSchedMaxG;
      const long long L = load[b];
      int r0 = 0, r1 = 0;
#pragma unroll 4
      for (int u2 = 0; u2 < G2; ++u2) {
        const longlong2 v = reinterpret_cast<const longlong2*>(load)[u2];
        const int u = 2 * u2;
        r0 += (v.x < L) | ((v.x == L) & (u < b));
        r1 += (v.y < L) | ((v.y == L) & (u + 1 < b));
      }
      cta_at[r0 + r1] = (int16_t)b;
    }
    __syncthreads();
    if (t < G) {
      const int i = item_at[t], b = cta_at[t];
      const int c = cost[i];
      out[w * G + b] = c >= 0 ? (int32_t)(base + i) : -1;
      if (c > 0) load[b] += c;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_sched(const int32_t* cnt_p, long long items, int cap, int P, int G, long long nwaves,
                         int32_t* sched, cudaStream_t st) {
  if (G < 1 || G > kSchedMaxG || P < 1 || nwaves * G < items) return cudaErrorInvalidValue;
  sched_kernel<<<(unsigned)P, 2 * kSchedMaxG, 0, st>>>(cnt_p, items, cap, G, nwaves, sched);
  return cudaGetLastError();
}

cudaError_t launch_exclusive(const int32_t* kv_idx, const int32_t* kv_cnt, int cap, const uint32_t* bits,
                             const int32_t* pairs, long long BH, int nb, int32_t* x_idx, int xcap, int32_t* x_cnt,
                             cudaStream_t st) {
  const int npairs = (nb + 1) / 2;
  const long long items = BH * npairs;
  exclusive_kernel<<<(unsigned)((items + kWarps - 1) / kWarps), 32 * kWarps, 0, st>>>(
      kv_idx, kv_cnt, cap, bits, pairs, BH, nb, npairs, x_idx, xcap, x_cnt);
  return cudaGetLastError();
}

cudaError_t launch_split_mask(const int32_t* kv_idx, const int32_t* kv_cnt, int cap, long long rows, int nb, int P,
                              int R, int32_t* idx_p, int32_t* cnt_p, cudaStream_t st) {
  if (P < 1 || P > 8) return cudaErrorInvalidValue;
  split_mask_kernel<<<(unsigned)((rows + kWarps - 1) / kWarps), 32 * kWarps, 0, st>>>(kv_idx, kv_cnt, cap, rows, nb,
                                                                                       P, R, idx_p, cnt_p);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* o_p, const float* lse_p, long long rows, int P, int d, void* out,
                           float* lse_out, cudaStream_t st) {
  const unsigned blocks = (unsigned)((rows + kWarps - 1) / kWarps);
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  if (d == 128) combine_kernel<128><<<blocks, 32 * kWarps, 0, st>>>(o_p, lse_p, rows, P, o, lse_out);
  else if (d == 64) combine_kernel<64><<<blocks, 32 * kWarps, 0, st>>>(o_p, lse_p, rows, P, o, lse_out);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace svsa
