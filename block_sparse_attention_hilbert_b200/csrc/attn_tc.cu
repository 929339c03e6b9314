// Block-sparse attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "SVG-EAR", problem statement: only the kept (query block, key block) pairs
// are computed; "SPADE" part 3: a per-head sparse engine built for the
// hardware.  Exact online-softmax attention over each 64-row query block's
// kept key blocks.
//
// Design (sm_100a):
//   * Work item = one 64-query block of one head; a persistent grid walks the
//     items.  Tiles are PAIRS of kept key blocks (128 keys), taken in list
//     order, so every MMA row does useful work whatever the mask looks like.
//   * Transposed products keep M = 128 on the tensor core although the mask
//     granularity is 64 queries:
//        S^T [128 keys x 64 queries] = K_pair [128 x d] . Q^T      (A, B: K-major)
//        O^T [d x 64 queries]       += V_pair^T [d x 128] . P^T    (A, B: MN-major)
//     Both accumulate in TMEM (S^T in a 3-deep ring, O^T resident).
//   * Warp roles: warp 0 issues the TMA copies of Q (once per item) and of
//     the K pairs, warp 2 those of the V pairs (separate 2-stage rings, 64-row
//     boxes, 128-byte swizzle); warp 1 issues the S^T MMAs and owns the TMEM
//     allocation, warp 3 the O^T MMAs; warps 4-19 are four softmax warpgroups,
//     one thread per key / head-dim lane, 16 query columns per group.  All
//     hand-offs are mbarriers; every wait is bounded in time and a timeout
//     sets an error word read by svsa_sync_status.
//   * Softmax: thread k holds key k's scores for its group's 16 columns.  A
//     column (query) maximum needs all 128 threads, so the running maximum is
//     lazy: a tile only updates it (a group vote, a warp transpose-reduction
//     + shared memory, then an in-TMEM rescale of O^T and of the partial
//     sums) when some score exceeds the current reference by more than 2^12;
//     otherwise exp2(x - m) is taken against the stale reference, which is
//     exact up to the final normalisation.  The exponentials are computed
//     before the vote, so the wait for the slowest warp overlaps them.  The
//     row sums stay per-thread partial sums until the epilogue.
//   * Compensation ("SVG-EAR" 2.A): after the kept pairs, an item walks
//     ceil(nb / 128) centroid tiles -- 128 key-block means as keys and value
//     means as values (16-bit copies of the fp32 means) -- through the same
//     two products.  The softmax gives centroid row J the bias log2(n_J)
//     (n_J identical keys) when block J is skipped and -inf when it is kept,
//     so the skipped blocks enter the same softmax as the exact ones.
//   * P^T is rounded to fp16 and written to shared memory in the MN-major
//     128-byte-swizzled layout the second MMA reads; the values arrive as
//     fp16 (the reordered V), so the second product is fp16 x fp16.  With the
//     lazy maximum the weights reach 2^12 and the dominant one is no longer
//     exactly 1, so fp16's 11-bit significand (vs bf16's 8) is what keeps
//     their rounding well inside the output tolerance.
#include <cstddef>

#include "tcgen05.cuh"

namespace svsa {
namespace tc {

#ifndef SVSA_TC_GROUPS
#define SVSA_TC_GROUPS 4
#endif
// warp 0 Q/K TMA, 1 S-MMA (and TMEM owner), 2 V TMA, 3 O-MMA, 4.. softmax warpgroups
constexpr int kGroups = SVSA_TC_GROUPS;          // softmax warpgroups; each owns 64 / kGroups query columns
constexpr int kCols = 64 / kGroups;
constexpr int kThreads = 32 * (4 + 4 * kGroups);
#ifndef SVSA_TC_KSTAGES
#define SVSA_TC_KSTAGES 2
#endif
#ifndef SVSA_TC_PBUFS
#define SVSA_TC_PBUFS 3
#endif
constexpr int kKStages = SVSA_TC_KSTAGES, kVStages = 2, kSBufs = SVSA_TC_PBUFS, kPBufs = SVSA_TC_PBUFS;
constexpr int kSoftmaxThreads = 128;             // one softmax warpgroup
constexpr uint32_t kBox = 8192;                  // one 64-row x 128-byte TMA box
constexpr float kLazyTh = 12.0f;                 // log2 headroom before a rescale (fp16 P <= 2^12)

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                               // 2 x 8 KB (head-dim chunks)
constexpr uint32_t kOffK = 16384;                           // kKStages x 32 KB
constexpr uint32_t kOffV = kOffK + kKStages * 32768;        // kVStages x 32 KB
constexpr uint32_t kOffP = kOffV + kVStages * 32768;        // kPBufs x 16 KB
constexpr uint32_t kOffMisc = kOffP + kPBufs * 16384;
constexpr uint32_t kSmemBytes = kOffMisc + 2048 + 1024;     // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// TMEM columns: the S^T ring (64 columns a buffer), then O^T; the allocation
// is the next power of two
constexpr uint32_t kColS0 = 0, kColO = 64u * kSBufs;
constexpr uint32_t kTmemCols = kColO + 64u <= 256u ? 256u : 512u;
static_assert(kColO + 64u <= 512u, "TMEM columns");


enum : uint32_t {
  BAR_Q_FULL = 0, BAR_Q_EMPTY, BAR_K_FULL, BAR_K_EMPTY = BAR_K_FULL + kKStages,
  BAR_V_FULL = BAR_K_EMPTY + kKStages, BAR_V_EMPTY = BAR_V_FULL + kVStages,
  BAR_S_FULL = BAR_V_EMPTY + kVStages,
  BAR_P_FULL = BAR_S_FULL + kSBufs, BAR_P_EMPTY = BAR_P_FULL + kPBufs, BAR_O_FULL = BAR_P_EMPTY + kPBufs,
  BAR_O_EMPTY, BAR_FINAL, BAR_FINAL2, NUM_BARS
};

struct Misc {
  uint64_t bar[NUM_BARS];
  uint32_t tmem_base;
  uint32_t abort;
  alignas(16) float m[64];          // running maximum per query (log2 domain); read as float4
  alignas(16) float alpha[64];      // rescale factors of the current tile
  alignas(16) float fin[64];        // shift of this tile's scores, then 1 / row sum
  alignas(16) float red[kGroups][4][kCols];  // per-warp partial column results of each warpgroup
};
static_assert(offsetof(Misc, m) % 16 == 0 && offsetof(Misc, alpha) % 16 == 0, "float4 access");
static_assert(sizeof(Misc) <= 2048, "misc region");

struct Args {
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  const uint32_t* bits;   // kept-block bitmap rows (compensation only)
  int cap;
  int nwords;             // words per bitmap row
  int ncent;              // centroid tiles per item (0 = no compensation)
  __nv_bfloat16* o;
  float* o32;              // non-null: fp32 output (a key-range pass of a split launch) instead of bf16
  float* lse;
  float lse_empty;         // lse of a row with no kept key: 0, or -inf for a split pass
  long long N, Npad;
  int nb;
  long long items;
  float scale_log2;
  int dense;
  const int32_t* sched;    // nullable [nwaves][gridDim.x]: each wave's item per CTA (-1 = none)
  long long nwaves;
};

// The j-th item of this CTA: wave j's entry of the schedule (-1 = none in
// that wave), or without one item blockIdx.x + j * gridDim.x.  False once
// the CTA has no further wave.  Every role of the CTA walks the same
// sequence.
__device__ __forceinline__ bool cta_item(const Args& a, long long j, long long& it) {
  if (a.sched == nullptr) {
    it = (long long)blockIdx.x + j * gridDim.x;
    return it < a.items;
  }
  if (j >= a.nwaves) return false;
  const int v = a.sched[j * gridDim.x + blockIdx.x];
  it = (v >= 0 && (long long)v < a.items) ? v : -1;
  return true;
}

// Column reduction of v[0..NC-1] across the 32 lanes of a warp: halving
// exchanges over lane bits log2(NC)-1 .. 0 leave lane l with column l % NC
// summed over the lanes that share its upper bits; xor-shuffles over those
// upper bits finish the reduction (31 shuffles for NC = 32, 16 for NC = 16).
template <bool MAX, int NC>
__device__ __forceinline__ float warp_colreduce(float* v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = NC / 2; w >= 1; w >>= 1) {
    const bool hi = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float keep = hi ? v[i + w] : v[i];
      const float send = hi ? v[i] : v[i + w];
      const float other = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = MAX ? fmaxf(keep, other) : keep + other;
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = NC; o < 32; o <<= 1) {
    const float other = __shfl_xor_sync(0xffffffffu, r, o);
    r = MAX ? fmaxf(r, other) : r + other;
  }
  return r;
}

// ---------------------------------------------------------------- the kernel
template <int D, bool COMP, bool O32>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              const __grid_constant__ CUtensorMap tmC,
                                                              const Args a) {
  constexpr int NCH = D / 64;                    // 128-byte chunks of the head dim
  constexpr int KSTEPS = D / 16;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Misc* ms = reinterpret_cast<Misc*>(smem + kOffMisc);
  const uint32_t sbase = su32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile uint32_t* abort_flag = &ms->abort;
  auto bar = [&](int i) { return su32(&ms->bar[i]); };

  if (tid == 0) {
    mbar_init(bar(BAR_Q_FULL), 1);
    mbar_init(bar(BAR_Q_EMPTY), 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(bar(BAR_K_FULL + i), 1);
      mbar_init(bar(BAR_K_EMPTY + i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(bar(BAR_V_FULL + i), 1);
      mbar_init(bar(BAR_V_EMPTY + i), 1);
    }
    for (int i = 0; i < kSBufs; ++i) mbar_init(bar(BAR_S_FULL + i), 1);
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(bar(BAR_P_FULL + i), 4 * kGroups);
      mbar_init(bar(BAR_P_EMPTY + i), 1);
    }
    mbar_init(bar(BAR_O_FULL), 1);
    mbar_init(bar(BAR_O_EMPTY), 4 * kGroups);
    mbar_init(bar(BAR_FINAL), 1);
    mbar_init(bar(BAR_FINAL2), 1);
    ms->abort = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (D < 128) {
    // the second head-dim chunk of every V stage stays zero: the MMA reads a
    // 128-row V^T, rows d >= D contribute nothing
    for (int s = 0; s < kVStages; ++s)
      for (int i = tid; i < 16384 / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem + kOffV + s * 32768 + 16384)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_async_smem();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&ms->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const int nb = a.nb;
  const int ncent = COMP ? a.ncent : 0;          // centroid tiles per item

  auto item_count = [&](long long it) -> int {
    if (a.dense) return nb;
    const int c = a.kv_cnt[it];
    return c < 0 ? 0 : (c > a.cap ? a.cap : c);
  };
  auto item_block = [&](long long it, int j) -> int {
    if (a.dense) return j;
    const int J = a.kv_idx[it * a.cap + j];
    return J < 0 ? 0 : (J >= nb ? nb - 1 : J);
  };

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: Q of each item and the K pair tiles; warp 2: the V pair tiles.
    // Separate producers keep a K load from queueing behind a V slot that only
    // frees after the (later) second MMA of an older tile.
    if (lane == 0) {
      const bool is_k = warp == 0;
      uint32_t qit = 0, it_n = 0;
      bool ok = true;
      for (long long j = 0; ok; ++j) {
        long long it;
        if (!cta_item(a, j, it)) break;
        if (it < 0) continue;
        const int cnt = item_count(it);
        const int npairs = (cnt + 1) >> 1;
        const int ntiles = npairs + ncent;
        if (ntiles == 0) continue;
        const long long bh = it / nb;
        const int I = (int)(it % nb);
        if (is_k) {
          const int row_q = (int)(bh * a.Npad + (long long)I * kBlock);
          ok = wait_bar(bar(BAR_Q_EMPTY), (qit & 1u) ^ 1u, abort_flag, 1);
          if (!ok) break;
          mbar_expect_tx(bar(BAR_Q_FULL), NCH * kBox);
          for (int c = 0; c < NCH; ++c) tma_load_2d(sbase + kOffQ + c * kBox, &tmQ, c * 64, row_q, bar(BAR_Q_FULL));
          ++qit;
        }
        const int stages = is_k ? kKStages : kVStages;
        const uint32_t full0 = is_k ? BAR_K_FULL : BAR_V_FULL;
        const uint32_t empty0 = is_k ? BAR_K_EMPTY : BAR_V_EMPTY;
        const uint32_t region = is_k ? kOffK : kOffV;
        for (int t = 0; t < ntiles && ok; ++t) {
          // kept pairs first, then the centroid tiles (128 block means each;
          // rows past this head's nb blocks are masked by the softmax)
          const CUtensorMap* map = is_k ? &tmK : &tmV;
          int r1, r2, x0 = 0;
          if (!COMP || t < npairs) {
            const int J1 = item_block(it, 2 * t);
            const int J2 = (2 * t + 1 < cnt) ? item_block(it, 2 * t + 1) : J1;
            r1 = (int)(bh * a.Npad + (long long)J1 * kBlock);
            r2 = (int)(bh * a.Npad + (long long)J2 * kBlock);
          } else {
            map = &tmC;
            r1 = (int)(bh * nb + (long long)(t - npairs) * 128);
            r2 = r1 + 64;
            x0 = is_k ? 0 : D;
          }
          const uint32_t stg = it_n % stages;
          ok = wait_bar(bar(empty0 + stg), ((it_n / stages) & 1u) ^ 1u, abort_flag, is_k ? 2 : 3);
          if (!ok) break;
          mbar_expect_tx(bar(full0 + stg), 2 * NCH * kBox);
          for (int c = 0; c < NCH; ++c) {
            const uint32_t dst = sbase + region + stg * 32768 + c * 16384;
            tma_load_2d(dst, map, x0 + c * 64, r1, bar(full0 + stg));
            tma_load_2d(dst + kBox, map, x0 + c * 64, r2, bar(full0 + stg));
          }
          ++it_n;
        }
      }
      // never leave with copies in flight: wait (bounded) for the last fill of every stage
      volatile uint32_t no_abort = 0u;
      if (is_k && qit > 0) wait_bar(bar(BAR_Q_FULL), (qit - 1) & 1u, &no_abort, 20);
      const uint32_t stages = is_k ? kKStages : kVStages;
      for (uint32_t j = 1; j <= stages && j <= it_n; ++j) {
        const uint32_t n = it_n - j;
        wait_bar(bar((is_k ? BAR_K_FULL : BAR_V_FULL) + n % stages), (n / stages) & 1u, &no_abort, 21);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues the first product S^T = K_pair . Q^T of every tile into
    // the kSBufs-deep S ring (it runs ahead as far as the softmax frees S
    // buffers: the P hand-off of a slot also frees the S buffer of that slot,
    // whose scores the softmax has read by then, so one arrive per warp and
    // tile serves both rings); warp 3 issues the second product
    // O^T += V^T . P^T.  Two
    // issuing threads keep the tensor core fed, and each commits (hence
    // waits for) only its own MMAs.  Descriptors are base values plus
    // compile-time offsets (the 14-bit address field never carries).
    if (lane == 0) {
      const bool first_mma = warp == 1;
      constexpr uint32_t ID_S = idesc_f16(true, false, false);    // bf16 K . Q^T
      constexpr uint32_t ID_O = idesc_f16(false, true, true);     // fp16 V^T . P^T
      const uint64_t dK = sdesc(sbase + kOffK, 16, 1024);
      const uint64_t dQ = sdesc(sbase + kOffQ, 16, 1024);
      const uint64_t dV = sdesc(sbase + kOffV, 16384, 1024);
      const uint64_t dP = sdesc(sbase + kOffP, 16384, 1024);
      uint32_t ring = 0, tiles = 0, qit = 0, oit = 0;
      bool ok = true;
      for (long long j = 0; ok; ++j) {
        long long it;
        if (!cta_item(a, j, it)) break;
        if (it < 0) continue;
        const int cnt = item_count(it);
        const int npairs = ((cnt + 1) >> 1) + ncent;       // pair tiles, then centroid tiles
        if (npairs == 0) continue;
        if (first_mma) {
          ok = wait_bar(bar(BAR_Q_FULL), qit & 1u, abort_flag, 4);
          ++qit;
          for (int t = 0; t < npairs && ok; ++t) {
            const uint32_t ks = ring % kKStages, sb = tiles % kSBufs;
            ok = wait_bar(bar(BAR_K_FULL + ks), (ring / kKStages) & 1u, abort_flag, 5) &&
                 wait_bar(bar(BAR_P_FULL + sb), ((tiles / kSBufs) & 1u) ^ 1u, abort_flag, 6);
            if (!ok) break;
            tc_fence_after();
            const uint64_t a0 = dK + ((ks * 32768u) >> 4);
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk)
              umma_f16(tmem + kColS0 + sb * 64, a0 + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                       dQ + (((kk >> 2) * kBox + (kk & 3) * 32) >> 4), ID_S, kk > 0 ? 1u : 0u);
            umma_commit(bar(BAR_K_EMPTY + ks));
            umma_commit(bar(BAR_S_FULL + sb));
            ++ring;
            ++tiles;
          }
          if (ok) umma_commit(bar(BAR_Q_EMPTY));
        } else {
          for (int t = 0; t < npairs && ok; ++t) {
            const uint32_t vs = ring % kVStages, pb = tiles % kPBufs;
            ok = wait_bar(bar(BAR_V_FULL + vs), (ring / kVStages) & 1u, abort_flag, 7) &&
                 wait_bar(bar(BAR_P_FULL + pb), (tiles / kPBufs) & 1u, abort_flag, 8) &&
                 (t > 0 || wait_bar(bar(BAR_O_EMPTY), (oit & 1u) ^ 1u, abort_flag, 9));
            if (!ok) break;
            tc_fence_after();
            const uint64_t a0 = dV + ((vs * 32768u) >> 4);
            const uint64_t b0 = dP + ((pb * 16384u) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_f16(tmem + kColO, a0 + ((kk * 2048) >> 4), b0 + ((kk * 2048) >> 4), ID_O,
                       (t > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar(BAR_V_EMPTY + vs));
            umma_commit(bar(BAR_P_EMPTY + pb));
            ++ring;
            ++tiles;
          }
          if (ok) {
            umma_commit(bar(BAR_O_FULL));
            ++oit;
          }
        }
      }
      // every MMA this thread issued has finished before TMEM is released
      const uint32_t fin = first_mma ? BAR_FINAL : BAR_FINAL2;
      umma_commit(bar(fin));
      volatile uint32_t no_abort = 0u;
      wait_bar(bar(fin), 0u, &no_abort, 23);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // kGroups warpgroups (warps 4.., four consecutive warps each) split the
    // 64 query columns of every tile: each covers all 128 TMEM lanes (one key /
    // head-dim row per thread) for its own kCols columns, with its own running
    // maxima, rescales and partial sums, so groups never wait for each other.
    // Inside a group the 128 threads meet at their named barrier in lock
    // step; a failed wait only sets the abort flag, and the group leaves
    // together after an OR-reduction over that flag.
    const int wg = (warp - 4) >> 2;                // warpgroup
    const int sw = (warp - 4) & 3;                 // warp within the group
    const int quad = warp & 3;                     // TMEM lane quadrant of this warp
    const int k = quad * 32 + lane;                // key row (S^T) / head-dim row (O^T)
    const int st = sw * 32 + lane;                 // 0..127 within the group
    const uint32_t gbar = 1u + (uint32_t)wg;       // named barrier of this group
    const int cb = kCols * wg;                     // first query column of this group
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    float* mcol = ms->m + cb;
    float* acol = ms->alpha + cb;
    float* fcol = ms->fin + cb;
    // S and P rings have the same depth and advance together here: one slot
    // index and phase serve both
    static_assert(kSBufs == kPBufs, "S and P rings share the softmax slot counter");
    uint32_t sb = 0, sph = 0, oit = 0;
    // shared address of this thread's first 16-byte chunk of its P^T row (key
    // k) for the group's columns, 128-byte swizzle; the row starts on a
    // 128-byte boundary and the group's two chunks are 16-byte slots 2 wg and
    // 2 wg + 1 before the swizzle, so the second chunk is the first ^ 16
    static_assert(kCols == 16, "two 16-byte chunks of fp16 P per row and group");
    const uint32_t pa0 = sbase + kOffP + (uint32_t)((k >> 3) * 1024 + (k & 7) * 128) +
                         (uint32_t)(((2 * wg) ^ (k & 7)) << 4);
    bool stop = false;
    for (long long j = 0; !stop; ++j) {
      long long it;
      if (!cta_item(a, j, it)) break;
      if (it < 0) continue;
      const int cnt = item_count(it);
      const long long bh = it / nb;
      const int I = (int)(it % nb);
      const long long q0 = (long long)I * kBlock;
      __nv_bfloat16* og = a.o + (bh * a.Npad + q0 + cb) * D;       // this group's kCols rows
      constexpr int CPR = D / 8;
      const int npairs = (cnt + 1) >> 1;
      const int ntiles = npairs + ncent;
      if (ntiles == 0) {
        if (O32) {
          float* og32 = a.o32 + (bh * a.Npad + q0 + cb) * D;
          for (int i = st; i < kCols * D / 4; i += kSoftmaxThreads)
            reinterpret_cast<float4*>(og32)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          for (int i = st; i < kCols * CPR; i += kSoftmaxThreads)
            reinterpret_cast<uint4*>(og)[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (a.lse != nullptr && st < kCols) a.lse[bh * a.Npad + q0 + cb + st] = a.lse_empty;
        continue;
      }
      const int32_t* lst = a.dense ? nullptr : a.kv_idx + it * a.cap;
      const int n_in_last = (int)(a.N - (long long)(nb - 1) * kBlock);   // valid keys of block nb-1
      float lp[kCols], nmref[kCols];
#pragma unroll
      for (int c = 0; c < kCols; ++c) {
        lp[c] = 0.f;
        nmref[c] = 0.f;                            // negated reference maxima; set by the first tile
      }
      // this thread's key block for the current pair (prefetched one tile ahead)
      const int slot = k >> 6;
      auto block_at = [&](int j) -> int {
        if (j >= cnt) return -1;
        if (a.dense) return j;
        const int J = lst[j];
        return J < 0 ? 0 : (J >= nb ? nb - 1 : J);
      };

      // kept-pair tiles, then (with compensation) the centroid tiles; the
      // phase loop is unrolled so that each phase's tile loop is compiled for
      // its own kind of tile and the pair loop carries no centroid code
      bool badp = false;                           // the last P-ring wait failed
#pragma unroll
      for (int phase = 0; phase < (COMP ? 2 : 1); ++phase) {
        const bool cent = phase == 1;
        for (int t = cent ? npairs : 0; t < (cent ? ntiles : npairs); ++t) {
          // kept lists are ascending: only the last pair can hold block nb - 1
          // (ragged) or a missing second block, so only it needs the list entry
          const bool tail = !cent && t >= npairs - 1;
          const int jcur = tail ? block_at(2 * t + slot) : 0;
          // centroid tile: this thread's block J and its kept bit (read before the wait)
          const int Jc = (t - npairs) * 128 + k;
          uint32_t kept_word = ~0u;
          if (cent && Jc < nb) kept_word = a.bits[it * a.nwords + (Jc >> 5)];
          const bool bad = !wait_bar(bar(BAR_S_FULL + sb), sph, abort_flag, 10);
          tc_fence_after();
          const bool valid = cent ? ((kept_word >> (Jc & 31)) & 1u) == 0u
                                  : !tail || (jcur >= 0 && (jcur < nb - 1 || (k & 63) < n_in_last));
          const bool first = t == 0;
          const float bias = cent ? (Jc == nb - 1 ? __log2f((float)n_in_last) : 6.0f) : 0.f;
          // y = scaled score (log2 domain) minus the reference of its column; a
          // skipped block's centroid enters n_J times: + log2(n_J).  The S slot
          // is held until after the vote, so the rare rescale path reads it
          // again instead of keeping y live next to the exponentials.
          auto load_y = [&](float (&y)[kCols]) {
            tmem_ld_cols<kCols>(tmem + lane_off + kColS0 + sb * 64 + cb, y);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
              for (int c = 0; c < kCols; c += 2) {
                if (cent) fma2(y[c], y[c + 1], sl2, bias + nmref[c], bias + nmref[c + 1]);
                else fma2(y[c], y[c + 1], sl2, nmref[c], nmref[c + 1]);
              }
            } else {
#pragma unroll
              for (int c = 0; c < kCols; ++c) y[c] = -INFINITY;
            }
          };
          // exponentials against the current reference before the group vote, so
          // the wait for the slowest warp overlaps with this warp's MUFU work;
          // only a rescale tile (rare after the first) recomputes them
          float pv[kCols];
          float excess = -INFINITY;
          {
            float y[kCols];
            load_y(y);
#pragma unroll
            for (int c = 0; c < kCols; c += 2) excess = max3(excess, y[c], y[c + 1]);
#pragma unroll
            for (int c = 0; c < kCols; ++c) pv[c] = ex2(y[c]);
          }
          // (a failed wait of this thread, here or at the P ring of the previous
          // tile, takes the slow path, whose second vote sees the abort flag)
          if (named_bar_or(gbar, kSoftmaxThreads, first || bad || badp || excess > kLazyTh)) {
            if (named_bar_or(gbar, kSoftmaxThreads, *abort_flag != 0u)) {
              stop = true;
              break;
            }
            // exact column maxima of this tile (in y units), then a new reference
            float y[kCols];
            load_y(y);
            {
              float v[kCols];
#pragma unroll
              for (int c = 0; c < kCols; ++c) v[c] = y[c];
              const float r = warp_colreduce<true, kCols>(v);
              if (lane < kCols) ms->red[wg][sw][lane] = r;
            }
            named_bar(gbar, kSoftmaxThreads);
            if (st < kCols) {
              const float ty = fmaxf(fmaxf(ms->red[wg][0][st], ms->red[wg][1][st]),
                                     fmaxf(ms->red[wg][2][st], ms->red[wg][3][st]));
              const float m_used = first ? 0.f : mcol[st];
              // (a first tile with no valid key keeps the reference at 0)
              const float m_new = first ? (cent && ty == -INFINITY ? 0.f : ty) : fmaxf(mcol[st], ty + m_used);
              mcol[st] = m_new;
              acol[st] = first ? 0.f : ex2(m_used - m_new);
              fcol[st] = m_new - m_used;              // shift to apply to this tile's y
            }
            named_bar(gbar, kSoftmaxThreads);
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
              y[c] -= fcol[c];
              lp[c] *= acol[c];
              nmref[c] = -mcol[c];
              pv[c] = ex2(y[c]);
            }
            if (!first) {
              // O^T holds the previous tiles' sum once their MMA has finished
              // the previous tile used the previous slot of the P ring
              const uint32_t pprev = sb == 0u ? (uint32_t)kPBufs - 1u : sb - 1u;
              wait_bar(bar(BAR_P_EMPTY + pprev), sb == 0u ? sph ^ 1u : sph, abort_flag, 11);
              tc_fence_after();
              float o[kCols];
              tmem_ld_cols<kCols>(tmem + lane_off + kColO + cb, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < kCols; ++c) o[c] *= acol[c];
              tmem_st_cols<kCols>(tmem + lane_off + kColO + cb, o);
              tmem_wait_st();
            }
          }
          // P^T row k, this group's columns: exp2(y), fp16, 128-byte swizzled MN-major layout
          uint32_t pk[kCols / 2];
#pragma unroll
          for (int c = 0; c < kCols; c += 2) {
            add2(lp[c], lp[c + 1], pv[c], pv[c + 1]);
            pk[c >> 1] = pack_f16x2(pv[c], pv[c + 1]);
          }
          badp = !wait_bar(bar(BAR_P_EMPTY + sb), sph ^ 1u, abort_flag, 12);
          st_shared_v4(pa0 + sb * 16384u, pk[0], pk[1], pk[2], pk[3]);
          st_shared_v4((pa0 ^ 16u) + sb * 16384u, pk[4], pk[5], pk[6], pk[7]);
          fence_async_smem();
          // P tile ready, and the S slot free: this warp's TMEM reads of it
          // (and any rescale of O^T) are complete and ordered before the arrive
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_P_FULL + sb));
          // advance the S and P rings and their phase
          if (++sb == (uint32_t)kSBufs) { sb = 0u; sph ^= 1u; }
        }
        if (stop) break;
      }
      if (stop) break;

      // ---- epilogue: column sums, normalise O^T, store
      {
        const float r = warp_colreduce<false, kCols>(lp);
        if (lane < kCols) ms->red[wg][sw][lane] = r;
      }
      named_bar(gbar, kSoftmaxThreads);
      if (st < kCols) {
        const float l = ms->red[wg][0][st] + ms->red[wg][1][st] + ms->red[wg][2][st] + ms->red[wg][3][st];
        fcol[st] = l > 0.f ? 1.f / l : 0.f;
        if (a.lse != nullptr) {
          const float ln2 = 0.6931471805599453f;
          const long long q = q0 + cb + st;
          a.lse[bh * a.Npad + q] = (q < a.N && l > 0.f) ? (mcol[st] + __log2f(l)) * ln2 : a.lse_empty;
        }
      }
      wait_bar(bar(BAR_O_FULL), oit & 1u, abort_flag, 13);
      ++oit;
      tc_fence_after();
      named_bar(gbar, kSoftmaxThreads);
      {
        // thread k holds O^T[k][kCols queries]: row q of O gets element k; a
        // warp writes 64 contiguous bytes per query row
        float o[kCols];
        tmem_ld_cols<kCols>(tmem + lane_off + kColO + cb, o);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_O_EMPTY));
        if (k < D) {
          if (O32) {
            float* og32 = a.o32 + (bh * a.Npad + q0 + cb) * D;
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
              const bool row_ok = q0 + cb + c < a.N;
              og32[(long long)c * D + k] = row_ok ? o[c] * fcol[c] : 0.f;
            }
          } else {
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
              const bool row_ok = q0 + cb + c < a.N;
              og[(long long)c * D + k] = __float2bfloat16_rn(row_ok ? o[c] * fcol[c] : 0.f);
            }
          }
        }
      }
      stop = named_bar_or(gbar, kSoftmaxThreads, *abort_flag != 0u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

}  // namespace tc

// ---------------------------------------------------------------- host side
namespace {

// 2D view [rows, d] of a 16-bit tensor, 64 x 64 boxes, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, long long rows, int d, bool f16) {
  return tc::make_map_2d(m, base, rows, d, 64, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

}  // namespace

// Persistent grid of the 64-row kernel for `items` work items: one CTA per SM.
long long attn_tc_grid(long long items) { return std::min<long long>(items, tc::sm_count()); }

cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, const int32_t* kv_idx,
                           const int32_t* kv_cnt, int cap, const uint32_t* bits, const void* cbar, void* o,
                           float* lse, long long BH, long long N, int nb, int d, bool dense, cudaStream_t st,
                           float* o32, float lse_empty, const int32_t* sched, long long nwaves) {
  CUtensorMap mq, mk, mv, mc;
  const long long rows = BH * (long long)nb * kBlock;
  if (!make_map(&mq, q, rows, d, false) || !make_map(&mk, k, rows, d, false) || !make_map(&mv, v, rows, d, true))
    return cudaErrorInvalidValue;
  // centroid rows [BH * nb, 2d]: bf16 key means, then fp16 value means (raw 16-bit copies)
  if (cbar != nullptr ? !make_map(&mc, cbar, BH * (long long)nb, 2 * d, false) : !make_map(&mc, k, rows, d, false))
    return cudaErrorInvalidValue;
  tc::Args a;
  a.kv_idx = kv_idx; a.kv_cnt = kv_cnt; a.cap = cap;
  a.bits = bits; a.nwords = (nb + 31) / 32;
  a.ncent = cbar != nullptr ? (nb + 127) / 128 : 0;
  a.o = (__nv_bfloat16*)o; a.lse = lse;
  a.o32 = o32; a.lse_empty = lse_empty;
  a.N = N; a.nb = nb; a.Npad = (long long)nb * kBlock;
  a.items = BH * nb;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  a.dense = dense ? 1 : 0;
  const long long grid = attn_tc_grid(a.items);
  a.sched = sched;
  a.nwaves = nwaves;
  if (sched != nullptr && nwaves < (a.items + grid - 1) / grid) return cudaErrorInvalidValue;
  const bool comp = a.ncent > 0;
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kSmemBytes);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)grid, tc::kThreads, tc::kSmemBytes, st>>>(mq, mk, mv, mc, a);
    return cudaGetLastError();
  };
  const bool split = o32 != nullptr;
  if (d == 128) {
    if (split) return comp ? go(tc::attn_tc_kernel<128, true, true>) : go(tc::attn_tc_kernel<128, false, true>);
    return comp ? go(tc::attn_tc_kernel<128, true, false>) : go(tc::attn_tc_kernel<128, false, false>);
  }
  if (d == 64) {
    if (split) return comp ? go(tc::attn_tc_kernel<64, true, true>) : go(tc::attn_tc_kernel<64, false, true>);
    return comp ? go(tc::attn_tc_kernel<64, true, false>) : go(tc::attn_tc_kernel<64, false, false>);
  }
  return cudaErrorInvalidValue;
}

// Self-test of the failure path: one thread waits on a barrier that nothing
// arrives at, gives up after `budget_ns` and records site 90 in the error
// word, as every bounded wait of the kernels does.  No fault, no trap.
__global__ void selftest_wait_kernel(unsigned long long budget_ns) {
  __shared__ uint64_t b;
  const uint32_t bar = tc::su32(&b);
  tc::mbar_init(bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  const unsigned long long t0 = tc::gtimer();
  while (!tc::mbar_try_wait(bar, 0u)) {
    if (tc::gtimer() - t0 > budget_ns) {
      atomicCAS(&tc::g_tc_error, 0u, 90u);
      return;
    }
  }
}

cudaError_t launch_selftest_timeout(unsigned long long budget_ns, cudaStream_t st) {
  selftest_wait_kernel<<<1, 1, 0, st>>>(budget_ns);
  return cudaGetLastError();
}

// Read and clear this kernel's device error word (0 = no failure).
cudaError_t attn_tc_error(unsigned int* code, cudaStream_t st) { return tc::read_error(code, st); }

}  // namespace svsa
