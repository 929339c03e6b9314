// Block-sparse attention on the 5th-generation tensor cores, one softmax
// thread per query row (sm_100a).
//
// "SVG-EAR", problem statement: only the kept (query block, key block) pairs
// are computed; "SPADE" part 3: a per-head sparse engine built for the
// hardware.  Exact online-softmax attention over each 64-row query block's
// kept key blocks.
//
// Design:
//   * Work item = two query blocks I0, I1 of one head (128 query rows, the
//     M of a full-rate MMA; the blocks 2p, 2p + 1, or entries 2p, 2p + 1 of
//     a pairing table).  The item walks the ascending union of their kept
//     lists -- or, for the shared pass of the paired-block split, only
//     their intersection -- two key blocks (128 keys) per tile; a 64 x 64
//     quarter whose key block the row's own query block does not keep is
//     masked (and costs no exponentials).
//        S [128 q x 128 k]  = Q [128 x d] . K_pair^T        (A, B from smem, K-major)
//        O [128 q x d]     += P [128 x 64] . V_block [64 x d]   (one per key block)
//     with P in tensor memory (the A operand), V from smem (MN-major).
//   * The two key blocks of a tile are two independent halves: softmax
//     warpgroup h (warps 4-7 for the first block, 8-11 for the second)
//     keeps, for every row, its own running maximum, row sum and output
//     accumulator O_h in TMEM, and the halves are merged once per item by
//     the log-sum-exp rule.  Neither half waits for the other inside a tile.
//   * TMEM: two S buffers of 128 columns; half h writes its P as fp16 pairs
//     over the first 32 of its own 64 S columns; O_A, O_B (d columns each).
//   * Warp roles: warp 0 TMA of Q (once per item) and of the K tiles, warp 1
//     TMA of the V tiles, warp 2 issues the S products and owns TMEM, warp 3
//     issues the P.V products, warps 4-11 the two softmax warpgroups; thread
//     t of a group owns query row t (TMEM lane t) of its half.
//   * Softmax: the row maximum is thread-local.  The reference maximum m is
//     lazy: a tile only raises it when a score exceeds m by more than 2^12
//     (fp16 P then stays <= 2^12); raising it rescales the row sum and the
//     half's O row in TMEM, after that half's previous P.V product has
//     finished.  Otherwise exp2(x - m) is taken against the stale m, exact
//     up to the final normalisation.  Every decision that guards a TMEM
//     access or a warp sync is warp-uniform (tcgen05.ld / st are
//     warp-collective).
//   * Merge mode (m_in, lse_in): the epilogue also folds in a partial result
//     over other keys -- normalised fp32 rows and their log-sum-exp, as the
//     64-row kernel writes them for the paired-block split -- by the same
//     rule; an item with no tile copies that partial.
//   * Every role walks the same merged list itself, so no schedule is
//     stored; all hand-offs are mbarriers, every wait is bounded in time and
//     a timeout sets an error word read by svsa_sync_status; exits are agreed
//     by the two warps of a row at an OR-barrier.
//   * Compensation ("SVG-EAR" 2.A): after the union tiles an item walks
//     ceil(nb / 128) centroid tiles (128 block means as keys, value means as
//     values, 16-bit copies of the fp32 means); a row's centroid column J
//     gets the bias log2(n_J) when its own block skips J and is masked when
//     it keeps J.
//   * Counts and indices read from the mask are clamped to the tensors, so a
//     malformed list gives a wrong result, never an access outside them.
//
// This kernel serves the dense denominator (every key block, no list) and
// the shared pass of svsa_attn_fwd_paired; the sparse entry points use the
// 64-row kernel (attn_tc.cu), which is faster on sparse lists.
#include <climits>
#include <cstddef>

#include "tcgen05.cuh"

namespace svsa {
namespace fa {

using namespace tc;

constexpr int kThreads = 384;                 // 4 role warps + 2 softmax warpgroups
constexpr int kQBufs = 1, kKStages = 3, kVStages = 2, kSBufs = 2;
constexpr uint32_t kBox = 8192;                 // one 64-row x 128-byte TMA box
constexpr uint32_t kSlot = 32768;               // one 128-row tile (d = 128; d = 64 uses half)
constexpr float kLazyTh = 12.0f;                // log2 headroom before a rescale (fp16 P <= 2^12)

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQBufs * kSlot;
constexpr uint32_t kOffV = kOffK + kKStages * kSlot;
constexpr uint32_t kOffMisc = kOffV + kVStages * kSlot;
constexpr uint32_t kSmemBytes = kOffMisc + 4096 + 1024;     // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;                 // S buffers at 0, 128; O_A at 256, O_B at 256 + d

enum : uint32_t {
  BAR_Q_FULL = 0, BAR_Q_EMPTY = BAR_Q_FULL + kQBufs,
  BAR_K_FULL = BAR_Q_EMPTY + kQBufs, BAR_K_EMPTY = BAR_K_FULL + kKStages,
  BAR_V_FULL = BAR_K_EMPTY + kKStages, BAR_V_EMPTY = BAR_V_FULL + kVStages,
  BAR_S_FULL = BAR_V_EMPTY + kVStages, BAR_P_FULL = BAR_S_FULL + kSBufs,   // P_FULL: [2 halves][kSBufs]
  BAR_SP_FREE = BAR_P_FULL + 2 * kSBufs,
  BAR_O_FULL = BAR_SP_FREE + kSBufs, BAR_O_EMPTY, BAR_FINAL, BAR_FINAL2, NUM_BARS
};

struct Misc {
  uint64_t bar[NUM_BARS];
  uint32_t tmem_base;
  uint32_t abort;
  float xch[4 * 128];               // exchanged by the two threads of a row at the end of an item:
                                    // [m, l] of each half
};
static_assert(sizeof(Misc) <= 4096, "misc region");

struct Args {
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  const uint32_t* bits;    // kept-block bitmap rows (compensation only)
  int cap;
  int nwords;              // words per bitmap row
  int ncent;               // centroid tiles per item (0 = no compensation)
  __nv_bfloat16* o;
  float* o32;              // non-null: fp32 output (a key-range pass of a split launch) instead of bf16
  float* lse;
  float lse_empty;         // lse of a row with no kept key: 0, or -inf for a split pass
  long long N, Npad;
  int nb;
  int npairs;              // items per head: ceil(nb / 2)
  long long items;
  float scale_log2;
  int dense;
  const int32_t* pairs;    // nullable [BH, nb]: query blocks in item order (default: 0, 1, 2, ...)
  int inter_only;          // 1: walk only the key blocks both query blocks keep (their intersection)
  const float* m_in;       // nullable fp32 [BH * Npad, D]: a partial result over other keys (normalised) ...
  const float* lse_in;     // ... and its natural-log sum-exp, merged into this launch's rows
};

// The ascending union of the kept lists of the item's two query blocks,
// walked one key block at a time; flags bit 0 = kept by the first block,
// bit 1 = by the second.  Entries are clamped to [0, nb), counts to
// [0, cap].
struct Merge {
  const int32_t* la;
  const int32_t* lb;
  int na, nb2, ia, ib, ca, cb, nkb;
  bool dense, inter;
  __device__ __forceinline__ int load(const int32_t* l, int i, int n) const {
    if (i >= n) return INT_MAX;
    if (dense) return i;
    const int J = l[i];
    return J < 0 ? 0 : (J >= nkb ? nkb - 1 : J);
  }
  __device__ __forceinline__ void init(const Args& a, long long bh, int I0, int I1) {
    nkb = a.nb;
    dense = a.dense != 0;
    // (a block without a partner has an empty intersection: its whole list
    // goes to the 64-row pass)
    inter = a.inter_only != 0;
    const long long r0 = bh * a.nb + I0;
    if (dense) {
      na = a.nb;
      nb2 = I1 >= 0 ? a.nb : 0;
      la = lb = nullptr;
    } else {
      const int c0 = a.kv_cnt[r0];
      na = c0 < 0 ? 0 : (c0 > a.cap ? a.cap : c0);
      la = a.kv_idx + r0 * a.cap;
      if (I1 >= 0) {
        const long long r1 = bh * a.nb + I1;
        const int c1 = a.kv_cnt[r1];
        nb2 = c1 < 0 ? 0 : (c1 > a.cap ? a.cap : c1);
        lb = a.kv_idx + r1 * a.cap;
      } else {
        nb2 = 0;
        lb = la;
      }
    }
    ia = ib = 0;
    ca = load(la, 0, na);
    cb = load(lb, 0, nb2);
  }
  // next union element (-1 when both lists are exhausted); with `inter`, the
  // next element of the intersection
  __device__ __forceinline__ int next(uint32_t& fl) {
    while (true) {
      const int J = ca < cb ? ca : cb;
      if (J == INT_MAX) {
        fl = 0u;
        return -1;
      }
      fl = (ca == J ? 1u : 0u) | (cb == J ? 2u : 0u);
      if (ca == J) ca = load(la, ++ia, na);
      if (cb == J) cb = load(lb, ++ib, nb2);
      if (!inter || fl == 3u) return J;
    }
  }
};

// Item it = (head bh, entries 2p and 2p + 1 of the head's pairing order);
// the order is the identity without a pairing table.  Entries are clamped to
// [0, nb): a table that is not a permutation gives a wrong result (rows
// written twice or not at all), never an access outside the tensors.
__device__ __forceinline__ void item_blocks(const Args& a, long long it, long long& bh, int& I0, int& I1) {
  bh = it / a.npairs;
  const int p = (int)(it % a.npairs);
  I0 = 2 * p;
  I1 = 2 * p + 1 < a.nb ? 2 * p + 1 : -1;
  if (a.pairs != nullptr) {
    const int32_t* pt = a.pairs + bh * a.nb;
    const int x = pt[I0];
    I0 = x < 0 ? 0 : (x >= a.nb ? a.nb - 1 : x);
    if (I1 >= 0) {
      const int y = pt[I1];
      I1 = y < 0 ? 0 : (y >= a.nb ? a.nb - 1 : y);
    }
  }
}

// The tiles of one item, in the order every role walks them: the union
// tiles (two key blocks each; the second is -1 when the union has an odd
// count), then `ncent` centroid tiles.
struct Tiles {
  Merge m;
  int J1;            // first block of the next union tile, -1 when the union is done
  uint32_t f1;
  int cent, ncent;
  __device__ __forceinline__ void init(const Args& a, long long bh, int I0, int I1, int nc) {
    m.init(a, bh, I0, I1);
    J1 = m.next(f1);
    cent = 0;
    ncent = nc;
  }
  __device__ __forceinline__ bool empty() const { return J1 < 0 && ncent == 0; }
  // the next union tile only (false once the union is done)
  __device__ __forceinline__ bool next_union(int& j1, int& j2, uint32_t& fl1, uint32_t& fl2) {
    if (J1 < 0) return false;
    j1 = J1;
    fl1 = f1;
    j2 = m.next(fl2);
    J1 = j2 >= 0 ? m.next(f1) : -1;
    return true;
  }
  // false when the item is done; c = -1 for a union tile, else the centroid tile index
  __device__ __forceinline__ bool next(int& j1, int& j2, uint32_t& fl1, uint32_t& fl2, int& c) {
    if (J1 >= 0) {
      j1 = J1;
      fl1 = f1;
      j2 = m.next(fl2);
      J1 = j2 >= 0 ? m.next(f1) : -1;
      c = -1;
      return true;
    }
    if (cent < ncent) {
      c = cent++;
      j1 = j2 = -1;
      fl1 = fl2 = 0u;
      return true;
    }
    return false;
  }
};

// (a, b) = (a * x + c0, b * y + c1), one packed instruction
__device__ __forceinline__ void fma2v(float& a, float& b, float x, float y, float c0, float c1) {
  asm("{\n .reg .b64 p, m, c;\n mov.b64 p, {%0, %1};\n mov.b64 m, {%2, %3};\n mov.b64 c, {%4, %5};\n"
      " fma.rn.f32x2 p, p, m, c;\n mov.b64 {%0, %1}, p;\n}\n"
      : "+f"(a), "+f"(b) : "f"(x), "f"(y), "f"(c0), "f"(c1));
}

// 2^a, 2^b on the FMA pipe instead of the MUFU unit (Cody-Waite range
// reduction): y = j + f with j = round(y) and f in [-1/2, 1/2]; 2^f by a
// cubic fitted here by linear programming for the least maximum relative
// error on [-1/2, 1/2] with p(1/2) = 2 p(-1/2), so that neighbouring binades
// join (max relative error 7.5e-5, below fp16's half ulp); 2^j by adding j
// to the exponent field.  Adding 1.5 * 2^23 rounds y to an integer held in
// the low mantissa bits of the sum, and those bits shifted left by 23 are j
// in the exponent position.  Arguments below -126 give (nearly) 0.
__device__ __forceinline__ void exp2_fma2(float& a, float& b) {
  constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23
  constexpr float c0 = 0.9999280571937561f, c1 = 0.6932609677314758f, c2 = 0.2426111251115799f,
                  c3 = 0.0551716685295105f;
  a = fmaxf(a, -126.0f);
  b = fmaxf(b, -126.0f);
  float ta = a, tb = b;
  add2(ta, tb, kMagic, kMagic);
  float ja = ta, jb = tb;
  add2(ja, jb, -kMagic, -kMagic);
  float fa = a, fb = b;
  add2(fa, fb, -ja, -jb);
  float pa = c3, pb = c3;
  fma2v(pa, pb, fa, fb, c2, c2);
  fma2v(pa, pb, fa, fb, c1, c1);
  fma2v(pa, pb, fa, fb, c0, c0);
  a = __int_as_float(__float_as_int(pa) + (__float_as_int(ta) << 23));
  b = __int_as_float(__float_as_int(pb) + (__float_as_int(tb) << 23));
}

#ifndef SVSA_FA_POLY_EVERY
#define SVSA_FA_POLY_EVERY 0          // 0: every exponential on MUFU; n: one column pair in n on the FMA pipe
#endif

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
      "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// ---------------------------------------------------------------- the kernel
template <int D, bool COMP, bool O32>
__global__ void __launch_bounds__(kThreads, 1) attn_fa_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              const __grid_constant__ CUtensorMap tmC,
                                                              const Args a) {
  constexpr int NCH = D / 64;                    // 128-byte chunks of the head dim
  constexpr int KSTEPS = D / 16;
  constexpr uint32_t TILE_TX = 2 * NCH * kBox;   // bytes of one 128-row tile
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Misc* ms = reinterpret_cast<Misc*>(smem + kOffMisc);
  const uint32_t sbase = su32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile uint32_t* abort_flag = &ms->abort;
  auto bar = [&](int i) { return su32(&ms->bar[i]); };

  if (tid == 0) {
    for (int i = 0; i < kQBufs; ++i) {
      mbar_init(bar(BAR_Q_FULL + i), 1);
      mbar_init(bar(BAR_Q_EMPTY + i), 1);
    }
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(bar(BAR_K_FULL + i), 1);
      mbar_init(bar(BAR_K_EMPTY + i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(bar(BAR_V_FULL + i), 1);
      mbar_init(bar(BAR_V_EMPTY + i), 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(bar(BAR_S_FULL + i), 1);
      mbar_init(bar(BAR_P_FULL + i), 4);               // the first half's warpgroup
      mbar_init(bar(BAR_P_FULL + kSBufs + i), 4);      // the second half's
      mbar_init(bar(BAR_SP_FREE + i), 1);
    }
    mbar_init(bar(BAR_O_FULL), 1);
    mbar_init(bar(BAR_O_EMPTY), 8);
    mbar_init(bar(BAR_FINAL), 1);
    mbar_init(bar(BAR_FINAL2), 1);
    ms->abort = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&ms->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const long long items = a.items;
  const int nb = a.nb;
  const int ncent = COMP ? a.ncent : 0;

  if (warp == 0 || warp == 1) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: Q of each item (two 64-row blocks) and the K tiles; warp 1: the
    // V tiles.  Separate producers keep a K load from queueing behind a V
    // slot that only frees after the (later) second product of an older tile.
    if (lane == 0) {
      const bool is_k = warp == 0;
      uint32_t qit = 0, it_n = 0;
      bool ok = true;
      const int stages = is_k ? kKStages : kVStages;
      const uint32_t full0 = is_k ? BAR_K_FULL : BAR_V_FULL;
      const uint32_t empty0 = is_k ? BAR_K_EMPTY : BAR_V_EMPTY;
      const uint32_t region = is_k ? kOffK : kOffV;
      for (long long it = blockIdx.x; it < items && ok; it += gridDim.x) {
        long long bh;
        int I0, I1;
        item_blocks(a, it, bh, I0, I1);
        Tiles ti;
        ti.init(a, bh, I0, I1, ncent);
        if (ti.empty()) continue;
        if (is_k) {
          const uint32_t qs = qit % kQBufs;
          ok = wait_bar(bar(BAR_Q_EMPTY + qs), ((qit / kQBufs) & 1u) ^ 1u, abort_flag, 1);
          if (!ok) break;
          const int rq0 = (int)(bh * a.Npad + (long long)I0 * kBlock);
          const int rq1 = (int)(bh * a.Npad + (long long)(I1 >= 0 ? I1 : I0) * kBlock);
          mbar_expect_tx(bar(BAR_Q_FULL + qs), TILE_TX);
          for (int c = 0; c < NCH; ++c) {
            const uint32_t dst = sbase + kOffQ + qs * kSlot + c * 16384;
            tma_load_2d(dst, &tmQ, c * 64, rq0, bar(BAR_Q_FULL + qs));
            tma_load_2d(dst + kBox, &tmQ, c * 64, rq1, bar(BAR_Q_FULL + qs));
          }
          ++qit;
        }
        int j1, j2, cix;
        uint32_t fl1, fl2;
        while (ok && ti.next(j1, j2, fl1, fl2, cix)) {
          int r1, r2, x0;
          const CUtensorMap* tm;
          if (cix < 0) {
            r1 = (int)(bh * a.Npad + (long long)j1 * kBlock);
            r2 = (int)(bh * a.Npad + (long long)(j2 >= 0 ? j2 : j1) * kBlock);
            x0 = 0;
            tm = is_k ? &tmK : &tmV;
          } else {
            // 128 block means: bf16 key means in the first d columns of cbar,
            // fp16 value means in the last d (rows past this head's blocks
            // are masked by the softmax; past the tensor they read zeros)
            r1 = (int)(bh * nb + (long long)cix * 128);
            r2 = r1 + 64;
            x0 = is_k ? 0 : D;
            tm = &tmC;
          }
          const uint32_t stg = it_n % stages;
          ok = wait_bar(bar(empty0 + stg), ((it_n / stages) & 1u) ^ 1u, abort_flag, is_k ? 2 : 3);
          if (!ok) break;
          mbar_expect_tx(bar(full0 + stg), TILE_TX);
          for (int c = 0; c < NCH; ++c) {
            const uint32_t dst = sbase + region + stg * kSlot + c * 16384;
            tma_load_2d(dst, tm, x0 + c * 64, r1, bar(full0 + stg));
            tma_load_2d(dst + kBox, tm, x0 + c * 64, r2, bar(full0 + stg));
          }
          ++it_n;
        }
      }
      // never leave with copies in flight: wait (bounded) for the last fill of every stage
      volatile uint32_t no_abort = 0u;
      if (is_k)
        for (uint32_t j = 1; j <= (uint32_t)kQBufs && j <= qit; ++j) {
          const uint32_t n = qit - j;
          wait_bar(bar(BAR_Q_FULL + n % kQBufs), (n / kQBufs) & 1u, &no_abort, 20);
        }
      for (uint32_t j = 1; j <= (uint32_t)stages && j <= it_n; ++j) {
        const uint32_t n = it_n - j;
        wait_bar(bar(full0 + n % stages), (n / stages) & 1u, &no_abort, 21);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 2: S = Q . K_pair^T into the S ring, as far ahead as the P.V
    // products free S buffers; warp 3: O += P . V_pair with P read from the
    // first 64 columns of the tile's S buffer.  Each commits (hence waits
    // for) only its own MMAs.  Descriptors are base values plus compile-time
    // offsets (the 14-bit address field never carries).
    if (lane == 0) {
      const bool first_mma = warp == 2;
      constexpr uint32_t ID_S = idesc_f16(true, false, false, 128, 128);   // bf16 Q . K^T
      constexpr uint32_t ID_O = idesc_f16(false, false, true, D, 128);     // fp16 P . V, V MN-major
      const uint64_t dQ = sdesc(sbase + kOffQ, 16, 1024);
      const uint64_t dK = sdesc(sbase + kOffK, 16, 1024);
      const uint64_t dV = sdesc(sbase + kOffV, 16384, 1024);
      uint32_t ring = 0, j = 0, qit = 0, oit = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < items && ok; it += gridDim.x) {
        long long bh;
        int I0, I1;
        item_blocks(a, it, bh, I0, I1);
        Tiles ti;
        ti.init(a, bh, I0, I1, ncent);
        if (ti.empty()) continue;
        int j1, j2, cix;
        uint32_t fl1, fl2;
        if (first_mma) {
          const uint32_t qs = qit % kQBufs;
          ok = wait_bar(bar(BAR_Q_FULL + qs), (qit / kQBufs) & 1u, abort_flag, 4);
          ++qit;
          const uint64_t a0 = dQ + ((qs * kSlot) >> 4);
          while (ok && ti.next(j1, j2, fl1, fl2, cix)) {
            const uint32_t ks = ring % kKStages, sb = j % kSBufs;
            ok = wait_bar(bar(BAR_K_FULL + ks), (ring / kKStages) & 1u, abort_flag, 5) &&
                 wait_bar(bar(BAR_SP_FREE + sb), ((j / kSBufs) & 1u) ^ 1u, abort_flag, 6);
            if (!ok) break;
            tc_fence_after();
            const uint64_t b0 = dK + ((ks * kSlot) >> 4);
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
              const uint32_t off = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
              umma_f16(tmem + sb * 128, a0 + off, b0 + off, ID_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(BAR_K_EMPTY + ks));
            umma_commit(bar(BAR_S_FULL + sb));
            ++ring;
            ++j;
          }
          if (ok) umma_commit(bar(BAR_Q_EMPTY + qs));
        } else {
          int t = 0;
          while (ok && ti.next(j1, j2, fl1, fl2, cix)) {
            const uint32_t vs = ring % kVStages, sb = j % kSBufs;
            ok = wait_bar(bar(BAR_V_FULL + vs), (ring / kVStages) & 1u, abort_flag, 7) &&
                 (t > 0 || wait_bar(bar(BAR_O_EMPTY), (oit & 1u) ^ 1u, abort_flag, 9));
            const uint64_t b0 = dV + ((vs * kSlot) >> 4);
            // each half's keys (64) into that half's accumulator, as soon as its P is ready
#pragma unroll
            for (int h = 0; h < 2 && ok; ++h) {
              ok = wait_bar(bar(BAR_P_FULL + h * kSBufs + sb), (j / kSBufs) & 1u, abort_flag, 8);
              if (!ok) break;
              tc_fence_after();
              // (half h's P sits over the first 32 columns of its own 64 S columns)
#pragma unroll
              for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
                umma_f16_ts(tmem + kColO + h * D, tmem + sb * 128 + 64 * h + (kk - 4 * h) * 8,
                            b0 + ((kk * 2048) >> 4), ID_O, (t > 0 || kk > 4 * h) ? 1u : 0u);
            }
            if (!ok) break;
            umma_commit(bar(BAR_V_EMPTY + vs));
            umma_commit(bar(BAR_SP_FREE + sb));
            ++ring;
            ++j;
            ++t;
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
    // Query row `row` (0..127) is shared by two threads: warp 4 + q of the
    // first warpgroup takes the first key block of every tile (columns 0-63
    // of S, accumulator O_A), warp 8 + q of the second the second block
    // (columns 64-127, O_B), both on TMEM lane quadrant q.  Each half runs an
    // online softmax of its own -- reference maximum, row sum, accumulator --
    // so the two never synchronise inside an item; at the item's end the two
    // partial results are merged as O = (O_A 2^(m_A - m) + O_B 2^(m_B - m)) /
    // (l_A 2^(m_A - m) + l_B 2^(m_B - m)), m = max(m_A, m_B), the softmax over
    // the union of two disjoint key sets.  Rows 0-63 are block I0, rows
    // 64-127 block I1, so every validity decision is uniform across a warp.
    const int wq = warp & 3;                       // TMEM lane quadrant
    const int half = warp >= 8 ? 1 : 0;            // which key block of the tile, which accumulator
    const int row = wq * 32 + lane;
    const uint32_t mine = row < 64 ? 0u : 1u;      // bit of the union flags for this row's block
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t qbar = 1u + (uint32_t)wq;       // named barrier of the quadrant's two warps
    constexpr int DH = D / 2;                      // output columns this thread stores
    const uint32_t col_own = kColO + half * D;     // this half's accumulator
    const float sl2 = a.scale_log2;
    const int n_last = (int)(a.N - (long long)(nb - 1) * kBlock);   // valid keys of block nb - 1
    const float bias_last = __log2f((float)n_last);
    float* xch = ms->xch;                          // [m, l][2 halves][128 rows]
    uint32_t j = 0, oit = 0;
    bool stop = false;
    for (long long it = blockIdx.x; it < items && !stop; it += gridDim.x) {
      long long bh;
      int I0, I1;
      item_blocks(a, it, bh, I0, I1);
      const int Im = mine ? I1 : I0;
      const long long q = Im >= 0 ? (long long)Im * kBlock + (row & 63) : -1;
      const bool row_ok = q >= 0 && q < a.N;
      Tiles ti;
      ti.init(a, bh, I0, I1, ncent);
      if (ti.empty()) {
        // no tile: the incoming partial as it is (merge mode), else zero rows
        // (each thread its half of the columns)
        if (q >= 0) {
          const bool pin = a.m_in != nullptr && row_ok && a.lse_in[bh * a.Npad + q] > -INFINITY;
          const float* src = a.m_in != nullptr ? a.m_in + (bh * a.Npad + q) * D + half * DH : nullptr;
          if (O32) {
            float4* og = reinterpret_cast<float4*>(a.o32 + (bh * a.Npad + q) * D + half * DH);
            for (int i = 0; i < DH / 4; ++i)
              og[i] = pin ? reinterpret_cast<const float4*>(src)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
          } else {
            uint4* og = reinterpret_cast<uint4*>(a.o + (bh * a.Npad + q) * D + half * DH);
            for (int i = 0; i < DH / 8; ++i) {
              uint4 v = make_uint4(0u, 0u, 0u, 0u);
              if (pin) {
                const float4 f0 = reinterpret_cast<const float4*>(src)[2 * i];
                const float4 f1 = reinterpret_cast<const float4*>(src)[2 * i + 1];
                v = make_uint4(pack_bf16x2(f0.x, f0.y), pack_bf16x2(f0.z, f0.w), pack_bf16x2(f1.x, f1.y),
                               pack_bf16x2(f1.z, f1.w));
              }
              og[i] = v;
            }
          }
          if (a.lse != nullptr && half == 0) a.lse[bh * a.Npad + q] = pin ? a.lse_in[bh * a.Npad + q] : a.lse_empty;
        }
        continue;
      }
      // (the reference stays finite before the first valid score, so that a
      // fully masked tile gives exp2(-inf - 0) = 0, never -inf - (-inf))
      bool have_ref = false;
      float mref = 0.f, l = 0.f;
      // the union tiles, then (with compensation) the centroid tiles: the
      // phase loop is unrolled so that each phase's tile loop is compiled for
      // its own kind of tile and the union loop carries no centroid code
      int cnext = 0;
#pragma unroll
      for (int phase = 0; phase < (COMP ? 2 : 1); ++phase) {
        const bool cent = phase == 1;
        float s[64];
        while (true) {
          int j1 = -1, j2 = -1, cix = -1;
          uint32_t fl1 = 0u, fl2 = 0u;
          if (!cent) {
            if (!ti.next_union(j1, j2, fl1, fl2)) break;
          } else {
            if (cnext >= ncent) break;
            cix = cnext++;
          }
          const uint32_t sb = j % kSBufs;
          const int Jh = half ? j2 : j1;
          const uint32_t flh = half ? fl2 : fl1;
          // centroid tile: this row's block's kept bits for this half's 64 means
          uint32_t kw[2] = {0u, 0u};
          if (COMP && cent && Im >= 0) {
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const int word = cix * 4 + half * 2 + w;
              kw[w] = word < a.nwords ? a.bits[(bh * nb + Im) * a.nwords + word] : ~0u;
            }
          }
          // (every decision that guards a TMEM access or a warp sync is made
          // warp-uniform: tcgen05.ld / st are warp-collective)
          if (!__all_sync(0xffffffffu, wait_bar(bar(BAR_S_FULL + sb), (j / kSBufs) & 1u, abort_flag, 10))) {
            stop = true;
            break;
          }
          tc_fence_after();
          tmem_ld32(tmem + lane_off + sb * 128 + 64 * half, s);
          tmem_ld32(tmem + lane_off + sb * 128 + 64 * half + 32, s + 32);
          tmem_wait_ld();
          // scaled scores (log2 units) with masked columns at -inf, and their maximum
          float tmax = -INFINITY;
          bool cheap = false, dead = true;
          if (COMP && cent) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int J = cix * 128 + 64 * half + c;
              const bool ok_c = Im >= 0 && J < nb && ((kw[c >> 5] >> (c & 31)) & 1u) == 0u;
              const float bias = J == nb - 1 ? bias_last : 6.0f;        // log2 n_J
              s[c] = ok_c ? fmaf(s[c], sl2, bias) : -INFINITY;
              tmax = fmaxf(tmax, s[c]);
            }
            dead = false;
          } else if (Jh >= 0 && ((flh >> mine) & 1u) != 0u && Im >= 0) {
            dead = false;
            if (Jh != nb - 1 || n_last == kBlock) {
              cheap = true;
              float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
              for (int c = 0; c < 64; c += 8) {
                m0 = max3(m0, s[c], s[c + 1]);
                m1 = max3(m1, s[c + 2], s[c + 3]);
                m2 = max3(m2, s[c + 4], s[c + 5]);
                m3 = max3(m3, s[c + 6], s[c + 7]);
              }
              tmax = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * sl2;
            } else {
              // the ragged last block: keys past n_last are pads
#pragma unroll
              for (int c = 0; c < 64; ++c) {
                s[c] = c < n_last ? s[c] * sl2 : -INFINITY;
                tmax = fmaxf(tmax, s[c]);
              }
            }
          }
          // this half's reference maximum: set by its first tile with a valid
          // score, raised (with a rescale of its row sum and accumulator row)
          // only when a score exceeds it by more than 2^kLazyTh
          float alpha = 1.f;
          if (tmax > -INFINITY) {
            if (!have_ref) {
              mref = tmax;
              have_ref = true;
            } else if (tmax > mref + kLazyTh) {
              alpha = ex2(mref - tmax);
              l *= alpha;
              mref = tmax;
            }
          }
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
            // the warp rescales its rows of this half's accumulator (factor 1
            // where nothing changed) once the previous P.V products have
            // finished: the accumulator holds the previous tiles' sum then
            // (their slot barrier; the same item, since a raised reference
            // needs an earlier tile)
            const uint32_t jp = j - 1u, sp = jp % kSBufs;
            if (!__all_sync(0xffffffffu, wait_bar(bar(BAR_SP_FREE + sp), (jp / kSBufs) & 1u, abort_flag, 11))) {
              stop = true;
            } else {
              tc_fence_after();
#pragma unroll
              for (int c0 = 0; c0 < D; c0 += 32) {
                float o[32];
                tmem_ld32(tmem + lane_off + col_own + c0, o);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] *= alpha;
                tmem_st32(tmem + lane_off + col_own + c0, o);
              }
              tmem_wait_st();
            }
          }
          // P = exp2(y - m) as fp16 pairs over the first 32 of this half's own 64 S
          // columns (never over the other half's scores, which may not be read yet)
          uint32_t pk[32];
          float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
          const float nm = -mref;
          if (dead) {
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = 0u;
          } else if (cheap) {
            // packed fp32 pairs (sm_100 f32x2 instructions, each rounding as its scalar form)
            const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(nm, nm);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
              const float2 y01 = __ffma2_rn(make_float2(s[c], s[c + 1]), sc2, nm2);
              const float2 y23 = __ffma2_rn(make_float2(s[c + 2], s[c + 3]), sc2, nm2);
              float2 p01, p23;
              if (SVSA_FA_POLY_EVERY > 0 && (c >> 2) % (SVSA_FA_POLY_EVERY > 0 ? SVSA_FA_POLY_EVERY : 1) ==
                                                (SVSA_FA_POLY_EVERY > 0 ? SVSA_FA_POLY_EVERY - 1 : 0)) {
                p01 = y01;
                exp2_fma2(p01.x, p01.y);
              } else {
                p01 = make_float2(ex2(y01.x), ex2(y01.y));
              }
              p23 = make_float2(ex2(y23.x), ex2(y23.y));
              acc0 = __fadd2_rn(acc0, p01);
              acc1 = __fadd2_rn(acc1, p23);
              pk[c >> 1] = pack_f16x2(p01.x, p01.y);
              pk[(c >> 1) + 1] = pack_f16x2(p23.x, p23.y);
            }
            ls0 = acc0.x;
            ls1 = acc0.y;
            ls2 = acc1.x;
            ls3 = acc1.y;
          } else {
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float p0 = ex2(s[c] + nm), p1 = ex2(s[c + 1] + nm);
              add2(ls0, ls1, p0, p1);
              pk[c >> 1] = pack_f16x2(p0, p1);
            }
          }
          l += (ls0 + ls1) + (ls2 + ls3);
          tmem_st32u(tmem + lane_off + sb * 128 + 64 * half, pk);
          tmem_wait_st();
          // this half's P ready (and this warp's reads of S and any rescale complete)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_P_FULL + half * kSBufs + sb));
          ++j;
          if (stop) break;
        }
        if (stop) break;
      }

      // ---- epilogue: merge the two halves, normalise this thread's half of the columns, store
      // (every exit is agreed by the row's two warps at an OR-barrier both
      // reach, so neither waits at a named barrier the other has left)
      const bool ok_o = !stop && __all_sync(0xffffffffu, wait_bar(bar(BAR_O_FULL), oit & 1u, abort_flag, 13));
      xch[(0 + half) * 128 + row] = mref;
      xch[(2 + half) * 128 + row] = l;
      if (named_bar_or(qbar, 64, !ok_o)) {
        stop = true;
        break;
      }
      const float m_o = xch[(0 + (half ^ 1)) * 128 + row], l_o = xch[(2 + (half ^ 1)) * 128 + row];
      named_bar(qbar, 64);                          // both read before the next item writes the slots
      ++oit;
      tc_fence_after();
      const float mA = half ? m_o : mref, mB = half ? mref : m_o;
      const float lA = half ? l_o : l, lB = half ? l : l_o;
      // (a half with no valid key has l = 0 and takes no part)
      const float mx = fmaxf(lA > 0.f ? mA : -INFINITY, lB > 0.f ? mB : -INFINITY);
      const float sA = lA > 0.f ? ex2(mA - mx) : 0.f, sB = lB > 0.f ? ex2(mB - mx) : 0.f;
      const float lt = lA * sA + lB * sB;
      const float ln2 = 0.6931471805599453f, log2e = 1.4426950408889634f;
      // this launch's log2 sum-exp, and (merge mode) the incoming partial's:
      // out = (o_here 2^(L_here - L) + o_in 2^(L_in - L)) / (2^(L_here - L) + 2^(L_in - L))
      const float L2h = lt > 0.f ? mx + __log2f(lt) : -INFINITY;
      float L2i = -INFINITY;
      if (a.m_in != nullptr && q >= 0 && row_ok) L2i = a.lse_in[bh * a.Npad + q] * log2e;
      const float L2m = fmaxf(L2h, L2i);
      const float eh = L2h > -INFINITY ? ex2(L2h - L2m) : 0.f, ei = L2i > -INFINITY ? ex2(L2i - L2m) : 0.f;
      const float es = eh + ei;
      const float wh = es > 0.f ? eh / es : 0.f, wi = es > 0.f ? ei / es : 0.f;
      const float inv = lt > 0.f ? wh / lt : 0.f;
      const float wA = sA * inv, wB = sB * inv;
      const float* pin = (a.m_in != nullptr && q >= 0) ? a.m_in + (bh * a.Npad + q) * D + half * DH : nullptr;
      if (a.lse != nullptr && q >= 0 && half == 0)
        a.lse[bh * a.Npad + q] = (row_ok && es > 0.f) ? (L2m + __log2f(es)) * ln2 : a.lse_empty;
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 16) {
        float oa[16], ob[16];
        tmem_ld16(tmem + lane_off + kColO + half * DH + c0, oa);
        tmem_ld16(tmem + lane_off + kColO + D + half * DH + c0, ob);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) oa[c] = oa[c] * wA + ob[c] * wB;
        if (pin != nullptr && wi > 0.f) {
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const float4 f = reinterpret_cast<const float4*>(pin + c0 + c)[0];
            oa[c] = fmaf(f.x, wi, oa[c]);
            oa[c + 1] = fmaf(f.y, wi, oa[c + 1]);
            oa[c + 2] = fmaf(f.z, wi, oa[c + 2]);
            oa[c + 3] = fmaf(f.w, wi, oa[c + 3]);
          }
        }
        if (q >= 0) {
          if (O32) {
            float4* og = reinterpret_cast<float4*>(a.o32 + (bh * a.Npad + q) * D + half * DH + c0);
#pragma unroll
            for (int c = 0; c < 16; c += 4)
              og[c >> 2] = row_ok ? make_float4(oa[c], oa[c + 1], oa[c + 2], oa[c + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
          } else {
            uint4* og = reinterpret_cast<uint4*>(a.o + (bh * a.Npad + q) * D + half * DH + c0);
#pragma unroll
            for (int c = 0; c < 16; c += 8) {
              uint4 v;
              v.x = row_ok ? pack_bf16x2(oa[c], oa[c + 1]) : 0u;
              v.y = row_ok ? pack_bf16x2(oa[c + 2], oa[c + 3]) : 0u;
              v.z = row_ok ? pack_bf16x2(oa[c + 4], oa[c + 5]) : 0u;
              v.w = row_ok ? pack_bf16x2(oa[c + 6], oa[c + 7]) : 0u;
              og[c >> 3] = v;
            }
          }
        }
      }
      // the accumulators are free for the next item
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_O_EMPTY));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

}  // namespace fa

// ---------------------------------------------------------------- host side
namespace {

// 2D view [rows, d] of a 16-bit tensor, 64 x 64 boxes, 128-byte swizzle.
bool make_map_fa(CUtensorMap* m, const void* base, long long rows, int d, bool f16) {
  return tc::make_map_2d(m, base, rows, d, 64, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

}  // namespace

cudaError_t launch_attn_fa(const void* q, const void* k, const void* v, const int32_t* kv_idx,
                           const int32_t* kv_cnt, int cap, const uint32_t* bits, const void* cbar, void* o,
                           float* lse, long long BH, long long N, int nb, int d, bool dense, cudaStream_t st,
                           float* o32, float lse_empty, const int32_t* pairs, int inter_only, const float* m_in,
                           const float* lse_in) {
  CUtensorMap mq, mk, mv, mc;
  const long long rows = BH * (long long)nb * kBlock;
  if (!make_map_fa(&mq, q, rows, d, false) || !make_map_fa(&mk, k, rows, d, false) ||
      !make_map_fa(&mv, v, rows, d, true))
    return cudaErrorInvalidValue;
  // centroid rows [BH * nb, 2d]: bf16 key means, then fp16 value means (raw 16-bit copies)
  if (cbar != nullptr ? !make_map_fa(&mc, cbar, BH * (long long)nb, 2 * d, false) : !make_map_fa(&mc, k, rows, d, false))
    return cudaErrorInvalidValue;
  fa::Args a;
  a.kv_idx = kv_idx; a.kv_cnt = kv_cnt; a.cap = cap;
  a.bits = bits; a.nwords = (nb + 31) / 32;
  a.ncent = cbar != nullptr ? (nb + 127) / 128 : 0;
  a.o = (__nv_bfloat16*)o; a.lse = lse;
  a.o32 = o32; a.lse_empty = lse_empty;
  a.N = N; a.nb = nb; a.Npad = (long long)nb * kBlock;
  a.npairs = (nb + 1) / 2;
  a.items = BH * a.npairs;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  a.dense = dense ? 1 : 0;
  a.pairs = dense ? nullptr : pairs;
  a.inter_only = inter_only;
  a.m_in = m_in;
  a.lse_in = lse_in;
  const long long grid = std::min<long long>(a.items, tc::sm_count());
  const bool comp = a.ncent > 0;
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fa::kSmemBytes);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)grid, fa::kThreads, fa::kSmemBytes, st>>>(mq, mk, mv, mc, a);
    return cudaGetLastError();
  };
  const bool split = o32 != nullptr;
  if (d == 128) {
    if (split) return comp ? go(fa::attn_fa_kernel<128, true, true>) : go(fa::attn_fa_kernel<128, false, true>);
    return comp ? go(fa::attn_fa_kernel<128, true, false>) : go(fa::attn_fa_kernel<128, false, false>);
  }
  if (d == 64) {
    if (split) return comp ? go(fa::attn_fa_kernel<64, true, true>) : go(fa::attn_fa_kernel<64, false, true>);
    return comp ? go(fa::attn_fa_kernel<64, true, false>) : go(fa::attn_fa_kernel<64, false, false>);
  }
  return cudaErrorInvalidValue;
}

// Read and clear this kernel's device error word (0 = no failure).
cudaError_t attn_fa_error(unsigned int* code, cudaStream_t st) { return tc::read_error(code, st); }

}  // namespace svsa
