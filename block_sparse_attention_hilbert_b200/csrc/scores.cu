// Pooled block scores S[bh, I, J] (fp32) on the tensor cores.
//
// SIZE = 64 ("DFSAttn" trick 2, block averages):
//   S_IJ = softmax_J(qbar_I . kbar_J / sqrt(d)) over all key blocks.
// SIZE = 16 (DFSAttn trick 2, sub-block scoring summed per block):
//   p_ij = softmax_j(qt_i . kt_j / sqrt(d)) over the non-empty key sub-blocks,
//   S_IJ = (1 / m_I) * sum_{i in I} sum_{j in J} p_ij over the m_I non-empty
//   query sub-blocks i of I.
//
// The selection needs the scores to ~1e-7, far below what one bf16 or fp16
// product gives, so each fp32 mean arrives split as fp16 hi + lo (the pooling
// kernel writes the split) and every logit is the fp32 accumulation of three
// fp16 products, hi.hi + hi.lo + lo.hi (the dropped lo.lo term and the
// rounding of lo are ~2^-22 of |q||k|).
//
// Work item = 128 pooled query rows of one head (M = 128); the pooled keys
// stream through in 128-row tiles (N = 128), twice: pass 1 keeps each row's
// running maximum and sum of exponentials, pass 2 recomputes the identical
// logits, normalises, and writes S (SIZE = 16: the 4 x 4 sub-pairs of each
// block pair are added first, columns in-thread and rows by warp shuffles).
// Warp 0 issues the TMA copies (Q tile once per item, K tiles into a 2-stage
// ring); the MMAs go into a 2-deep TMEM ring (warp 1 owns the allocation).
// SIZE = 16: warps 1 and 10 issue the MMAs of the even and the odd tiles,
// warps 2-5 and 6-9 hold one query row per thread for the first and the
// second 64 keys of every tile and merge their pass-1 maxima and sums once
// per item.  SIZE = 64: warp 1 issues every tile, warps 2-5 take whole tiles.
// Every wait is bounded.
//
// SIZE = 64 can also write the raw logits L_IJ = qbar_I . kbar_J / sqrt(d) *
// log2(e) (the centroid logits of the error-aware routing); with S = NULL
// the kernel makes that single pass only.
#include "tcgen05.cuh"

namespace svsa {
namespace tc {
namespace scores {

// Thread layout by sub-block size.  SIZE = 16 (many tiles per item): warps
// 0 TMA, 1 and 10 MMA, 2-5 and 6-9 the two key halves of every tile.
// SIZE = 64 (few items, short rows): warps 0 TMA, 1 MMA, 2-5 whole tiles.
template <int SIZE> struct Layout {
  static constexpr int kHalves = SIZE == 16 ? 2 : 1;
  static constexpr int kIssuers = kHalves;
  static constexpr int kRowThreads = 128 * kHalves;
  static constexpr int kThreads = 64 + kRowThreads + 32 * (kIssuers - 1);
};
constexpr uint32_t kMergeBar = 1;           // named barrier of the row warps
constexpr int kRows = 128;                  // pooled query rows per item
constexpr int kKeys = 128;                  // pooled keys per tile
constexpr int kKStages = 2, kSBufs = 2;
constexpr uint32_t kChunk = kRows * 128;    // 128 rows x 64 fp16 (one swizzled column chunk)
constexpr uint32_t kTmemCols = kSBufs * kKeys;

template <int D>
struct Smem {
  static constexpr int NCH = D / 64;
  static constexpr uint32_t kTile = 2 * NCH * kChunk;          // hi and lo chunks of 128 rows
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kTile;
  static constexpr uint32_t kOffMisc = kOffK + kKStages * kTile;
  static constexpr uint32_t kBytes = kOffMisc + 2560 + 1024;   // Misc + alignment slack
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

enum : uint32_t {
  BAR_Q_FULL = 0, BAR_Q_EMPTY, BAR_K_FULL, BAR_K_EMPTY = BAR_K_FULL + kKStages,
  BAR_S_FULL = BAR_K_EMPTY + kKStages, BAR_S_EMPTY = BAR_S_FULL + kSBufs, BAR_FINAL = BAR_S_EMPTY + kSBufs,
  BAR_FINAL2, NUM_BARS
};

struct Misc {
  uint64_t bar[NUM_BARS];
  uint32_t tmem_base;
  uint32_t abort;
  float pm[2][kRows], pl[2][kRows];          // pass-1 (max, sum) of each half, merged per item
};
static_assert(sizeof(Misc) <= 2560, "Misc fits its reservation");

struct Args {
  float* S;            // nullable: normalised scores
  float* L;            // nullable: raw log2-domain logits (SIZE = 64)
  int passes;          // 2 (scores), or 1 (logits only)
  long long N;
  int ng;              // pooled rows per head
  int nvc;             // non-empty pooled rows per head (the rest are padding)
  int nb;
  int nqt, nkt;        // query / key tiles per head
  long long items;
  float scale_log2;
};

template <int D, int SIZE>
__global__ void __launch_bounds__(Layout<SIZE>::kThreads, 1) scores_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                const __grid_constant__ CUtensorMap tmK,
                                                                const Args a) {
  constexpr int NCH = D / 64;
  constexpr int KSTEPS = D / 16;
  using L = Smem<D>;
  using Y = Layout<SIZE>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Misc* ms = reinterpret_cast<Misc*>(smem + L::kOffMisc);
  const uint32_t sbase = su32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile uint32_t* abort_flag = &ms->abort;
  auto bar = [&](int i) { return su32(&ms->bar[i]); };

  if (tid == 0) {
    mbar_init(bar(BAR_Q_FULL), 1);
    mbar_init(bar(BAR_Q_EMPTY), Y::kIssuers);      // every MMA issuer
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(bar(BAR_K_FULL + i), 1);
      mbar_init(bar(BAR_K_EMPTY + i), 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(bar(BAR_S_FULL + i), 1);
      mbar_init(bar(BAR_S_EMPTY + i), 4 * Y::kHalves);   // every row warp
    }
    mbar_init(bar(BAR_FINAL), 1);
    mbar_init(bar(BAR_FINAL2), 1);
    ms->abort = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
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
  const int ntiles = a.passes * a.nkt;            // one or two passes over the key tiles

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t qit = 0, kn = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
        const long long bh = it / a.nqt;
        const int qt = (int)(it % a.nqt);
        ok = wait_bar(bar(BAR_Q_EMPTY), (qit & 1u) ^ 1u, abort_flag, 31);
        if (!ok) break;
        mbar_expect_tx(bar(BAR_Q_FULL), L::kTile);
        const int yq = (int)(bh * a.ng + (long long)qt * kRows);
        for (int c = 0; c < 2 * NCH; ++c) tma_load_2d(sbase + L::kOffQ + c * kChunk, &tmQ, c * 64, yq, bar(BAR_Q_FULL));
        ++qit;
        for (int t = 0; t < ntiles && ok; ++t) {
          const int kt = t % a.nkt;
          const uint32_t stg = kn % kKStages;
          ok = wait_bar(bar(BAR_K_EMPTY + stg), ((kn / kKStages) & 1u) ^ 1u, abort_flag, 32);
          if (!ok) break;
          mbar_expect_tx(bar(BAR_K_FULL + stg), L::kTile);
          const int yk = (int)(bh * a.ng + (long long)kt * kKeys);
          for (int c = 0; c < 2 * NCH; ++c)
            tma_load_2d(sbase + L::kOffK + stg * L::kTile + c * kChunk, &tmK, c * 64, yk, bar(BAR_K_FULL + stg));
          ++kn;
        }
      }
      // never leave with copies in flight
      volatile uint32_t no_abort = 0u;
      if (qit > 0) wait_bar(bar(BAR_Q_FULL), (qit - 1) & 1u, &no_abort, 40);
      for (uint32_t j = 1; j <= (uint32_t)kKStages && j <= kn; ++j) {
        const uint32_t n = kn - j;
        wait_bar(bar(BAR_K_FULL + n % kKStages), (n / kKStages) & 1u, &no_abort, 41);
      }
    }
  } else if (warp == 1 || (Y::kIssuers == 2 && warp == 10)) {
    // ------------------------------------------------------------ MMA issuers
    // tile n (counted over this CTA's items) uses K stage and S buffer n % 2.
    // With two issuers warp 1 issues the even tiles and warp 10 the odd ones;
    // both wait for every item's Q tile and release it after their tiles.
    static_assert(kKStages == 2 && kSBufs == 2, "one K stage and one S buffer per issuer");
    if (lane == 0) {
      const uint32_t parity = warp == 1 ? 0u : 1u;
      const uint32_t stride_mask = Y::kIssuers == 2 ? 1u : 0u;   // tiles this issuer skips
      constexpr uint32_t ID = idesc_f16(false, false, false, kKeys, kRows);   // fp16, K-major A and B
      const uint64_t dQ = sdesc(sbase + L::kOffQ, 16, 1024);
      const uint64_t dK = sdesc(sbase + L::kOffK, 16, 1024);
      uint32_t qit = 0, n = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
        ok = wait_bar(bar(BAR_Q_FULL), qit & 1u, abort_flag, 33);
        ++qit;
        for (int t = 0; t < ntiles && ok; ++t, ++n) {
          if ((n & stride_mask) != parity) continue;
          const uint32_t ks = n & 1u, sb = n & 1u, ph = (n >> 1) & 1u;
          ok = wait_bar(bar(BAR_K_FULL + ks), ph, abort_flag, 34) &&
               wait_bar(bar(BAR_S_EMPTY + sb), ph ^ 1u, abort_flag, 35);
          if (!ok) break;
          tc_fence_after();
          const uint64_t k0 = dK + ((ks * L::kTile) >> 4);
          // chunk c of the hi part at c * kChunk, of the lo part at (NCH + c) * kChunk
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            const uint32_t qpart = term == 2 ? NCH : 0;      // hi.hi, hi.lo, lo.hi
            const uint32_t kpart = term == 1 ? NCH : 0;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
              const uint32_t off_in = (kk & 3) * 32;
              umma_f16(tmem + sb * kKeys, dQ + (((qpart + (kk >> 2)) * kChunk + off_in) >> 4),
                       k0 + (((kpart + (kk >> 2)) * kChunk + off_in) >> 4), ID, (term > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(bar(BAR_K_EMPTY + ks));
          umma_commit(bar(BAR_S_FULL + sb));
        }
        if (ok) umma_commit(bar(BAR_Q_EMPTY));
      }
      // every MMA this thread issued has finished before TMEM is released
      const uint32_t fin = parity == 0u ? BAR_FINAL : BAR_FINAL2;
      umma_commit(bar(fin));
      volatile uint32_t no_abort = 0u;
      wait_bar(bar(fin), 0u, &no_abort, 42);
    }
  } else {
    // ------------------------------------------------------------ one pooled query row per thread
    // warps 2-5 take keys 0-63 of every tile, warps 6-9 keys 64-127
    const int half = Y::kHalves == 2 && warp >= 6 ? 1 : 0;
    constexpr int kChunks = kKeys / 32 / Y::kHalves;   // 32-key chunks of a tile per warp
    const int quad = warp & 3;                      // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    uint32_t sn = 0;
    bool stop = false;
    for (long long it = blockIdx.x; it < a.items && !stop; it += gridDim.x) {
      const long long bh = it / a.nqt;
      const int qt = (int)(it % a.nqt);
      const int g = qt * kRows + row;               // pooled query row within the head
      const bool row_ok = g < a.nvc;
      float m = -INFINITY, l = 0.f, inv = 0.f;
      // SIZE = 16: block I = g / 4 and its non-empty sub-row count
      const int I = g / (kBlock / SIZE);
      float inv_m = 0.f;
      if (SIZE != kBlock) {
        const long long nval = std::max<long long>(0, std::min<long long>(kBlock, a.N - (long long)I * kBlock));
        const int m_sub = (int)((nval + SIZE - 1) / SIZE);
        inv_m = m_sub > 0 ? 1.f / (float)m_sub : 0.f;
      }
      const long long roff = (bh * a.nb + (I < a.nb ? I : 0)) * (long long)a.nb;   // row I of S / L
      float* srow = a.S != nullptr ? a.S + roff : nullptr;
      // a failed wait only marks the item: the warp keeps meeting the other
      // row warps at their barriers, and they all leave after the item's vote
      bool bad = false;
      for (int t = 0; t < ntiles; ++t, ++sn) {
        const uint32_t sb = sn % kSBufs;
        const bool pass2 = t >= a.nkt || a.passes == 1;
        if (a.passes == 2 && t == a.nkt) {
          if (Y::kHalves == 2) {
            // merge the two halves' running (max, sum) of pass 1
            ms->pm[half][row] = m;
            ms->pl[half][row] = l;
            named_bar(kMergeBar, Y::kRowThreads);
            const float m0 = ms->pm[0][row], m1 = ms->pm[1][row];
            const float l0 = ms->pl[0][row], l1 = ms->pl[1][row];
            m = fmaxf(m0, m1);
            l = m == -INFINITY ? 0.f
                               : (m0 == -INFINITY ? 0.f : l0 * ex2(m0 - m)) + (m1 == -INFINITY ? 0.f : l1 * ex2(m1 - m));
            named_bar(kMergeBar, Y::kRowThreads);    // both halves have read before the next item writes
          }
          inv = (row_ok && l > 0.f) ? 1.f / l : 0.f;
        }
        if (bad || !wait_bar(bar(BAR_S_FULL + sb), (sn / kSBufs) & 1u, abort_flag, 36)) {
          bad = true;
          continue;
        }
        tc_fence_after();
        const int kt = t >= a.nkt ? t - a.nkt : t;
        const int c0 = kt * kKeys;
#pragma unroll 1
        for (int ch = kChunks * half; ch < kChunks * half + kChunks; ++ch) {
          float x[32];
          tmem_ld32(tmem + lane_off + sb * kKeys + ch * 32, x);
          tmem_wait_ld();
          if (ch == kChunks * half + kChunks - 1) {
            // this half of the S tile is in registers: hand it back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_S_EMPTY + sb));
          }
          const int cb = c0 + ch * 32;              // first pooled key of this chunk
          const int nvalid = a.nvc - cb;            // keys >= nvc are padding
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = c < nvalid ? x[c] * sl2 : -INFINITY;
          if (!pass2) {
            float cm = x[0];
#pragma unroll
            for (int c = 1; c < 32; ++c) cm = fmaxf(cm, x[c]);
            const float mn = fmaxf(m, cm);
            if (mn > -INFINITY) {
              float sum = 0.f;
#pragma unroll
              for (int c = 0; c < 32; ++c) sum += ex2(x[c] - mn);
              l = (m == -INFINITY ? 0.f : l * ex2(m - mn)) + sum;
              m = mn;
            }
          } else if (SIZE == kBlock) {
            if (row_ok && I < a.nb) {
              if (a.L != nullptr) {
                float* lrow = a.L + roff;
#pragma unroll
                for (int c = 0; c < 32; ++c)
                  if (cb + c < a.nb) lrow[cb + c] = x[c];
              }
              if (a.S != nullptr) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                  const float p = ex2(x[c] - m) * inv;
                  if (cb + c < a.nb) srow[cb + c] = p;
                }
              }
            }
          } else {
            // 8 key blocks of 4 sub-columns each; then the 4 sub-rows of the block (lanes 4i .. 4i+3)
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              v[j] = 0.f;
#pragma unroll
              for (int u = 0; u < 4; ++u) v[j] += ex2(x[4 * j + u] - m);
              v[j] *= inv;
              v[j] += __shfl_xor_sync(0xffffffffu, v[j], 1);
              v[j] += __shfl_xor_sync(0xffffffffu, v[j], 2);
            }
            const int q = lane & 3;
            const int J0 = cb / 4 + 2 * q;
            if (I < a.nb) {
              const float w0 = q == 0 ? v[0] : q == 1 ? v[2] : q == 2 ? v[4] : v[6];
              const float w1 = q == 0 ? v[1] : q == 1 ? v[3] : q == 2 ? v[5] : v[7];
              if (J0 < a.nb) srow[J0] = w0 * inv_m;
              if (J0 + 1 < a.nb) srow[J0 + 1] = w1 * inv_m;
            }
          }
        }
      }
      stop = named_bar_or(kMergeBar, Y::kRowThreads, bad);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

}  // namespace scores
}  // namespace tc

// qsplit, ksplit: fp16 [BH, ng, 2d] (hi | lo of each pooled row), ng = Npad / size.
cudaError_t launch_scores(const void* qsplit, const void* ksplit, float* S, float* L, long long BH, long long N,
                          int ng, int nb, int d, int size, cudaStream_t st) {
  if (S == nullptr && (L == nullptr || size != kBlock)) return cudaErrorInvalidValue;
  using namespace tc::scores;
  CUtensorMap mq, mk;
  if (!tc::make_map_2d(&mq, qsplit, BH * ng, 2 * d, kRows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
      !tc::make_map_2d(&mk, ksplit, BH * ng, 2 * d, kKeys, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return cudaErrorInvalidValue;
  Args a;
  a.S = S;
  a.L = size == kBlock ? L : nullptr;
  a.passes = S != nullptr ? 2 : 1;
  a.N = N;
  a.ng = ng;
  a.nvc = (int)std::min<long long>(ng, (N + size - 1) / size);
  a.nb = nb;
  a.nqt = (ng + kRows - 1) / kRows;
  a.nkt = (ng + kKeys - 1) / kKeys;
  a.items = BH * a.nqt;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  const long long grid = std::min<long long>(a.items, tc::sm_count());
  auto go = [&](auto kernel, uint32_t smem, int threads) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)grid, threads, smem, st>>>(mq, mk, a);
    return cudaGetLastError();
  };
  if (d == 128 && size == 64) return go(scores_tc_kernel<128, 64>, Smem<128>::kBytes, Layout<64>::kThreads);
  if (d == 128 && size == 16) return go(scores_tc_kernel<128, 16>, Smem<128>::kBytes, Layout<16>::kThreads);
  if (d == 64 && size == 64) return go(scores_tc_kernel<64, 64>, Smem<64>::kBytes, Layout<64>::kThreads);
  if (d == 64 && size == 16) return go(scores_tc_kernel<64, 16>, Smem<64>::kBytes, Layout<16>::kThreads);
  return cudaErrorInvalidValue;
}

cudaError_t scores_tc_error(unsigned int* code, cudaStream_t st) { return tc::read_error(code, st); }

}  // namespace svsa
