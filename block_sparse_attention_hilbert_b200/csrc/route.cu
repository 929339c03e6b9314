// Error-aware routing ratios ("SVG-EAR", technical summary 2.B) on the tensor
// cores.
//
// The query centroid qbar_I stands in for the queries of block I.  With
// s_j = qbar_I . k_j / sqrt(d) over all valid keys, M = max_j s_j and
// Z = sum_j e^{s_j - M}, block J's compensation error is
//   e_IJ = || sum_{j in J} e^{s_j - M} v_j - n_J e^{qbar_I . kbar_J / sqrt(d) - M} vbar_J ||_2
// (the change of the un-normalised proxy output when J's keys/values are
// replaced by their means) and the routed ratio is r_IJ = e_IJ / Z * 64 / n_J
// (error per unit of block size).
//
// Work item = 128 proxies (query blocks) of one head and a contiguous range
// of key blocks.  Per key block J (one 64-key tile):
//   S [128 x 64]  = Qbar . K_J^T   qbar split as bf16 hi + lo against the exact
//                                   bf16 keys (two MMA passes, ~16-bit qbar);
//   E = 2^(S log2e - m)             m = the proxy's running maximum, E <= 1;
//   O [128 x d]   = E . V_J         E split as fp16 hi + lo against the fp16
//                                   values (two MMA passes, ~22-bit weights);
//   e_IJ(m)       = || O_I - n_J 2^(L_IJ - m) vbar_J ||, stored with m,
// where L_IJ is the log2-domain centroid logit from the scores kernel.  The
// running maximum only grows, so each e_IJ is exact for the m it was taken
// against; per item the proxies' (m, Z) partials are stored and a fix-up
// kernel combines the key ranges and rescales: r_IJ = e_IJ 2^(m_IJ - M) / Z
// * 64 / n_J.
//
// Warp 0 issues the TMA copies of the qbar tile per item and of K_J per tile
// (3-stage ring, freed when S_J is done); warp 10 those of V_J (2-stage ring,
// freed when E.V_J is done) and the fp32 centroid value row vbar_J (4-deep
// ring, freed by the error epilogue).  Warp 1 issues the S MMAs and owns
// TMEM, warp 11 the E.V MMAs.  Two warpgroups hold one
// proxy per thread: warps 2-5 take the exponentials and the E split of every
// tile, warps 6-9 the error epilogue of the tiles whose E.V has finished, so
// the two run side by side on different tiles.  Every wait is bounded.
#include "tcgen05.cuh"

namespace svsa {
namespace tc {
namespace route {

constexpr int kThreads = 384;
constexpr int kRows = 128;                   // proxies per item
constexpr int kKStages = 3, kVStages = 2, kSBufs = 2, kEBufs = 2, kOBufs = 2, kVbBufs = 4, kMBufs = 4;
constexpr uint32_t kBoxQ = kRows * 128;      // 128 rows x 64 bf16 (16 KB)
constexpr uint32_t kBoxK = kBlock * 128;     // 64 rows x 64 elements (8 KB)
constexpr uint32_t kEPart = kRows * 128;     // E hi or lo: 128 proxies x 64 fp16 (16 KB)

template <int D>
struct Smem {
  static constexpr int NCH = D / 64;
  static constexpr uint32_t kQ = 2 * NCH * kBoxQ;          // qbar hi and lo
  static constexpr uint32_t kStage = NCH * kBoxK;          // one K_J or V_J tile
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kQ;
  static constexpr uint32_t kOffV = kOffK + kKStages * kStage;
  static constexpr uint32_t kOffE = kOffV + kVStages * kStage;
  static constexpr uint32_t kVb = D * 4;                      // one fp32 centroid value row
  static constexpr uint32_t kOffVb = kOffE + kEBufs * 2 * kEPart;
  static constexpr uint32_t kOffM = kOffVb + kVbBufs * kVb;     // per-tile maxima, kMBufs x kRows floats
  static constexpr uint32_t kOffMisc = kOffM + kMBufs * kRows * 4;
  static constexpr uint32_t kBytes = kOffMisc + 512 + 1024;
  static_assert(kBytes <= 232448, "shared memory per CTA");
  // TMEM: S buffers (64 columns each), then O buffers (D columns each)
  static constexpr uint32_t kColS = 0, kColO = kSBufs * 64;
  static constexpr uint32_t kCols = kColO + kOBufs * D <= 256 ? 256 : 512;
};

enum : uint32_t {
  BAR_Q_FULL = 0, BAR_Q_EMPTY, BAR_K_FULL, BAR_K_EMPTY = BAR_K_FULL + kKStages,
  BAR_V_FULL = BAR_K_EMPTY + kKStages, BAR_V_EMPTY = BAR_V_FULL + kVStages,
  BAR_S_FULL = BAR_V_EMPTY + kVStages, BAR_S_EMPTY = BAR_S_FULL + kSBufs,
  BAR_E_FULL = BAR_S_EMPTY + kSBufs, BAR_E_EMPTY = BAR_E_FULL + kEBufs,
  BAR_O_FULL = BAR_E_EMPTY + kEBufs, BAR_O_EMPTY = BAR_O_FULL + kOBufs,
  BAR_VB_FULL = BAR_O_EMPTY + kOBufs, BAR_VB_EMPTY = BAR_VB_FULL + kVbBufs,
  BAR_M_FULL = BAR_VB_EMPTY + kVbBufs, BAR_M_EMPTY = BAR_M_FULL + kMBufs, BAR_FINAL = BAR_M_EMPTY + kMBufs,
  BAR_FINAL2, NUM_BARS
};

struct Misc {
  uint64_t bar[NUM_BARS];
  uint32_t tmem_base;
  uint32_t abort;
};

struct Args {
  const float* L;       // [BH, nb, nb] centroid logits, log2 domain
  const float* vbar;    // [BH, nb, d]
  float* R;             // [BH, nb, nb] e_IJ against m_IJ
  float* Rm;            // [BH, nb, nb] m_IJ (log2 domain)
  float* Mp;            // [BH, nb, nsplit] partial maxima
  float* Zp;            // [BH, nb, nsplit] partial sums against Mp
  long long N, Npad;
  int nb, nqt, nsplit, per;   // proxy tiles per head, key ranges, key blocks per range
  long long items;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) route_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                               const __grid_constant__ CUtensorMap tmK,
                                                               const __grid_constant__ CUtensorMap tmV,
                                                               const Args a) {
  constexpr int NCH = D / 64;
  constexpr int KSTEPS = D / 16;
  using L = Smem<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Misc* ms = reinterpret_cast<Misc*>(smem + L::kOffMisc);
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
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(bar(BAR_S_FULL + i), 1);
      mbar_init(bar(BAR_S_EMPTY + i), 4);
    }
    for (int i = 0; i < kEBufs; ++i) {
      mbar_init(bar(BAR_E_FULL + i), 4);
      mbar_init(bar(BAR_E_EMPTY + i), 1);
    }
    for (int i = 0; i < kOBufs; ++i) {
      mbar_init(bar(BAR_O_FULL + i), 1);
      mbar_init(bar(BAR_O_EMPTY + i), 4);
    }
    for (int i = 0; i < kVbBufs; ++i) {
      mbar_init(bar(BAR_VB_FULL + i), 1);
      mbar_init(bar(BAR_VB_EMPTY + i), 4);
    }
    for (int i = 0; i < kMBufs; ++i) {
      mbar_init(bar(BAR_M_FULL + i), 4);
      mbar_init(bar(BAR_M_EMPTY + i), 4);
    }
    mbar_init(bar(BAR_FINAL), 1);
    mbar_init(bar(BAR_FINAL2), 1);
    ms->abort = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&ms->tmem_base)),
                 "r"(L::kCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const int nb = a.nb;
  // item -> (head, proxy tile, key range)
  auto decode = [&](long long it, long long& bh, int& qt, int& j0, int& j1) {
    const int sp = (int)(it % a.nsplit);
    const long long r = it / a.nsplit;
    qt = (int)(r % a.nqt);
    bh = r / a.nqt;
    j0 = sp * a.per;
    j1 = min(nb, j0 + a.per);
  };

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: the qbar tile of each item and K_J per tile (freed when S_J is
    // done); warp 10: V_J per tile (freed when E.V_J is done) and the fp32
    // centroid value row vbar_J (freed by the error epilogue).  Separate rings
    // let the K loads run ahead of the slower V turnover.
    if (lane == 0) {
      const bool is_k = warp == 0;
      uint32_t qit = 0, kn = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
        long long bh;
        int qt, j0, j1;
        decode(it, bh, qt, j0, j1);
        if (j0 >= j1) continue;
        if (is_k) {
          ok = wait_bar(bar(BAR_Q_EMPTY), (qit & 1u) ^ 1u, abort_flag, 51);
          if (!ok) break;
          mbar_expect_tx(bar(BAR_Q_FULL), L::kQ);
          const int yq = (int)(bh * nb + (long long)qt * kRows);
          for (int c = 0; c < 2 * NCH; ++c)
            tma_load_2d(sbase + L::kOffQ + c * kBoxQ, &tmQ, c * 64, yq, bar(BAR_Q_FULL));
          ++qit;
        }
        for (int J = j0; J < j1 && ok; ++J) {
          const int yk = (int)(bh * a.Npad + (long long)J * kBlock);
          if (is_k) {
            const uint32_t stg = kn % kKStages;
            ok = wait_bar(bar(BAR_K_EMPTY + stg), ((kn / kKStages) & 1u) ^ 1u, abort_flag, 52);
            if (!ok) break;
            mbar_expect_tx(bar(BAR_K_FULL + stg), L::kStage);
            for (int c = 0; c < NCH; ++c)
              tma_load_2d(sbase + L::kOffK + stg * L::kStage + c * kBoxK, &tmK, c * 64, yk, bar(BAR_K_FULL + stg));
          } else {
            const uint32_t stg = kn % kVStages;
            ok = wait_bar(bar(BAR_V_EMPTY + stg), ((kn / kVStages) & 1u) ^ 1u, abort_flag, 69);
            if (!ok) break;
            mbar_expect_tx(bar(BAR_V_FULL + stg), L::kStage);
            for (int c = 0; c < NCH; ++c)
              tma_load_2d(sbase + L::kOffV + stg * L::kStage + c * kBoxK, &tmV, c * 64, yk, bar(BAR_V_FULL + stg));
            const uint32_t vs = kn % kVbBufs;
            ok = wait_bar(bar(BAR_VB_EMPTY + vs), ((kn / kVbBufs) & 1u) ^ 1u, abort_flag, 64);
            if (!ok) break;
            mbar_expect_tx(bar(BAR_VB_FULL + vs), L::kVb);
            bulk_load(sbase + L::kOffVb + vs * L::kVb, a.vbar + (bh * nb + J) * (long long)D, L::kVb,
                      bar(BAR_VB_FULL + vs));
          }
          ++kn;
        }
      }
      // never leave with copies in flight: wait (bounded) for the last fill of every ring slot
      volatile uint32_t no_abort = 0u;
      if (qit > 0) wait_bar(bar(BAR_Q_FULL), (qit - 1) & 1u, &no_abort, 60);
      const uint32_t stages = is_k ? (uint32_t)kKStages : (uint32_t)kVStages;
      for (uint32_t j = 1; j <= stages && j <= kn; ++j) {
        const uint32_t n = kn - j;
        wait_bar(bar((is_k ? BAR_K_FULL : BAR_V_FULL) + n % stages), (n / stages) & 1u, &no_abort, 61);
      }
      if (!is_k)
        for (uint32_t j = 1; j <= (uint32_t)kVbBufs && j <= kn; ++j) {
          const uint32_t n = kn - j;
          wait_bar(bar(BAR_VB_FULL + n % kVbBufs), (n / kVbBufs) & 1u, &no_abort, 65);
        }
    }
  } else if (warp == 1 || warp == 11) {
    // ------------------------------------------------------------ MMA issuers
    // warp 1: S = Qbar . K_J^T of every tile (runs ahead as far as the S ring
    // allows); warp 11: O = E . V_J.  Two issuing threads keep the tensor core
    // fed, and each commits (hence waits for) only its own MMAs.
    if (lane == 0) {
      const bool s_issuer = warp == 1;
      constexpr uint32_t ID_S = idesc_f16(true, false, false, 64, kRows);     // bf16 Qbar . K^T
      constexpr uint32_t ID_O = idesc_f16(false, false, true, D, kRows);      // fp16 E . V (V MN-major)
      const uint64_t dQ = sdesc(sbase + L::kOffQ, 16, 1024);
      const uint64_t dK = sdesc(sbase + L::kOffK, 16, 1024);
      const uint64_t dVm = sdesc(sbase + L::kOffV, kBoxK, 1024);
      const uint64_t dE = sdesc(sbase + L::kOffE, 16, 1024);
      uint32_t qit = 0, n = 0;              // this issuer's next tile
      bool ok = true;
      auto issue_s = [&](uint32_t n) -> bool {
        const uint32_t stg = n % kKStages, sb = n % kSBufs;
        if (!wait_bar(bar(BAR_K_FULL + stg), (n / kKStages) & 1u, abort_flag, 53) ||
            !wait_bar(bar(BAR_S_EMPTY + sb), ((n / kSBufs) & 1u) ^ 1u, abort_flag, 54))
          return false;
        tc_fence_after();
        const uint64_t k0 = dK + ((stg * L::kStage) >> 4);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk)
            umma_f16(tmem + L::kColS + sb * 64, dQ + ((((part * NCH) + (kk >> 2)) * kBoxQ + (kk & 3) * 32) >> 4),
                     k0 + ((((kk >> 2)) * kBoxK + (kk & 3) * 32) >> 4), ID_S, (part > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(BAR_K_EMPTY + stg));
        umma_commit(bar(BAR_S_FULL + sb));
        return true;
      };
      auto issue_o = [&](uint32_t n) -> bool {
        const uint32_t stg = n % kVStages, eb = n % kEBufs, ob = n % kOBufs;
        if (!wait_bar(bar(BAR_V_FULL + stg), (n / kVStages) & 1u, abort_flag, 70) ||
            !wait_bar(bar(BAR_E_FULL + eb), (n / kEBufs) & 1u, abort_flag, 55) ||
            !wait_bar(bar(BAR_O_EMPTY + ob), ((n / kOBufs) & 1u) ^ 1u, abort_flag, 56))
          return false;
        tc_fence_after();
        const uint64_t v0 = dVm + ((stg * L::kStage) >> 4);
        const uint64_t e0 = dE + ((eb * 2 * kEPart) >> 4);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + L::kColO + ob * D, e0 + ((part * kEPart + kk * 32) >> 4), v0 + ((kk * 2048) >> 4), ID_O,
                     (part > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(BAR_V_EMPTY + stg));
        umma_commit(bar(BAR_E_EMPTY + eb));
        umma_commit(bar(BAR_O_FULL + ob));
        return true;
      };
      for (long long it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
        long long bh;
        int qt, j0, j1;
        decode(it, bh, qt, j0, j1);
        if (j0 >= j1) continue;
        if (s_issuer) {
          ok = wait_bar(bar(BAR_Q_FULL), qit & 1u, abort_flag, 57);
          ++qit;
        }
        for (int J = j0; J < j1 && ok; ++J) {
          ok = s_issuer ? issue_s(n) : issue_o(n);
          ++n;
        }
        if (s_issuer && ok) umma_commit(bar(BAR_Q_EMPTY));   // the item's S products have read qbar
      }
      // every MMA this thread issued has finished before TMEM is released
      const uint32_t fin = s_issuer ? BAR_FINAL : BAR_FINAL2;
      umma_commit(bar(fin));
      volatile uint32_t no_abort = 0u;
      wait_bar(bar(fin), 0u, &no_abort, 62);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ proxies: exponentials
    // One proxy per thread (warps 2-5): the tile's exponentials against the
    // running maximum, the E split into shared memory, and the maximum used
    // for the tile into the M ring for the error warps.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    const int n_in_last = (int)(a.N - (long long)(nb - 1) * kBlock);
    // this thread's E row in the K-major 128-byte-swizzled layout
    unsigned char* const erow0 = smem + L::kOffE + (row >> 3) * 1024 + (row & 7) * 128;
    float* const mring = reinterpret_cast<float*>(smem + L::kOffM);
    uint32_t sn = 0;
    bool stop = false;
    for (long long it = blockIdx.x; it < a.items && !stop; it += gridDim.x) {
      long long bh;
      int qt, j0, j1;
      decode(it, bh, qt, j0, j1);
      const int I = qt * kRows + row;
      const bool row_ok = I < nb;
      if (j0 >= j1) {
        // an empty key range contributes nothing to the proxy's max and sum
        if (row_ok) {
          const long long p = (bh * nb + I) * (long long)a.nsplit + it % a.nsplit;
          a.Mp[p] = -INFINITY;
          a.Zp[p] = 0.f;
        }
        continue;
      }
      float m = -INFINITY, Z = 0.f;
      for (int J = j0; J < j1; ++J) {
        const uint32_t sb = sn % kSBufs, eb = sn % kEBufs, mb = sn % kMBufs;
        if (!wait_bar(bar(BAR_S_FULL + sb), (sn / kSBufs) & 1u, abort_flag, 59)) { stop = true; break; }
        tc_fence_after();
        float x[64];
        tmem_ld32(tmem + lane_off + L::kColS + sb * 64, x);
        tmem_ld32(tmem + lane_off + L::kColS + sb * 64 + 32, x + 32);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_S_EMPTY + sb));
        const int nval = J == nb - 1 ? n_in_last : kBlock;
        // short dependency chains (one warp per scheduler runs this): packed
        // scaling, a tree of 3-input maxima, four partial sums
#pragma unroll
        for (int c = 0; c < 64; c += 2) fma2(x[c], x[c + 1], sl2, 0.f, 0.f);
        if (nval < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= nval) x[c] = -INFINITY;
        }
        float t16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) t16[i] = max3(x[4 * i], x[4 * i + 1], fmaxf(x[4 * i + 2], x[4 * i + 3]));
#pragma unroll
        for (int i = 0; i < 5; ++i) t16[i] = max3(t16[3 * i], t16[3 * i + 1], t16[3 * i + 2]);
        const float tmax = max3(max3(t16[0], t16[1], t16[2]), max3(t16[3], t16[4], t16[15]), -INFINITY);
        const float mn = fmaxf(m, tmax);
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float e0 = ex2(x[c] - mn), e1 = ex2(x[c + 1] - mn);
          s4[(c >> 1) & 3] += e0 + e1;
          const __half2 h = __floats2half2_rn(e0, e1);
          const float2 hf = __half22float2(h);
          const __half2 l = __floats2half2_rn(e0 - hf.x, e1 - hf.y);
          hi[c / 2] = *reinterpret_cast<const uint32_t*>(&h);
          lo[c / 2] = *reinterpret_cast<const uint32_t*>(&l);
        }
        const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        Z = (m == -INFINITY ? 0.f : Z * ex2(m - mn)) + sum;
        m = mn;
        if (!wait_bar(bar(BAR_E_EMPTY + eb), ((sn / kEBufs) & 1u) ^ 1u, abort_flag, 63) ||
            !wait_bar(bar(BAR_M_EMPTY + mb), ((sn / kMBufs) & 1u) ^ 1u, abort_flag, 67)) {
          stop = true;
          break;
        }
        unsigned char* erow = erow0 + eb * 2 * kEPart;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t off = (uint32_t)((ch ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(erow + off) = make_uint4(hi[4 * ch], hi[4 * ch + 1], hi[4 * ch + 2], hi[4 * ch + 3]);
          *reinterpret_cast<uint4*>(erow + kEPart + off) =
              make_uint4(lo[4 * ch], lo[4 * ch + 1], lo[4 * ch + 2], lo[4 * ch + 3]);
        }
        mring[mb * kRows + row] = m;
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(BAR_E_FULL + eb));
          mbar_arrive(bar(BAR_M_FULL + mb));
        }
        ++sn;
      }
      if (stop) break;
      if (row_ok) {
        const long long p = (bh * nb + I) * (long long)a.nsplit + it % a.nsplit;
        a.Mp[p] = m;
        a.Zp[p] = Z;
      }
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ proxies: error epilogue
    // One proxy per thread (warps 6-9, same TMEM lane quadrants as 2-5): for
    // every tile, in the same order, e_IJ = || O_I - n_J 2^(L_IJ - m) vbar_J ||
    // against the maximum m the exponential warps used for that tile.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int n_in_last = (int)(a.N - (long long)(nb - 1) * kBlock);
    const float* const mring = reinterpret_cast<const float*>(smem + L::kOffM);
    uint32_t n = 0;
    bool stop = false;
    for (long long it = blockIdx.x; it < a.items && !stop; it += gridDim.x) {
      long long bh;
      int qt, j0, j1;
      decode(it, bh, qt, j0, j1);
      if (j0 >= j1) continue;
      const int I = qt * kRows + row;
      const bool row_ok = I < nb;
      const long long rbase = (bh * nb + (row_ok ? I : 0)) * (long long)nb;
      float L_next = row_ok ? __ldg(a.L + rbase + j0) : 0.f;     // centroid logits, one tile ahead
      for (int J = j0; J < j1; ++J) {
        const float LJ = L_next;
        if (J + 1 < j1) L_next = row_ok ? __ldg(a.L + rbase + J + 1) : 0.f;
        const uint32_t ob = n % kOBufs, vs = n % kVbBufs, mb = n % kMBufs;
        if (!wait_bar(bar(BAR_M_FULL + mb), (n / kMBufs) & 1u, abort_flag, 68) ||
            !wait_bar(bar(BAR_O_FULL + ob), (n / kOBufs) & 1u, abort_flag, 58) ||
            !wait_bar(bar(BAR_VB_FULL + vs), (n / kVbBufs) & 1u, abort_flag, 66)) {
          stop = true;
          break;
        }
        tc_fence_after();
        const float m_used = mring[mb * kRows + row];
        const int nJ = J == nb - 1 ? n_in_last : kBlock;
        const float cw = row_ok ? (float)nJ * ex2(LJ - m_used) : 0.f;
        const float4* vb = reinterpret_cast<const float4*>(smem + L::kOffVb + vs * L::kVb);
        float err2 = 0.f;
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          float o[32];
          tmem_ld32(tmem + lane_off + L::kColO + ob * D + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 v4 = vb[ch * 8 + c / 4];       // same address in every lane: broadcast
            const float d0 = fmaf(-cw, v4.x, o[c]), d1 = fmaf(-cw, v4.y, o[c + 1]);
            const float d2 = fmaf(-cw, v4.z, o[c + 2]), d3 = fmaf(-cw, v4.w, o[c + 3]);
            err2 = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, err2))));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(BAR_O_EMPTY + ob));
          mbar_arrive(bar(BAR_VB_EMPTY + vs));
          mbar_arrive(bar(BAR_M_EMPTY + mb));
        }
        if (row_ok) {
          a.R[rbase + J] = sqrtf(err2);
          a.Rm[rbase + J] = m_used;
        }
        ++n;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(L::kCols));
  }
}

// r_IJ = e_IJ 2^(m_IJ - M) / Z * 64 / n_J with M, Z combined over the key ranges.
__global__ void route_fixup_kernel(float* __restrict__ R, const float* __restrict__ Rm, const float* __restrict__ Mp,
                                   const float* __restrict__ Zp, long long N, int nb, int nsplit) {
  const long long rowi = blockIdx.x;                 // (bh, I)
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, Mp[rowi * nsplit + s]);
  float Z = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float mp = Mp[rowi * nsplit + s];
    if (mp > -INFINITY) Z += Zp[rowi * nsplit + s] * ex2(mp - M);
  }
  const float iz = Z > 0.f ? 1.f / Z : 0.f;
  for (int J = threadIdx.x; J < nb; J += blockDim.x) {
    const long long i = rowi * nb + J;
    const int nJ = (int)std::max<long long>(1, std::min<long long>(kBlock, N - (long long)J * kBlock));
    const float e = R[i];
    R[i] = e > 0.f ? e * ex2(Rm[i] - M) * iz * ((float)kBlock / (float)nJ) : 0.f;
  }
}

}  // namespace route
}  // namespace tc

// Key ranges per (head, proxy tile): 8 gives the persistent grid several
// items per SM on every configuration, at a small per-item cost.
int route_nsplit(int nb) { return std::max(1, std::min(nb, 8)); }

// qsplit_bf: bf16 [BH, nb, 2d] (hi | lo of each query block mean); kp bf16 and vp fp16 [BH, Npad, d];
// L: [BH, nb, nb] log2-domain centroid logits; R, Rm: [BH, nb, nb]; Mp, Zp: [BH, nb, nsplit].
cudaError_t launch_route(const void* qsplit_bf, const void* kp, const void* vp, const float* L, const float* vbar,
                         float* R, float* Rm, float* Mp, float* Zp, int nsplit, long long BH, long long N, int nb,
                         int d, cudaStream_t st) {
  using namespace tc::route;
  const long long Npad = (long long)nb * kBlock;
  CUtensorMap mq, mk, mv;
  if (!tc::make_map_2d(&mq, qsplit_bf, BH * nb, 2 * d, kRows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
      !tc::make_map_2d(&mk, kp, BH * Npad, d, 64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
      !tc::make_map_2d(&mv, vp, BH * Npad, d, 64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return cudaErrorInvalidValue;
  Args a;
  a.L = L; a.vbar = vbar; a.R = R; a.Rm = Rm; a.Mp = Mp; a.Zp = Zp;
  a.N = N; a.Npad = Npad; a.nb = nb;
  a.nqt = (nb + kRows - 1) / kRows;
  a.nsplit = nsplit;
  a.per = (nb + nsplit - 1) / nsplit;
  a.items = BH * a.nqt * nsplit;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  const long long grid = std::min<long long>(a.items, tc::sm_count());
  auto go = [&](auto kernel, uint32_t smem) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)grid, kThreads, smem, st>>>(mq, mk, mv, a);
    return cudaGetLastError();
  };
  cudaError_t e;
  if (d == 128) e = go(route_tc_kernel<128>, Smem<128>::kBytes);
  else if (d == 64) e = go(route_tc_kernel<64>, Smem<64>::kBytes);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  route_fixup_kernel<<<(unsigned)(BH * nb), 128, 0, st>>>(R, Rm, Mp, Zp, N, nb, nsplit);
  return cudaGetLastError();
}

cudaError_t route_tc_error(unsigned int* code, cudaStream_t st) { return tc::read_error(code, st); }

}  // namespace svsa
