// Semantic token order by bidirectional query-key co-clustering.
//
// "Training-Free Sparse Attention for Fast Video Generation via Offline
// Layer-Wise Sparsity Profiling and Online Bidirectional Co-Clustering"
// (SVOO), technical summary 2.B: alternate a query-aware partition of the keys
// (each key joins the query centroid it has the highest affinity with) and a
// key-aware partition of the queries (each query joins the updated key
// centroid of highest affinity); "SVG-EAR" 2.A: permute the tokens so that a
// cluster is contiguous in memory.  Per (batch, head), C = nb clusters,
// initial query centroids = the means of the raster 64-token blocks,
// affinity = the dot product, ties to the lower cluster index, an empty
// cluster takes the centroid it was matched against; the order sorts tokens
// by (cluster, raster index).
//
// Every argmax is decided on the exact affinity of a bf16 token and a float32
// centroid (the value an fp64 dot product gives):
//   * the tensor cores compute it with the centroid split exactly into three
//     bf16 parts (c = h + m + l: 8 + 8 + 8 significand bits) -- every product
//     is exact and only the fp32 accumulation of the 3d products rounds, by
//     at most 3d * 2^-20 * sum|x_c c_c| <= 3d * 2^-20 * |x| |c| (a bound with
//     a 16x margin over round-to-nearest, for the accumulator's alignment);
//   * a token whose best and second-best affinities lie within twice that
//     bound of each other is decided again in fp64: fp32 scores of every
//     centroid narrow it to those within twice the bound of the best, and
//     their fp64 dot products decide (every centroid's, when a lane's list of
//     its four best cannot hold them all).
// Centroids are the float32 rounding of fp64 sums of bf16 values.
#include "tcgen05.cuh"

namespace svsa {
namespace tc {
namespace clu {

// ---------------------------------------------------------------- small kernels
constexpr int kWarpsPerBlock = 8;

// |x| of every token row, rounded up by one part in 2^20 (an upper bound).
template <int D>
__global__ void norms_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ nrm, long long rows) {
  const long long r = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < D / 32; ++u) {
    const float v = __bfloat162float(x[r * D + lane + 32 * u]);
    s = fmaf(v, v, s);
  }
  s = warp_sum(s);
  if (lane == 0) nrm[r] = sqrtf(s) * (1.f + 9.5367431640625e-7f);
}

// Centroid j of head bh: the float32 mean of its member rows (fp64 sums),
// or the partner centroid when it has none.  Writes the float32 centroid,
// its three-way bf16 split [h | m | l] and raises the head's largest centroid
// norm (upper-rounded; non-negative floats order like their bit patterns).
// Members: order[bh, starts[j] + i] for i < counts[j]; with order == NULL the
// raster block j (tokens 64 j .. 64 j + 63 below N).
template <int D>
__global__ void means_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ order,
                             const int32_t* __restrict__ starts, const int32_t* __restrict__ counts,
                             const float* __restrict__ partner, float* __restrict__ cent,
                             __nv_bfloat16* __restrict__ cent3, unsigned int* __restrict__ cmax, long long BH,
                             long long N, int C) {
  const long long w = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= BH * C) return;
  const long long bh = w / C;
  const int j = (int)(w % C);
  int n, s0;
  if (order == nullptr) {
    s0 = j * kBlock;
    n = (int)std::max<long long>(0, std::min<long long>(kBlock, N - (long long)s0));
  } else {
    s0 = starts[w];
    n = counts[w];
  }
  constexpr int U = D / 32;
  double acc[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc[u] = 0.0;
  // members in order; four rows are loaded ahead of their (ordered) adds
  auto member = [&](int i) -> long long {
    return order == nullptr ? (long long)(s0 + i) : (long long)order[bh * N + s0 + i];
  };
  int i = 0;
  for (; i + 4 <= n; i += 4) {
    float r[4][U];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const __nv_bfloat16* row = x + (bh * N + member(i + m)) * D;
#pragma unroll
      for (int u = 0; u < U; ++u) r[m][u] = __bfloat162float(row[lane + 32 * u]);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int u = 0; u < U; ++u) acc[u] += (double)r[m][u];
  }
  for (; i < n; ++i) {
    const __nv_bfloat16* row = x + (bh * N + member(i)) * D;
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u] += (double)__bfloat162float(row[lane + 32 * u]);
  }
  float v[U];
#pragma unroll
  for (int u = 0; u < U; ++u)
    v[u] = n > 0 ? (float)(acc[u] / (double)n) : partner[w * D + lane + 32 * u];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = lane + 32 * u;
    cent[w * D + c] = v[u];
    const __nv_bfloat16 h = __float2bfloat16_rn(v[u]);
    const float r1 = v[u] - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
    cent3[w * 3 * D + c] = h;
    cent3[w * 3 * D + D + c] = m;
    cent3[w * 3 * D + 2 * D + c] = l;
    ss = fmaf(v[u], v[u], ss);
  }
  ss = warp_sum(ss);
  if (lane == 0) atomicMax(&cmax[bh], __float_as_uint(sqrtf(ss) * (1.f + 9.5367431640625e-7f)));
}

// The five largest values a lane has seen (t[0] >= ... >= t[4]) and the
// indices of the first four (-1 while empty).  Strict comparisons keep the
// earlier of equal values in front; insertion is branch-free and taken only
// by a value above t[4].
struct Top5 {
  float t[5] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
  int id[4] = {-1, -1, -1, -1};
  __device__ __forceinline__ void push(float x, int j) {
    if (!(x > t[4])) return;
    const bool c0 = x > t[0], c1 = x > t[1], c2 = x > t[2], c3 = x > t[3];
    t[4] = c3 ? t[3] : x;
    t[3] = c3 ? (c2 ? t[2] : x) : t[3];
    id[3] = c3 ? (c2 ? id[2] : j) : id[3];
    t[2] = c2 ? (c1 ? t[1] : x) : t[2];
    id[2] = c2 ? (c1 ? id[1] : j) : id[2];
    t[1] = c1 ? (c0 ? t[0] : x) : t[1];
    id[1] = c1 ? (c0 ? id[0] : j) : id[1];
    t[0] = c0 ? x : t[0];
    id[0] = c0 ? j : id[0];
  }
};

// Exact argmax for the tokens the tensor-core pass could not separate, first
// index on ties.  Per head, list[bh * N + i] (i < count[bh]) holds those
// tokens.  A warp takes kFixTok tokens of one head, so that every centroid row
// it loads serves kFixTok dot products; lanes split the head dimension
// (U = D / 32 consecutive values each).
//   1. fp32 scores s_j of every centroid, kFixCent centroids at a time: the
//      kFixCent x kFixTok partial sums of a lane go through a transpose-
//      reduction that leaves lane L with the full score of centroid
//      j0 + L / kFixTok for token L % kFixTok.  Each lane keeps the five best
//      it has seen (its token, every kFixCent-th centroid).  The fp32 error is
//      far below the tensor-core bound gamma |x| |c_j|.
//   2. With s1 a token's largest score and thr = 2 gamma |x| max|c|, its exact
//      maximum is among the centroids with s_j >= s1 - thr.  When no lane of
//      the token has a fifth value reaching that line, they are all in its
//      lanes' first four: fp64 dot products of just them decide.  Otherwise
//      every centroid is scored in fp64 for that token.
constexpr int kFixTok = 8, kFixCent = 32 / kFixTok;

template <int D>
__global__ void fix_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ cent,
                           const int32_t* __restrict__ list, const unsigned int* __restrict__ count,
                           const float* __restrict__ xnorm, const unsigned int* __restrict__ cmax, float gamma,
                           int32_t* __restrict__ assign, long long N, int C) {
  constexpr int U = D / 32;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int n = (int)count[bh];
  const int32_t* lst = list + bh * N;
  const float* ch = cent + bh * (long long)C * D;
  const int my = lane % kFixTok;                     // the token this lane scores
  for (int g = (blockIdx.x * kWarpsPerBlock + wid) * kFixTok; g < n; g += gridDim.x * kWarpsPerBlock * kFixTok) {
    // the group's tokens (a short last group repeats its last token)
    long long tk[kFixTok];
    float xf[kFixTok][U];
#pragma unroll
    for (int t = 0; t < kFixTok; ++t) {
      tk[t] = bh * N + lst[min(g + t, n - 1)];
#pragma unroll
      for (int u = 0; u < U; ++u) xf[t][u] = __bfloat162float(x[tk[t] * D + lane * U + u]);
    }
    // 1. fp32 scores, five best per lane
    Top5 top;
    for (int j0 = 0; j0 < C; j0 += kFixCent) {
      float acc[kFixCent * kFixTok];                 // [centroid c][token t] at c * kFixTok + t
#pragma unroll
      for (int c = 0; c < kFixCent; ++c) {
        float cv[U];
        if (j0 + c < C) {
#pragma unroll
          for (int u = 0; u < U; ++u) cv[u] = ch[(long long)(j0 + c) * D + lane * U + u];
        } else {
#pragma unroll
          for (int u = 0; u < U; ++u) cv[u] = 0.f;
        }
#pragma unroll
        for (int t = 0; t < kFixTok; ++t) {
          float v = 0.f;
#pragma unroll
          for (int u = 0; u < U; ++u) v = fmaf(xf[t][u], cv[u], v);
          acc[c * kFixTok + t] = v;
        }
      }
      // halving exchanges: lane L ends with the full sum of value L
#pragma unroll
      for (int w = 16; w >= 1; w >>= 1) {
        const bool hi = (lane & w) != 0;
#pragma unroll
        for (int c = 0; c < w; ++c) {
          const float keep = hi ? acc[c + w] : acc[c];
          const float send = hi ? acc[c] : acc[c + w];
          acc[c] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
      }
      const int j = j0 + lane / kFixTok;
      if (j < C) top.push(acc[0], j);
    }
    // per token (lanes my, my + kFixTok, ...): the largest score and the line
    float s1 = top.t[0];
#pragma unroll
    for (int o = kFixTok; o < 32; o <<= 1) s1 = fmaxf(s1, __shfl_xor_sync(0xffffffffu, s1, o));
    long long tok = tk[0];                           // this lane's token (static indices only)
#pragma unroll
    for (int t = 1; t < kFixTok; ++t) tok = my == t ? tk[t] : tok;
    const double line = (double)s1 - 2.0 * (double)gamma * (double)xnorm[tok] * (double)__uint_as_float(cmax[bh]);
    bool reach = (double)top.t[4] >= line;
#pragma unroll
    for (int o = kFixTok; o < 32; o <<= 1) reach |= __shfl_xor_sync(0xffffffffu, reach ? 1 : 0, o) != 0;
    // 2. token by token: fp64 dot products of the candidates (or of all centroids)
#pragma unroll 1
    for (int t = 0; t < kFixTok && g + t < n; ++t) {
      const long long tt = bh * N + lst[g + t];     // (reloaded: no dynamic index into registers)
      double xv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) xv[u] = (double)__bfloat162float(x[tt * D + lane * U + u]);
      const bool full = __shfl_sync(0xffffffffu, reach ? 1 : 0, t) != 0;
      double best = -INFINITY;
      int bi = 0x7fffffff;
      auto score = [&](int j) -> double {             // warp-wide fp64 dot product, one value in every lane
        const float* row = ch + (long long)j * D;
        double a = 0.0;
#pragma unroll
        for (int u = 0; u < U; ++u) a = fma(xv[u], (double)row[lane * U + u], a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        return __shfl_sync(0xffffffffu, a, 0);
      };
      if (!full) {
        const double ln = __shfl_sync(0xffffffffu, line, t);
        const uint32_t mine = my == t ? 0xffffffffu : 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t m = __ballot_sync(0xffffffffu, top.id[k] >= 0 && (double)top.t[k] >= ln) & __ballot_sync(0xffffffffu, mine != 0u);
          while (m) {
            const int src = __ffs(m) - 1;
            m &= m - 1u;
            const int j = __shfl_sync(0xffffffffu, top.id[k], src);
            const double v = score(j);
            if (v > best || (v == best && j < bi)) { best = v; bi = j; }
          }
        }
      } else {
        for (int j = 0; j < C; ++j) {
          const double v = score(j);
          if (v > best) { best = v; bi = j; }      // increasing j: the first index on ties
        }
      }
      if (lane == 0) assign[tt] = bi;
    }
  }
}

// Stable counting sort of one head's tokens by cluster: order[bh, :] lists the
// tokens by (cluster, index); starts / counts per cluster.  One CTA per head;
// its S warps own S consecutive segments of the tokens: each counts its
// segment per cluster, a block-wide scan turns the counts into every
// segment's first slot per cluster (clusters in order, segments in order
// within a cluster), and each warp then scatters its segment in index order.
__global__ void sort_kernel(const int32_t* __restrict__ assign, int32_t* __restrict__ order,
                            int32_t* __restrict__ starts, int32_t* __restrict__ counts, long long N, int C) {
  extern __shared__ int32_t off[];                   // [S][C]: counts, then first slots
  __shared__ int32_t wsum[32];
  const int S = blockDim.x >> 5;
  const long long bh = blockIdx.x;
  const int tid = threadIdx.x, seg = tid >> 5, lane = tid & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const int32_t* a = assign + bh * N;
  const long long L = (N + S - 1) / S;
  const long long t0 = seg * L, t1 = std::min<long long>(N, t0 + L);
  for (int i = tid; i < S * C; i += blockDim.x) off[i] = 0;
  __syncthreads();
  for (long long t = t0 + lane; t < t1; t += 32) atomicAdd(&off[seg * C + a[t]], 1);
  __syncthreads();
  // thread tid takes a contiguous run of clusters; exclusive scan of the cluster totals
  const int per = (C + (int)blockDim.x - 1) / (int)blockDim.x;
  const int j0 = min(C, tid * per), j1 = min(C, j0 + per);
  int run = 0;
  for (int j = j0; j < j1; ++j)
    for (int sg = 0; sg < S; ++sg) run += off[sg * C + j];
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[seg] = incl;
  __syncthreads();
  int base = incl - run;
  for (int w = 0; w < seg; ++w) base += wsum[w];
  for (int j = j0; j < j1; ++j) {
    starts[bh * C + j] = base;
    int tot = 0;
    for (int sg = 0; sg < S; ++sg) {
      const int c = off[sg * C + j];
      off[sg * C + j] = base + tot;
      tot += c;
    }
    counts[bh * C + j] = tot;
    base += tot;
  }
  __syncthreads();
  int32_t* my = off + seg * C;
  for (long long b = t0; b < t1; b += 32) {
    const long long t = b + lane;
    const bool ok = t < t1;
    const int c = ok ? a[t] : -1;
    const uint32_t vm = __ballot_sync(0xffffffffu, ok);
    if (ok) {
      const uint32_t peers = __match_any_sync(vm, c);
      order[bh * N + my[c] + __popc(peers & lt)] = (int32_t)t;
      __syncwarp(vm);
      if ((peers & lt) == 0u) my[c] += __popc(peers);
    }
    __syncwarp();
  }
}

// perm[bh, i] = order[bh, i] (i < N), -1 for the pads; iperm[bh, order[i]] = i.
__global__ void perm_kernel(const int32_t* __restrict__ order, int32_t* __restrict__ perm, int32_t* __restrict__ iperm,
                            long long N, long long Npad) {
  const long long bh = blockIdx.y;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < Npad; i += (long long)gridDim.x * blockDim.x) {
    const int32_t t = i < N ? order[bh * N + i] : -1;
    perm[bh * Npad + i] = t;
    if (t >= 0) iperm[bh * N + t] = (int32_t)i;
  }
}

// ---------------------------------------------------------------- tensor-core assignment
constexpr int kThreads = 192;          // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 one token per thread
constexpr int kRows = 128;             // tokens per item
constexpr int kCent = 128;             // centroids per tile
constexpr int kStages = 2, kSBufs = 2;
constexpr uint32_t kChunk = kRows * 128;   // 128 rows x 64 bf16
constexpr uint32_t kTmemCols = kSBufs * kCent;

template <int D>
struct Smem {
  static constexpr int NCH = D / 64;
  static constexpr uint32_t kX = NCH * kChunk;            // the token tile
  static constexpr uint32_t kStage = 3 * NCH * kChunk;    // a centroid tile: h, m, l
  static constexpr uint32_t kOffX = 0;
  static constexpr uint32_t kOffC = kX;
  static constexpr uint32_t kOffMisc = kOffC + kStages * kStage;
  static constexpr uint32_t kBytes = kOffMisc + 256 + 1024;
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

enum : uint32_t {
  BAR_X_FULL = 0, BAR_X_EMPTY, BAR_C_FULL, BAR_C_EMPTY = BAR_C_FULL + kStages,
  BAR_S_FULL = BAR_C_EMPTY + kStages, BAR_S_EMPTY = BAR_S_FULL + kSBufs, BAR_FINAL = BAR_S_EMPTY + kSBufs,
  NUM_BARS
};

struct Misc {
  uint64_t bar[NUM_BARS];
  uint32_t tmem_base;
  uint32_t abort;
};

struct Args {
  const float* xnorm;           // [BH * N] token norms (upper bounds)
  const unsigned int* cmax;     // [BH] largest centroid norm (float bits, upper bound)
  int32_t* assign;              // [BH * N]
  int32_t* fix_list;            // [BH, N] per head: tokens to decide exactly
  unsigned int* fix_count;      // [BH] their counts
  long long N;
  int C, nxt, nct;              // clusters, token tiles and centroid tiles per head
  long long items;
  float gamma;                  // relative accumulation bound, 3 d 2^-20
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) assign_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                                                                const __grid_constant__ CUtensorMap tmC,
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
    mbar_init(bar(BAR_X_FULL), 1);
    mbar_init(bar(BAR_X_EMPTY), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(BAR_C_FULL + i), 1);
      mbar_init(bar(BAR_C_EMPTY + i), 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(bar(BAR_S_FULL + i), 1);
      mbar_init(bar(BAR_S_EMPTY + i), 4);
    }
    mbar_init(bar(BAR_FINAL), 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t xit = 0, cn = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
        const long long bh = it / a.nxt;
        const int xt = (int)(it % a.nxt);
        ok = wait_bar(bar(BAR_X_EMPTY), (xit & 1u) ^ 1u, abort_flag, 71);
        if (!ok) break;
        mbar_expect_tx(bar(BAR_X_FULL), L::kX);
        const int yx = (int)(bh * a.N + (long long)xt * kRows);
        for (int c = 0; c < NCH; ++c) tma_load_2d(sbase + L::kOffX + c * kChunk, &tmX, c * 64, yx, bar(BAR_X_FULL));
        ++xit;
        for (int ct = 0; ct < a.nct && ok; ++ct) {
          const uint32_t stg = cn % kStages;
          ok = wait_bar(bar(BAR_C_EMPTY + stg), ((cn / kStages) & 1u) ^ 1u, abort_flag, 72);
          if (!ok) break;
          mbar_expect_tx(bar(BAR_C_FULL + stg), L::kStage);
          const int yc = (int)(bh * a.C + (long long)ct * kCent);
          for (int c = 0; c < 3 * NCH; ++c)
            tma_load_2d(sbase + L::kOffC + stg * L::kStage + c * kChunk, &tmC, c * 64, yc, bar(BAR_C_FULL + stg));
          ++cn;
        }
      }
      volatile uint32_t no_abort = 0u;
      if (xit > 0) wait_bar(bar(BAR_X_FULL), (xit - 1) & 1u, &no_abort, 80);
      for (uint32_t j = 1; j <= (uint32_t)kStages && j <= cn; ++j) {
        const uint32_t n = cn - j;
        wait_bar(bar(BAR_C_FULL + n % kStages), (n / kStages) & 1u, &no_abort, 81);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID = idesc_f16(true, false, false, kCent, kRows);     // bf16, K-major A and B
      const uint64_t dX = sdesc(sbase + L::kOffX, 16, 1024);
      const uint64_t dC = sdesc(sbase + L::kOffC, 16, 1024);
      uint32_t xit = 0, cn = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
        ok = wait_bar(bar(BAR_X_FULL), xit & 1u, abort_flag, 73);
        ++xit;
        for (int ct = 0; ct < a.nct && ok; ++ct) {
          const uint32_t stg = cn % kStages, sb = cn % kSBufs;
          ok = wait_bar(bar(BAR_C_FULL + stg), (cn / kStages) & 1u, abort_flag, 74) &&
               wait_bar(bar(BAR_S_EMPTY + sb), ((cn / kSBufs) & 1u) ^ 1u, abort_flag, 75);
          if (!ok) break;
          tc_fence_after();
          const uint64_t c0 = dC + ((stg * L::kStage) >> 4);
          // x . (h + m + l): three passes over the head dimension into one accumulator
#pragma unroll
          for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
              const uint32_t off = (kk & 3) * 32;
              umma_f16(tmem + sb * kCent, dX + (((kk >> 2) * kChunk + off) >> 4),
                       c0 + (((part * NCH + (kk >> 2)) * kChunk + off) >> 4), ID, (part > 0 || kk > 0) ? 1u : 0u);
            }
          umma_commit(bar(BAR_C_EMPTY + stg));
          umma_commit(bar(BAR_S_FULL + sb));
          ++cn;
        }
        if (ok) umma_commit(bar(BAR_X_EMPTY));
      }
      umma_commit(bar(BAR_FINAL));
      volatile uint32_t no_abort = 0u;
      wait_bar(bar(BAR_FINAL), 0u, &no_abort, 82);
    }
  } else {
    // ------------------------------------------------------------ one token per thread
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t cn = 0;
    bool stop = false;
    for (long long it = blockIdx.x; it < a.items && !stop; it += gridDim.x) {
      const long long bh = it / a.nxt;
      const int xt = (int)(it % a.nxt);
      const long long t = (long long)xt * kRows + row;
      // running (best, second, index of best) over the even and the odd
      // columns separately (two independent dependency chains), merged at the
      // end; branch-free updates, strict > keeps the first index on ties
      float best0 = -INFINITY, second0 = -INFINITY, best1 = -INFINITY, second1 = -INFINITY;
      int bi0 = 0x7fffffff, bi1 = 0x7fffffff;
      auto update = [](float x, int j, float& b, float& s, int& bi) {
        const bool gt = x > b;
        s = gt ? b : fmaxf(s, x);
        bi = gt ? j : bi;
        b = gt ? x : b;
      };
      for (int ct = 0; ct < a.nct; ++ct) {
        const uint32_t sb = cn % kSBufs;
        if (!wait_bar(bar(BAR_S_FULL + sb), (cn / kSBufs) & 1u, abort_flag, 76)) { stop = true; break; }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < kCent / 32; ++ch) {
          float v[32];
          tmem_ld32(tmem + lane_off + sb * kCent + ch * 32, v);
          tmem_wait_ld();
          if (ch == kCent / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_S_EMPTY + sb));
          }
          const int j0 = ct * kCent + ch * 32;
          if (j0 + 32 > a.C) {               // the ragged last centroid tile
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (j0 + c >= a.C) v[c] = -INFINITY;
          }
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            update(v[c], j0 + c, best0, second0, bi0);
            update(v[c + 1], j0 + c + 1, best1, second1, bi1);
          }
        }
        ++cn;
      }
      if (stop) break;
      // merge: the larger best (the lower index on equal values); the second
      // is the larger of the two seconds and the smaller best
      const bool one = best1 > best0 || (best1 == best0 && bi1 < bi0);
      const float best = one ? best1 : best0;
      const int bi = min(one ? bi1 : bi0, a.C - 1);        // (no comparable score at all: NaN input)
      const float second = fmaxf(fmaxf(second0, second1), one ? best0 : best1);
      if (t < a.N) {
        const long long tok = bh * a.N + t;
        a.assign[tok] = bi;
        const float thr = 2.f * a.gamma * a.xnorm[tok] * __uint_as_float(a.cmax[bh]);
        if (best - second <= thr) a.fix_list[bh * a.N + atomicAdd(a.fix_count + bh, 1u)] = (int32_t)t;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

}  // namespace clu
}  // namespace tc

namespace {

struct CluWs {
  size_t xnq, xnk, cq, ck, c3q, c3k, cmq, cmk, assign, oq, ok, starts, counts, list, count, total;
};

CluWs clu_layout(long long BH, long long N, int C, int d) {
  CluWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~(size_t)255; return o; };
  w.xnq = take(BH * N * 4);
  w.xnk = take(BH * N * 4);
  w.cq = take(BH * C * d * 4);
  w.ck = take(BH * C * d * 4);
  w.c3q = take(BH * C * 3 * d * 2);
  w.c3k = take(BH * C * 3 * d * 2);
  w.cmq = take(BH * 4);
  w.cmk = take(BH * 4);
  w.assign = take(BH * N * 4);
  w.oq = take(BH * N * 4);
  w.ok = take(BH * N * 4);
  w.starts = take(BH * C * 4);
  w.counts = take(BH * C * 4);
  w.list = take(BH * N * 4);
  w.count = take(BH * 4);
  w.total = off;
  return w;
}

}  // namespace

size_t cocluster_workspace_bytes(long long BH, long long N, int nb, int d) { return clu_layout(BH, N, nb, d).total; }

// q, k: raster bf16 [BH, N, d].  C = nb clusters, `rounds` rounds.  perm_* [BH, Npad], iperm_* [BH, N].
cudaError_t launch_cocluster(const void* q, const void* k, long long BH, long long N, int nb, int d, int rounds,
                             int32_t* perm_q, int32_t* iperm_q, int32_t* perm_k, int32_t* iperm_k, void* ws,
                             cudaStream_t st, int* launches) {
  using namespace tc::clu;
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  const int C = nb;
  const long long Npad = (long long)nb * kBlock;
  const CluWs w = clu_layout(BH, N, C, d);
  char* base = reinterpret_cast<char*>(ws);
  auto F = [&](size_t o) { return reinterpret_cast<float*>(base + o); };
  auto I = [&](size_t o) { return reinterpret_cast<int32_t*>(base + o); };
  auto U = [&](size_t o) { return reinterpret_cast<unsigned int*>(base + o); };
  auto B = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(base + o); };
  const __nv_bfloat16* xq = reinterpret_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* xk = reinterpret_cast<const __nv_bfloat16*>(k);
  int n_launch = 0;
  cudaError_t e;
#define SVSA_CLU_CHECK() do { e = cudaGetLastError(); if (e != cudaSuccess) return e; ++n_launch; } while (0)

  const unsigned row_blocks = (unsigned)((BH * N + kWarpsPerBlock - 1) / kWarpsPerBlock);
  // fix-up: about four CTAs per SM over all heads, at least one per head
  const dim3 fix_grid((unsigned)std::max<long long>(1, (tc::sm_count() * 4 + BH - 1) / BH), (unsigned)BH);
  const unsigned cent_blocks = (unsigned)((BH * C + kWarpsPerBlock - 1) / kWarpsPerBlock);
  auto norms = [&](const __nv_bfloat16* x, float* out) -> cudaError_t {
    if (d == 128) tc::clu::norms_kernel<128><<<row_blocks, 32 * kWarpsPerBlock, 0, st>>>(x, out, BH * N);
    else tc::clu::norms_kernel<64><<<row_blocks, 32 * kWarpsPerBlock, 0, st>>>(x, out, BH * N);
    SVSA_CLU_CHECK();
    return cudaSuccess;
  };
  auto means = [&](const __nv_bfloat16* x, const int32_t* order, const float* partner, float* cent,
                   __nv_bfloat16* c3, unsigned int* cmax) -> cudaError_t {
    e = cudaMemsetAsync(cmax, 0, BH * 4, st);
    if (e != cudaSuccess) return e;
    const int32_t* sp = order ? I(w.starts) : nullptr;
    const int32_t* cp = order ? I(w.counts) : nullptr;
    if (d == 128)
      tc::clu::means_kernel<128><<<cent_blocks, 32 * kWarpsPerBlock, 0, st>>>(x, order, sp, cp, partner, cent, c3, cmax,
                                                                                BH, N, C);
    else
      tc::clu::means_kernel<64><<<cent_blocks, 32 * kWarpsPerBlock, 0, st>>>(x, order, sp, cp, partner, cent, c3, cmax,
                                                                               BH, N, C);
    SVSA_CLU_CHECK();
    return cudaSuccess;
  };
  const int nxt = (int)((N + kRows - 1) / kRows);
  const int nct = (C + kCent - 1) / kCent;
  // one assignment pass: tokens x against the centroids (cent, c3, cmax); exact fix-up; stable sort into `order`
  auto pass = [&](const __nv_bfloat16* x, const float* xnorm, const float* cent, const __nv_bfloat16* c3,
                  const unsigned int* cmax, int32_t* order) -> cudaError_t {
    CUtensorMap mx, mc;
    if (!tc::make_map_2d(&mx, x, BH * N, d, kRows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
        !tc::make_map_2d(&mc, c3, BH * C, 3 * d, kCent, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      return cudaErrorInvalidValue;
    e = cudaMemsetAsync(U(w.count), 0, BH * 4, st);
    if (e != cudaSuccess) return e;
    Args a;
    a.xnorm = xnorm; a.cmax = cmax; a.assign = I(w.assign); a.fix_list = I(w.list); a.fix_count = U(w.count);
    a.N = N; a.C = C; a.nxt = nxt; a.nct = nct;
    a.items = BH * nxt;
    a.gamma = (float)(3 * d) * 9.5367431640625e-7f;    // 3d * 2^-20
    const unsigned grid = (unsigned)std::min<long long>(a.items, tc::sm_count());
    if (d == 128) {
      e = cudaFuncSetAttribute(assign_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Smem<128>::kBytes);
      if (e != cudaSuccess) return e;
      assign_tc_kernel<128><<<grid, kThreads, Smem<128>::kBytes, st>>>(mx, mc, a);
      SVSA_CLU_CHECK();
      fix_kernel<128><<<fix_grid, 32 * kWarpsPerBlock, 0, st>>>(
          x, cent, I(w.list), U(w.count), xnorm, cmax, a.gamma, I(w.assign), N, C);
      SVSA_CLU_CHECK();
    } else {
      e = cudaFuncSetAttribute(assign_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Smem<64>::kBytes);
      if (e != cudaSuccess) return e;
      assign_tc_kernel<64><<<grid, kThreads, Smem<64>::kBytes, st>>>(mx, mc, a);
      SVSA_CLU_CHECK();
      fix_kernel<64><<<fix_grid, 32 * kWarpsPerBlock, 0, st>>>(
          x, cent, I(w.list), U(w.count), xnorm, cmax, a.gamma, I(w.assign), N, C);
      SVSA_CLU_CHECK();
    }
    // as many segment warps as 200 KB of counters allow, at most 32
    const int segs = std::max(1, std::min(32, (int)(204800 / ((size_t)C * sizeof(int32_t)))));
    const size_t sort_smem = (size_t)segs * C * sizeof(int32_t);
    e = cudaFuncSetAttribute(sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sort_smem);
    if (e != cudaSuccess) return e;
    sort_kernel<<<(unsigned)BH, 32 * segs, sort_smem, st>>>(I(w.assign), order, I(w.starts), I(w.counts), N, C);
    SVSA_CLU_CHECK();
    return cudaSuccess;
  };

  if ((e = norms(xq, F(w.xnq))) != cudaSuccess) return e;
  if ((e = norms(xk, F(w.xnk))) != cudaSuccess) return e;
  // initial query centroids: raster block means
  if ((e = means(xq, nullptr, nullptr, F(w.cq), B(w.c3q), U(w.cmq))) != cudaSuccess) return e;
  for (int r = 0; r < rounds; ++r) {
    // query-aware partition of the keys, then the key centroids
    if ((e = pass(xk, F(w.xnk), F(w.cq), B(w.c3q), U(w.cmq), I(w.ok))) != cudaSuccess) return e;
    if ((e = means(xk, I(w.ok), F(w.cq), F(w.ck), B(w.c3k), U(w.cmk))) != cudaSuccess) return e;
    // key-aware partition of the queries, then the query centroids (not needed after the last round)
    if ((e = pass(xq, F(w.xnq), F(w.ck), B(w.c3k), U(w.cmk), I(w.oq))) != cudaSuccess) return e;
    if (r + 1 < rounds && (e = means(xq, I(w.oq), F(w.ck), F(w.cq), B(w.c3q), U(w.cmq))) != cudaSuccess) return e;
  }
  dim3 pg((unsigned)std::min<long long>((Npad + 255) / 256, 1024), (unsigned)BH);
  perm_kernel<<<pg, 256, 0, st>>>(I(w.oq), perm_q, iperm_q, N, Npad);
  SVSA_CLU_CHECK();
  perm_kernel<<<pg, 256, 0, st>>>(I(w.ok), perm_k, iperm_k, N, Npad);
  SVSA_CLU_CHECK();
#undef SVSA_CLU_CHECK
  *launches = n_launch;
  return cudaSuccess;
}

cudaError_t cocluster_tc_error(unsigned int* code, cudaStream_t st) { return tc::read_error(code, st); }

}  // namespace svsa
