// SICS block scorer: block coherence from the sum of intra-block cosine
// similarities of the keys, and the list it selects for every query block of
// a head.
//
// "SPADE: An Input-Adaptive Sparse Attention Engine for Fast Video Diffusion
// Models Inference", part 2: instead of estimating every block pair, a quick
// coherence check -- the sum of the cosine similarities inside a block --
// decides per head and per step which blocks attention focuses on: a block
// whose tokens agree is kept, one whose tokens disagree is skipped.
//
// For key block J with n_J valid keys,
//   SICS_J = sum_{i, j in J} cos(k_i, k_j) = || sum_{i in J} k_i / ||k_i|| ||^2
// (the double sum of unit-vector products is the squared norm of their sum;
// a zero key counts as the zero vector), c_J = SICS_J / n_J^2 in [0, 1] and
// S_J = c_J / sum_J' c_J'.  The closed form reads each block once: the kernel
// is one HBM pass over K, as the pooling is.
//
// sics_kernel       one CTA per (block, head): per-key norms, the sum of the
//                   unit keys, its squared norm -> c[bh, J]
// sics_norm_kernel  one CTA per head: S[bh, J] = c_J / sum c (fixed-order sum)
// broadcast_kernel  the head's selected list (from the select kernel, one row
//                   per head) copied into the row of every query block, with
//                   its bitmap
// Also here: check_mask_kernel, the optional validation of caller-built lists
// before the attention, with its status word.
#include "common.cuh"

namespace svsa {

constexpr int kSicsThreads = 256;

// Status bits of this translation unit (kFlagMask: a malformed mask list).
static __device__ unsigned int g_sics_flags;

template <int D>
__global__ void __launch_bounds__(kSicsThreads) sics_kernel(const __nv_bfloat162* __restrict__ kp,
                                                            float* __restrict__ coh, long long N, long long Npad,
                                                            int nb) {
  constexpr int CPR = D / 8;                   // 16-byte chunks per key row
  constexpr int RL = kSicsThreads / CPR;       // row lanes
  constexpr int RPT = kBlock / RL;             // rows per thread
  __shared__ float red[RL][D];
  __shared__ float wsum[kSicsThreads / 32];
  const int J = blockIdx.x;
  const long long bh = blockIdx.y;
  const int ch = threadIdx.x % CPR, rl = threadIdx.x / CPR;
  const long long row0 = (long long)J * kBlock;
  const __nv_bfloat162* base = kp + (bh * Npad + row0) * (D / 2);

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const int r = rl + RL * u;
    const bool ok = row0 + r < N;              // uniform over the CPR lanes of a row
    float x[8];
    float ss = 0.f;
    if (ok) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + (long long)r * (D / 2)) + ch);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    // squared norm of the row: the CPR lanes of a row are consecutive lanes
#pragma unroll
    for (int o = CPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float nrm = sqrtf(ss);
    if (nrm > 0.f) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += x[e] / nrm;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rl][ch * 8 + e] = acc[e];
  __syncthreads();
  // ||sum of the unit keys||^2: column sums in a fixed row-lane order, then a
  // fixed-order reduction of the squares
  float part = 0.f;
  for (int c = threadIdx.x; c < D; c += kSicsThreads) {
    float s = 0.f;
#pragma unroll 8
    for (int l = 0; l < RL; ++l) s += red[l][c];
    part = fmaf(s, s, part);
  }
  part = warp_sum(part);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kSicsThreads / 32; ++w) tot += wsum[w];
    const long long n = std::max<long long>(0, std::min<long long>(kBlock, N - row0));
    coh[bh * nb + J] = n > 0 ? tot / (float)(n * n) : 0.f;
  }
}

// S[bh, J] = c[bh, J] / sum_J c[bh, J]; all zero when the sum is zero (the
// threshold rule then keeps every block, top-k the first k).
__global__ void __launch_bounds__(256) sics_norm_kernel(const float* __restrict__ coh, float* __restrict__ S,
                                                        int nb) {
  __shared__ float wsum[8];
  const long long bh = blockIdx.x;
  const float* c = coh + bh * nb;
  float part = 0.f;
  for (int J = threadIdx.x; J < nb; J += 256) part += c[J];
  part = warp_sum(part);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = part;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += wsum[w];
  for (int J = threadIdx.x; J < nb; J += 256) S[bh * nb + J] = tot > 0.f ? c[J] / tot : 0.f;
}

// Copy the head's list (one row per head: idx[bh, :cnt[bh]], row stride
// hcap) into the rows of kRowsPerCta query blocks of that head.
constexpr int kRowsPerCta = 16;
__global__ void __launch_bounds__(256) broadcast_kernel(const int32_t* __restrict__ hidx,
                                                        const int32_t* __restrict__ hcnt, int hcap, int nb, int cap,
                                                        int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
                                                        uint32_t* __restrict__ bits) {
  extern __shared__ uint32_t bm[];             // the head's bitmap, ceil(nb / 32) words
  const long long bh = blockIdx.y;
  const int words = (nb + 31) / 32;
  const int cnt = hcnt[bh];
  const int32_t* src = hidx + bh * hcap;
  if (bits != nullptr) {
    for (int w = threadIdx.x; w < words; w += 256) bm[w] = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < cnt; j += 256) atomicOr(&bm[src[j] >> 5], 1u << (src[j] & 31));
    __syncthreads();
  }
  const int I0 = blockIdx.x * kRowsPerCta;
  const int I1 = min(nb, I0 + kRowsPerCta);
  for (int I = I0; I < I1; ++I) {
    const long long row = bh * nb + I;
    for (int j = threadIdx.x; j < cnt; j += 256) kv_idx[row * cap + j] = src[j];
    if (threadIdx.x == 0) kv_cnt[row] = cnt;
    if (bits != nullptr)
      for (int w = threadIdx.x; w < words; w += 256) bits[row * words + w] = bm[w];
  }
}

cudaError_t launch_sics(const void* kp, float* coh, float* S, long long BH, long long N, int nb, int d,
                        cudaStream_t st) {
  dim3 grid((unsigned)nb, (unsigned)BH);
  const __nv_bfloat162* k = reinterpret_cast<const __nv_bfloat162*>(kp);
  const long long Npad = (long long)nb * kBlock;
  if (d == 128) sics_kernel<128><<<grid, kSicsThreads, 0, st>>>(k, coh, N, Npad, nb);
  else if (d == 64) sics_kernel<64><<<grid, kSicsThreads, 0, st>>>(k, coh, N, Npad, nb);
  else return cudaErrorInvalidValue;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sics_norm_kernel<<<(unsigned)BH, 256, 0, st>>>(coh, S, nb);
  return cudaGetLastError();
}

cudaError_t launch_broadcast(const int32_t* hidx, const int32_t* hcnt, int hcap, long long BH, int nb, int cap,
                             int32_t* kv_idx, int32_t* kv_cnt, uint32_t* bits, cudaStream_t st) {
  dim3 grid((unsigned)((nb + kRowsPerCta - 1) / kRowsPerCta), (unsigned)BH);
  const size_t smem = bits != nullptr ? (size_t)((nb + 31) / 32) * sizeof(uint32_t) : 0;
  broadcast_kernel<<<grid, 256, smem, st>>>(hidx, hcnt, hcap, nb, cap, kv_idx, kv_cnt, bits);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- mask check
// One warp per row: kv_cnt in [0, cap], every kept index in [0, nb) and each
// larger than the one before.  A malformed row ORs bit 2 into the status word;
// nothing is written anywhere else.
__global__ void __launch_bounds__(256) check_mask_kernel(const int32_t* __restrict__ kv_idx,
                                                         const int32_t* __restrict__ kv_cnt, long long rows, int cap,
                                                         int nb) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int cnt = kv_cnt[r];
  bool bad = cnt < 0 || cnt > cap;
  if (!bad) {
    const int32_t* row = kv_idx + r * cap;
    for (int j = lane; j < cnt; j += 32) {
      const int J = row[j];
      const int P = j > 0 ? row[j - 1] : -1;
      bad |= J < 0 || J >= nb || J <= P;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_sics_flags, kFlagMask);
}

cudaError_t launch_check_mask(const int32_t* kv_idx, const int32_t* kv_cnt, long long rows, int cap, int nb,
                              cudaStream_t st) {
  check_mask_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(kv_idx, kv_cnt, rows, cap, nb);
  return cudaGetLastError();
}

// One CTA per head: the pairing table must be a permutation of 0..nb-1 (every
// entry in range, none twice); a bit per block in shared memory catches a
// repeat.  A bad table ORs kFlagMask into the status word.
__global__ void __launch_bounds__(256) check_pairs_kernel(const int32_t* __restrict__ pairs, int nb) {
  extern __shared__ uint32_t seen[];          // ceil(nb / 32) words
  const int words = (nb + 31) / 32;
  for (int w = threadIdx.x; w < words; w += 256) seen[w] = 0u;
  __syncthreads();
  const int32_t* row = pairs + (long long)blockIdx.x * nb;
  bool bad = false;
  for (int i = threadIdx.x; i < nb; i += 256) {
    const int J = row[i];
    if (J < 0 || J >= nb) {
      bad = true;
    } else {
      const uint32_t bit = 1u << (J & 31);
      bad |= (atomicOr(&seen[J >> 5], bit) & bit) != 0u;
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&g_sics_flags, kFlagMask);
}

cudaError_t launch_check_pairs(const int32_t* pairs, long long BH, int nb, cudaStream_t st) {
  check_pairs_kernel<<<(unsigned)BH, 256, (size_t)((nb + 31) / 32) * sizeof(uint32_t), st>>>(pairs, nb);
  return cudaGetLastError();
}

cudaError_t sics_flags(unsigned int* v, cudaStream_t st) { return read_and_clear_flags(g_sics_flags, v, st); }

}  // namespace svsa
