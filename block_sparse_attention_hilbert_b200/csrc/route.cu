// Error-aware routing ratios ("SVG-EAR", technical summary 2.B).
//
// The query centroid qbar_I stands in for the queries of block I.  With
// s_j = qbar_I . k_j / sqrt(d) over all valid keys, M = max_j s_j and
// Z = sum_j e^{s_j - M}, block J's compensation error is
//   e_IJ = || sum_{j in J} e^{s_j - M} v_j - n_J e^{qbar_I . kbar_J / sqrt(d) - M} vbar_J ||_2
// (the change of the un-normalised proxy output when J's keys/values are
// replaced by their means) and the routed ratio is r_IJ = e_IJ / Z * 64 / n_J
// (error per unit of block size).
//
// One CTA owns 16 query blocks of one head and streams the key/value blocks
// once (O(C_q N_k d) work, as the page states).  The running maximum grows as
// tiles arrive, so each e_IJ is first taken against the maximum m_J known at
// tile J and stored with m_J; a final sweep turns it into
// e * exp(m_J - M) / Z * 64 / n_J.  fp32 throughout.
#include <cuda_fp16.h>

#include "common.cuh"

namespace svsa {

constexpr int kRouteThreads = 256;
constexpr int kRouteRows = 16;

template <int D>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(
    const float* __restrict__ qbar, const __nv_bfloat16* __restrict__ kp,
    const __half* __restrict__ vp, const float* __restrict__ kbar,
    const float* __restrict__ vbar, float* __restrict__ R, float* __restrict__ Rm, long long N, int nb,
    float scale) {
  constexpr int CH = D / 16;                          // channels per thread in the value phase
  __shared__ float q_s[kRouteRows][D];
  __shared__ __nv_bfloat16 k_s[kBlock][D + 8];
  __shared__ __half v_s[kBlock][D];
  __shared__ float e_s[kRouteRows][kBlock];
  __shared__ float m_s[kRouteRows], z_s[kRouteRows];

  const long long bh = blockIdx.y;
  const int I0 = blockIdx.x * kRouteRows;
  const int tid = threadIdx.x;
  const int row = tid >> 4, sub = tid & 15;           // 16 threads per proxy row
  const long long Npad = (long long)nb * kBlock;

  for (int o = tid; o < kRouteRows * D; o += kRouteThreads) {
    const int r = o / D, c = o % D;
    q_s[r][c] = (I0 + r < nb) ? qbar[(bh * nb + I0 + r) * (long long)D + c] : 0.f;
  }
  if (tid < kRouteRows) { m_s[tid] = -INFINITY; z_s[tid] = 0.f; }
  const bool row_ok = I0 + row < nb;
  float* rrow = R + (bh * nb + (row_ok ? I0 + row : 0)) * (long long)nb;
  float* mrow = Rm + (bh * nb + (row_ok ? I0 + row : 0)) * (long long)nb;

  for (int J = 0; J < nb; ++J) {
    __syncthreads();
    const __nv_bfloat16* kb = kp + (bh * Npad + (long long)J * kBlock) * D;
    const __half* vb = vp + (bh * Npad + (long long)J * kBlock) * D;
    for (int o = tid; o < kBlock * D / 8; o += kRouteThreads) {
      const int r = o / (D / 8), c = (o % (D / 8)) * 8;
      const uint4 kv = *reinterpret_cast<const uint4*>(kb + (long long)r * D + c);
      const uint4 vv = *reinterpret_cast<const uint4*>(vb + (long long)r * D + c);
      *reinterpret_cast<uint4*>(&k_s[r][c]) = kv;
      *reinterpret_cast<uint4*>(&v_s[r][c]) = vv;
    }
    __syncthreads();
    const long long key0 = (long long)J * kBlock;
    const int nJ = (int)std::max<long long>(0, std::min<long long>(kBlock, N - key0));
    // logits: row `row`, keys sub + 16*u
    float s[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) s[u] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float q = q_s[row][c];
#pragma unroll
      for (int u = 0; u < 4; ++u) s[u] = fmaf(q, __bfloat162float(k_s[sub + 16 * u][c]), s[u]);
    }
    float tmax = -INFINITY;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      s[u] = (sub + 16 * u < nJ) ? s[u] * scale : -INFINITY;
      tmax = fmaxf(tmax, s[u]);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float m_old = m_s[row];
    const float m_new = fmaxf(m_old, tmax);
    float zs = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float e = s[u] == -INFINITY ? 0.f : expf(s[u] - m_new);
      e_s[row][sub + 16 * u] = e;
      zs += e;
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
    __syncwarp();
    // centroid logit qbar_I . kbar_J (fp32 mean of block J)
    const float* kbJ = kbar + (bh * nb + J) * (long long)D;
    const float* vbJ = vbar + (bh * nb + J) * (long long)D;
    float lc = 0.f;
#pragma unroll
    for (int u = 0; u < CH; ++u) lc = fmaf(q_s[row][sub * CH + u], kbJ[sub * CH + u], lc);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) lc += __shfl_xor_sync(0xffffffffu, lc, o);
    const float cw = nJ > 0 ? (float)nJ * expf(lc * scale - m_new) : 0.f;
    __syncthreads();                                  // e_s complete
    // exact weighted value sum minus centroid term, channels sub*CH .. +CH
    float err2 = 0.f;
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      const int c = sub * CH + u;
      float a = 0.f;
#pragma unroll 8
      for (int j = 0; j < kBlock; ++j) a = fmaf(e_s[row][j], __half2float(v_s[j][c]), a);
      const float diff = a - cw * vbJ[c];
      err2 = fmaf(diff, diff, err2);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) err2 += __shfl_xor_sync(0xffffffffu, err2, o);
    if (sub == 0) {
      m_s[row] = m_new;
      z_s[row] = (m_old == -INFINITY ? 0.f : z_s[row] * expf(m_old - m_new)) + zs;
      if (row_ok) { rrow[J] = sqrtf(err2); mrow[J] = m_new; }
    }
  }
  __syncthreads();
  if (!row_ok) return;
  const float M = m_s[row], Z = z_s[row];
  for (int J = sub; J < nb; J += 16) {
    const long long key0 = (long long)J * kBlock;
    const int nJ = (int)std::max<long long>(1, std::min<long long>(kBlock, N - key0));
    const float e = rrow[J];
    rrow[J] = e > 0.f ? e * expf(mrow[J] - M) / Z * ((float)kBlock / (float)nJ) : 0.f;
  }
}

cudaError_t launch_route(const float* qbar, const void* kp, const void* vp, const float* kbar,
                         const float* vbar, float* R, float* Rm, long long BH, long long N, int nb,
                         int d, cudaStream_t st) {
  dim3 grid((unsigned)((nb + kRouteRows - 1) / kRouteRows), (unsigned)BH);
  const float scale = 1.0f / sqrtf((float)d);
  const __nv_bfloat16* k = reinterpret_cast<const __nv_bfloat16*>(kp);
  const __half* v = reinterpret_cast<const __half*>(vp);
  if (d == 128) route_kernel<128><<<grid, kRouteThreads, 0, st>>>(qbar, k, v, kbar, vbar, R, Rm, N, nb, scale);
  else if (d == 64) route_kernel<64><<<grid, kRouteThreads, 0, st>>>(qbar, k, v, kbar, vbar, R, Rm, N, nb, scale);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace svsa
