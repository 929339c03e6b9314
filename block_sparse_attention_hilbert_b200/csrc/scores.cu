// Pooled block scores S[bh, I, J] (fp32), one row per 64-token query block.
//
// SIZE = 64 ("DFSAttn" trick 2, block averages):
//   S_IJ = softmax_J(qbar_I . kbar_J / sqrt(d)) over all key blocks.
// SIZE = 16 (DFSAttn trick 2, sub-block scoring summed per block):
//   p_ij = softmax_j(qt_i . kt_j / sqrt(d)) over the non-empty key sub-blocks,
//   S_IJ = (1 / m_I) * sum_{i in I} sum_{j in J} p_ij over the m_I non-empty
//   query sub-blocks i of I.
//
// fp32 SIMT products (the selection needs scores to ~1e-7, far below what a
// bf16 product gives).  A CTA owns 32 pooled query rows of one head and
// streams the pooled keys through shared memory in 64-row tiles, twice: pass
// 1 keeps each row's running max and sum of exponentials, pass 2 recomputes
// the identical logits, normalises, and (SIZE = 16) adds the 4 x 4 sub-pairs
// of every block pair with warp shuffles before one store per (I, J).
#include "common.cuh"

namespace svsa {

constexpr int kScoreThreads = 256;
constexpr int kQRows = 32;     // pooled query rows per CTA
constexpr int kKRows = 64;     // pooled key rows per tile

template <int D, int SIZE>
__global__ void __launch_bounds__(kScoreThreads) scores_kernel(
    const float* __restrict__ qs, const float* __restrict__ ks, float* __restrict__ S,
    long long N, int ng, int nb, float scale) {
  constexpr int PER = kBlock / SIZE;          // sub-rows per block (1 or 4)
  constexpr int LD = D + 4;                   // padded smem row (floats)
  extern __shared__ float smem[];
  float* q_s = smem;                          // [kQRows][LD]
  float* k_s = smem + kQRows * LD;            // [kKRows][LD]

  const long long bh = blockIdx.y;
  const int row0 = blockIdx.x * kQRows;       // first pooled query row
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;     // 16 x 16 threads; ty pairs of rows, tx columns
  const float* qb = qs + bh * (long long)ng * D;
  const float* kb = ks + bh * (long long)ng * D;

  for (int o = tid; o < kQRows * D / 4; o += kScoreThreads) {
    const int r = o / (D / 4), c = (o % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row0 + r < ng) v = *reinterpret_cast<const float4*>(qb + (long long)(row0 + r) * D + c);
    *reinterpret_cast<float4*>(q_s + r * LD + c) = v;
  }

  // valid rows: a pooled row is empty when its first position is >= N
  auto row_ok = [&](int g) { return g < ng && (long long)g * SIZE < N; };
  const int r_a = row0 + 2 * ty, r_b = r_a + 1;
  const bool ok_a = row_ok(r_a), ok_b = row_ok(r_b);

  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  const int ntiles = (ng + kKRows - 1) / kKRows;

  for (int pass = 0; pass < 2; ++pass) {
    for (int kt = 0; kt < ntiles; ++kt) {
      __syncthreads();
      for (int o = tid; o < kKRows * D / 4; o += kScoreThreads) {
        const int r = o / (D / 4), c = (o % (D / 4)) * 4;
        const int g = kt * kKRows + r;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (g < ng) v = *reinterpret_cast<const float4*>(kb + (long long)g * D + c);
        *reinterpret_cast<float4*>(k_s + r * LD + c) = v;
      }
      __syncthreads();
      float acc[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
      const float* qa = q_s + (2 * ty) * LD;
      const float* qbp = qa + LD;
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 a0 = *reinterpret_cast<const float4*>(qa + c);
        const float4 a1 = *reinterpret_cast<const float4*>(qbp + c);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 b = *reinterpret_cast<const float4*>(k_s + (tx + 16 * j) * LD + c);
          acc[0][j] = fmaf(a0.x, b.x, acc[0][j]); acc[0][j] = fmaf(a0.y, b.y, acc[0][j]);
          acc[0][j] = fmaf(a0.z, b.z, acc[0][j]); acc[0][j] = fmaf(a0.w, b.w, acc[0][j]);
          acc[1][j] = fmaf(a1.x, b.x, acc[1][j]); acc[1][j] = fmaf(a1.y, b.y, acc[1][j]);
          acc[1][j] = fmaf(a1.z, b.z, acc[1][j]); acc[1][j] = fmaf(a1.w, b.w, acc[1][j]);
        }
      }
      // scaled logits; empty key rows -> -inf
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int g = kt * kKRows + tx + 16 * j;
        const bool kok = row_ok(g);
        acc[0][j] = kok ? acc[0][j] * scale : -INFINITY;
        acc[1][j] = kok ? acc[1][j] * scale : -INFINITY;
      }
      if (pass == 0) {
        float ta = fmaxf(fmaxf(acc[0][0], acc[0][1]), fmaxf(acc[0][2], acc[0][3]));
        float tb = fmaxf(fmaxf(acc[1][0], acc[1][1]), fmaxf(acc[1][2], acc[1][3]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, o));
          tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, o));
        }
        const float na = fmaxf(m_a, ta), nbm = fmaxf(m_b, tb);
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sa += (acc[0][j] == -INFINITY) ? 0.f : expf(acc[0][j] - na);
          sb += (acc[1][j] == -INFINITY) ? 0.f : expf(acc[1][j] - nbm);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          sa += __shfl_xor_sync(0xffffffffu, sa, o);
          sb += __shfl_xor_sync(0xffffffffu, sb, o);
        }
        l_a = (m_a == -INFINITY ? 0.f : l_a * expf(m_a - na)) + sa;
        l_b = (m_b == -INFINITY ? 0.f : l_b * expf(m_b - nbm)) + sb;
        m_a = na; m_b = nbm;
      } else {
        const float ia = ok_a ? 1.f / l_a : 0.f, ib = ok_b ? 1.f / l_b : 0.f;
        float p[2][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          p[0][j] = (ok_a && acc[0][j] != -INFINITY) ? expf(acc[0][j] - m_a) * ia : 0.f;
          p[1][j] = (ok_b && acc[1][j] != -INFINITY) ? expf(acc[1][j] - m_b) * ib : 0.f;
        }
        if constexpr (SIZE == kBlock) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int J = kt * kKRows + tx + 16 * j;
            if (J < nb) {
              if (r_a < nb) S[(bh * nb + r_a) * (long long)nb + J] = p[0][j];
              if (r_b < nb) S[(bh * nb + r_b) * (long long)nb + J] = p[1][j];
            }
          }
        } else {
          // rows 2ty, 2ty+1 and the partner half-warp's two rows form one query
          // block; columns tx..tx^3 (same j) form one key block
          float v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[j] = p[0][j] + p[1][j];
            v[j] += __shfl_xor_sync(0xffffffffu, v[j], 1);
            v[j] += __shfl_xor_sync(0xffffffffu, v[j], 2);
            v[j] += __shfl_xor_sync(0xffffffffu, v[j], 16);
          }
          // number of non-empty sub-rows of this query block
          const int I = (row0 + 2 * ty) / PER;
          const long long first = (long long)I * kBlock;
          const long long nval = std::max<long long>(0, std::min<long long>(kBlock, N - first));
          const int m_sub = (int)((nval + SIZE - 1) / SIZE);
          if ((tx & 3) == 0 && (ty & 1) == 0 && I < nb && m_sub > 0) {
            const float inv = 1.f / (float)m_sub;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int J = (kt * kKRows + tx + 16 * j) / PER;
              if (J < nb) S[(bh * nb + I) * (long long)nb + J] = v[j] * inv;
            }
          }
        }
      }
    }
  }
}

size_t scores_smem_bytes(int d) { return (size_t)(kQRows + kKRows) * (d + 4) * sizeof(float); }

cudaError_t launch_scores(const float* qs, const float* ks, float* S, long long BH, long long N,
                          int ng, int nb, int d, int size, cudaStream_t st) {
  dim3 grid((unsigned)((ng + kQRows - 1) / kQRows), (unsigned)BH);
  const size_t smem = scores_smem_bytes(d);
  const float scale = 1.0f / sqrtf((float)d);
#define SVSA_SCORES(DD, SS)                                                                      \
  do {                                                                                           \
    cudaError_t e = cudaFuncSetAttribute(scores_kernel<DD, SS>,                                  \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                              \
    scores_kernel<DD, SS><<<grid, kScoreThreads, smem, st>>>(qs, ks, S, N, ng, nb, scale);       \
  } while (0)
  if (d == 128 && size == 64) SVSA_SCORES(128, 64);
  else if (d == 128 && size == 16) SVSA_SCORES(128, 16);
  else if (d == 64 && size == 64) SVSA_SCORES(64, 64);
  else if (d == 64 && size == 16) SVSA_SCORES(64, 16);
  else return cudaErrorInvalidValue;
#undef SVSA_SCORES
  return cudaGetLastError();
}

}  // namespace svsa
