// Block / sub-block means of a reordered tensor.
//
// "DFSAttn", trick 2 (the block "average" stands for the block) and "SVG-EAR"
// 2.A (a cluster centroid is its mean).  out[bh, g, :] = mean of the valid
// rows (position < N) of group g = rows [g*SIZE, g*SIZE + SIZE); 0 if none.
//
// One CTA reads one 64-row block (d*128 bytes) with 16-byte loads: CPR chunk
// lanes x 256 / CPR row lanes, row lane l taking the consecutive rows
// [l * RPT, l * RPT + RPT), so a warp covers 8 consecutive rows and lies in
// one group (groups are 16 or 64 rows).  Each thread sums its rows in fp32,
// the row lanes of a warp are added by shuffles, and the warps of a group in
// a fixed order through shared memory, so the result is deterministic.  One
// accumulator row per thread and one partial row per warp keep registers and
// shared memory small, so many CTAs -- and their loads -- are resident.
//
// Optional second output for the tensor-core scores: each mean m as an fp16
// pair, split[bh, g, :] = [hi (d) | lo (d)] with hi = fp16(m) and
// lo = fp16(m - hi) (m - hi is exact in fp32), so hi + lo carries m to ~22
// bits.  Means beyond the fp16 range saturate.  A third optional output holds
// the same split in bf16 (hi = bf16(m), lo = bf16(m - hi): ~16 bits, fp32
// range) for products against raw bf16 keys.
#include <cuda_fp16.h>

#include "common.cuh"

namespace svsa {

constexpr int kPoolThreads = 256;

// Status bits of this translation unit (kFlagRangeMean: a mean that the fp16
// split of the scores saturated, or a non-finite one).
static __device__ unsigned int g_pool_flags;

__device__ __forceinline__ float2 pair_to_float2(const __nv_bfloat162& v) { return __bfloat1622float2(v); }
__device__ __forceinline__ float2 pair_to_float2(const __half2& v) { return __half22float2(v); }

// T2 = __nv_bfloat162 (queries, keys) or __half2 (values)
template <int D, int SIZE, typename T2>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(
    const T2* __restrict__ xp, float* __restrict__ out, __half* __restrict__ split,
    __nv_bfloat16* __restrict__ split_bf, int32_t* __restrict__ nvalid, long long N, long long Npad) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int RL = kPoolThreads / CPR;     // row lanes
  constexpr int RPT = kBlock / RL;           // consecutive rows per thread
  constexpr int G = kBlock / SIZE;           // groups per 64-row block
  constexpr int NW = kPoolThreads / 32;      // warps
  constexpr int WR = kBlock / NW;            // rows per warp (8)
  static_assert(WR * NW == kBlock && SIZE % WR == 0, "a warp's rows lie in one group");
  __shared__ float red[NW][D];

  const int blk = blockIdx.x;
  const long long bh = blockIdx.y;
  const int ch = threadIdx.x % CPR, rl = threadIdx.x / CPR;
  const long long row0 = (long long)blk * kBlock;
  const T2* base = xp + (bh * Npad + row0) * (D / 2);

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  uint4 v[RPT];
#pragma unroll
  for (int u = 0; u < RPT; ++u) {            // all loads first
    const int r = rl * RPT + u;
    v[u] = row0 + r < N ? __ldg(reinterpret_cast<const uint4*>(base + (long long)r * (D / 2)) + ch)
                        : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const T2* p = reinterpret_cast<const T2*>(&v[u]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = pair_to_float2(p[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
  // the warp's row lanes (lanes ch, ch + CPR, ...) into its first CPR lanes
#pragma unroll
  for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) < CPR) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][ch * 8 + e] = acc[e];
  }
  __syncthreads();
  for (int o = threadIdx.x; o < G * D; o += kPoolThreads) {
    const int g = o / D, c = o % D;
    float s = 0.f;                           // the group's warps, in order
#pragma unroll
    for (int l = 0; l < SIZE / WR; ++l) s += red[g * (SIZE / WR) + l][c];
    const long long grow = row0 + (long long)g * SIZE;
    const long long n = std::max<long long>(0, std::min<long long>(SIZE, N - grow));
    const long long gidx = (long long)blk * G + g;
    const float mean = n > 0 ? s / (float)n : 0.f;
    const long long row = bh * (Npad / SIZE) + gidx;
    if (out != nullptr) out[row * D + c] = mean;
    if (split != nullptr) {
      if (!(fabsf(mean) <= 65504.f)) atomicOr(&g_pool_flags, kFlagRangeMean);
      const __half hi = __float2half_rn(fminf(fmaxf(mean, -65504.f), 65504.f));
      split[row * 2 * D + c] = hi;
      split[row * 2 * D + D + c] = __float2half_rn(fminf(fmaxf(mean - __half2float(hi), -65504.f), 65504.f));
    }
    if (split_bf != nullptr) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
      split_bf[row * 2 * D + c] = hi;
      split_bf[row * 2 * D + D + c] = __float2bfloat16_rn(mean - __bfloat162float(hi));
    }
    if (nvalid != nullptr && bh == 0 && c == 0) nvalid[gidx] = (int32_t)n;
  }
}

__global__ void nvalid_kernel(int32_t* __restrict__ nvalid, long long N, int nb) {
  for (int J = blockIdx.x * blockDim.x + threadIdx.x; J < nb; J += gridDim.x * blockDim.x)
    nvalid[J] = (int32_t)std::max<long long>(0, std::min<long long>(kBlock, N - (long long)J * kBlock));
}

cudaError_t launch_nvalid(int32_t* nvalid, long long N, int nb, cudaStream_t st) {
  nvalid_kernel<<<(nb + 255) / 256, 256, 0, st>>>(nvalid, N, nb);
  return cudaGetLastError();
}

template <typename T2>
static cudaError_t launch_pool_t(const void* xp, float* out, void* split, void* split_bf, int32_t* nvalid,
                                 long long BH, long long N, long long Npad, int d, int size, cudaStream_t st) {
  dim3 grid((unsigned)(Npad / kBlock), (unsigned)BH);
  const T2* x = reinterpret_cast<const T2*>(xp);
  __half* sp = reinterpret_cast<__half*>(split);
  __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(split_bf);
#define SVSA_POOL(DD, SS) pool_kernel<DD, SS, T2><<<grid, kPoolThreads, 0, st>>>(x, out, sp, sb, nvalid, N, Npad)
  if (d == 128 && size == 64) SVSA_POOL(128, 64);
  else if (d == 128 && size == 16) SVSA_POOL(128, 16);
  else if (d == 64 && size == 64) SVSA_POOL(64, 64);
  else if (d == 64 && size == 16) SVSA_POOL(64, 16);
  else return cudaErrorInvalidValue;
#undef SVSA_POOL
  return cudaGetLastError();
}

// bf16 input (queries, keys); `out` (fp32 means), `split` (fp16 hi | lo) and
// `split_bf` (bf16 hi | lo) are each nullable
cudaError_t launch_pool(const void* xp, float* out, void* split, void* split_bf, int32_t* nvalid, long long BH,
                        long long N, long long Npad, int d, int size, cudaStream_t st) {
  return launch_pool_t<__nv_bfloat162>(xp, out, split, split_bf, nvalid, BH, N, Npad, d, size, st);
}

// fp16 input (reordered values)
cudaError_t launch_pool_f16(const void* xp, float* out, int32_t* nvalid, long long BH, long long N,
                            long long Npad, int d, int size, cudaStream_t st) {
  return launch_pool_t<__half2>(xp, out, nullptr, nullptr, nvalid, BH, N, Npad, d, size, st);
}

// 16-bit centroid rows for the tensor-core compensation: row r of cbar is
// [kbar_r as bf16 (d) | vbar_r as fp16 (d)], both rounded to nearest even.
__global__ void centroid16_kernel(const float4* __restrict__ kbar, const float4* __restrict__ vbar,
                                  uint2* __restrict__ cbar, long long rows, int d4) {
  const long long total = rows * d4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / d4;
    const int c = (int)(i % d4);
    const float4 kv = kbar[i], vv = vbar[i];
    __nv_bfloat162 k01 = __floats2bfloat162_rn(kv.x, kv.y), k23 = __floats2bfloat162_rn(kv.z, kv.w);
    __half2 v01 = __floats2half2_rn(vv.x, vv.y), v23 = __floats2half2_rn(vv.z, vv.w);
    cbar[r * 2 * d4 + c] = make_uint2(*reinterpret_cast<uint32_t*>(&k01), *reinterpret_cast<uint32_t*>(&k23));
    cbar[r * 2 * d4 + d4 + c] = make_uint2(*reinterpret_cast<uint32_t*>(&v01), *reinterpret_cast<uint32_t*>(&v23));
  }
}

cudaError_t launch_centroid16(const float* kbar, const float* vbar, void* cbar, long long rows, int d,
                              cudaStream_t st) {
  const long long total = rows * (d / 4);
  const int blocks = (int)std::min<long long>((total + 255) / 256, 148LL * 16);
  centroid16_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4*>(kbar),
                                            reinterpret_cast<const float4*>(vbar), reinterpret_cast<uint2*>(cbar),
                                            rows, d / 4);
  return cudaGetLastError();
}

cudaError_t pool_flags(unsigned int* v, cudaStream_t st) { return read_and_clear_flags(g_pool_flags, v, st); }

}  // namespace svsa
