// Row gathers between raster order and the reordered, padded layout.
//
// Forward  ("DFSAttn", trick 1):  xp[bh, i, :] = x[bh, perm[i], :]   (zeros where perm[i] < 0)
// Inverse:                        o[bh, r, :]  = op[bh, iperm[r], :]
// The map is shared by all (batch, head) rows (map_stride = 0) or given per
// row (map_stride = its length), as the semantic orders are.
// The value tensor's forward gather also converts bf16 -> fp16 (the P.V
// product runs in fp16).
//
// Both are pure data movement (HBM-bound): every thread moves 16-byte chunks,
// consecutive threads cover consecutive bytes of the destination (coalesced
// stores) and a source row (128 or 256 bytes) is read whole by 8 or 16
// neighbouring threads.  Each thread issues kUnroll independent loads before
// its stores to keep enough bytes in flight.
#include "common.cuh"

namespace svsa {

constexpr int kGatherThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// grid.y = bh; grid.x covers rows_dst * chunks-per-row in tiles of
// kGatherThreads * kUnroll chunks.
template <int CPR>
__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, const int32_t* __restrict__ map_all,
    long long map_stride, long long rows_dst, long long rows_src) {
  const long long bh = blockIdx.y;
  const int32_t* map = map_all + bh * map_stride;
  const long long total = rows_dst * CPR;
  const uint4* s_base = src + bh * rows_src * CPR;
  uint4* d_base = dst + bh * rows_dst * CPR;
  const long long tile = (long long)kGatherThreads * kUnroll;
  for (long long base = (long long)blockIdx.x * tile; base < total; base += (long long)gridDim.x * tile) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long c = base + u * kGatherThreads + threadIdx.x;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (c < total) {
        const int32_t srow = __ldg(map + c / CPR);
        if (srow >= 0) v[u] = ld_stream(s_base + (long long)srow * CPR + (c % CPR));
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long c = base + u * kGatherThreads + threadIdx.x;
      if (c < total) d_base[c] = v[u];
    }
  }
}

// Status bits of this translation unit (kFlagRangeValue: a value given to the
// fp16 gather lies beyond the fp16 range or is not finite).
static __device__ unsigned int g_reorder_flags;

// True when one of the 8 bf16 values of a chunk is beyond fp16's range or
// not finite: |x| >= 65536 (the bf16 value after 65280 is 65536) is an
// exponent field >= 143, i.e. magnitude bits > 0x477F.
__device__ __forceinline__ bool bf16x8_out_of_f16(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  bool bad = false;
#pragma unroll
  for (int e = 0; e < 4; ++e) bad |= (w[e] & 0x7FFFu) > 0x477Fu || ((w[e] >> 16) & 0x7FFFu) > 0x477Fu;
  return bad;
}

// bf16 -> fp16 conversion of one 16-byte chunk (8 values), saturating at
// +-65504; exact for every bf16 value in fp16's normal range.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
  uint4 out;
  uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(b[e]);
    uint32_t h;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;\n" : "=r"(h) : "f"(f.y), "f"(f.x));
    o[e] = h;
  }
  return out;
}

template <int CPR>
__global__ void __launch_bounds__(kGatherThreads) gather_rows_f16_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, const int32_t* __restrict__ map_all,
    long long map_stride, long long rows_dst, long long rows_src) {
  const long long bh = blockIdx.y;
  const int32_t* map = map_all + bh * map_stride;
  const long long total = rows_dst * CPR;
  const uint4* s_base = src + bh * rows_src * CPR;
  uint4* d_base = dst + bh * rows_dst * CPR;
  const long long tile = (long long)kGatherThreads * kUnroll;
  for (long long base = (long long)blockIdx.x * tile; base < total; base += (long long)gridDim.x * tile) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long c = base + u * kGatherThreads + threadIdx.x;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (c < total) {
        const int32_t srow = __ldg(map + c / CPR);
        if (srow >= 0) v[u] = ld_stream(s_base + (long long)srow * CPR + (c % CPR));
      }
    }
    bool bad = false;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long c = base + u * kGatherThreads + threadIdx.x;
      if (c < total) d_base[c] = bf16x8_to_f16x8(v[u]);
      bad |= bf16x8_out_of_f16(v[u]);          // (zero chunks never flag)
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_reorder_flags, kFlagRangeValue);
  }
}

cudaError_t launch_gather_rows_f16(const void* src, void* dst, const int32_t* map, long long map_stride,
                                   long long BH, long long rows_dst, long long rows_src, int d, cudaStream_t st) {
  const int cpr = d * 2 / 16;
  const long long total = rows_dst * cpr;
  const long long tile = (long long)kGatherThreads * kUnroll;
  const long long gx = std::max<long long>(1, (total + tile - 1) / tile);
  dim3 grid((unsigned)gx, (unsigned)BH);
  if (cpr == 16)
    gather_rows_f16_kernel<16><<<grid, kGatherThreads, 0, st>>>((const uint4*)src, (uint4*)dst, map, map_stride, rows_dst, rows_src);
  else if (cpr == 8)
    gather_rows_f16_kernel<8><<<grid, kGatherThreads, 0, st>>>((const uint4*)src, (uint4*)dst, map, map_stride, rows_dst, rows_src);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, void* dst, const int32_t* map, long long map_stride, long long BH,
                               long long rows_dst, long long rows_src, int d, cudaStream_t st) {
  const int cpr = d * 2 / 16;
  const long long total = rows_dst * cpr;
  const long long tile = (long long)kGatherThreads * kUnroll;
  const long long gx = std::max<long long>(1, (total + tile - 1) / tile);
  dim3 grid((unsigned)gx, (unsigned)BH);
  if (cpr == 16)
    gather_rows_kernel<16><<<grid, kGatherThreads, 0, st>>>(
        (const uint4*)src, (uint4*)dst, map, map_stride, rows_dst, rows_src);
  else if (cpr == 8)
    gather_rows_kernel<8><<<grid, kGatherThreads, 0, st>>>(
        (const uint4*)src, (uint4*)dst, map, map_stride, rows_dst, rows_src);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t reorder_flags(unsigned int* v, cudaStream_t st) { return read_and_clear_flags(g_reorder_flags, v, st); }

}  // namespace svsa
