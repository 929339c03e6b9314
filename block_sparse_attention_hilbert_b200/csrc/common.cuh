// Shared device/host helpers of libsvsa (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

namespace svsa {

constexpr int kBlock = 64;          // tokens per mask block
constexpr int kNumSMs = 148;        // B200

struct Dims {
  int B, heads, T, H, W, d;
  long long N, Npad;
  int nb;
  long long BH;
};

inline Dims make_dims(int B, int heads, int T, int H, int W, int d) {
  Dims g;
  g.B = B; g.heads = heads; g.T = T; g.H = H; g.W = W; g.d = d;
  g.N = (long long)T * H * W;
  g.nb = (int)((g.N + kBlock - 1) / kBlock);
  g.Npad = (long long)g.nb * kBlock;
  g.BH = (long long)B * heads;
  return g;
}

__host__ __device__ inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// Round-to-nearest-even float -> bf16 pair packed in a uint32 (lo = a, hi = b).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Status bits that kernels OR into a word of their translation unit (each
// unit that raises one keeps a static word and a reader): bit 0 = a value
// beyond the fp16 range in a bf16 -> fp16 conversion, bit 1 = a block mean
// beyond the fp16 range in the scores' split, bit 2 = a malformed mask list.
constexpr unsigned int kFlagRangeValue = 1u, kFlagRangeMean = 2u, kFlagMask = 4u;

// Read a status word of the calling translation unit and clear it.
template <typename Word>
inline cudaError_t read_and_clear_flags(const Word& word, unsigned int* v, cudaStream_t st) {
  unsigned int zero = 0u;
  cudaError_t e = cudaMemcpyFromSymbolAsync(v, word, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  if (*v != 0u) {
    e = cudaMemcpyToSymbolAsync(word, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(st);
  }
  return e;
}

}  // namespace svsa
