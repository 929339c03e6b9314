// Query-block pairing for the 128-row attention items.
//
// The attention processes two 64-row query blocks per item and walks the
// union of their kept lists, so a pair costs |A u B| = |A| + |B| - |A n B|
// key blocks: the fewer blocks the two lists share, the more tensor work is
// spent on masked quarters.  The query blocks of every head are ordered so
// that consecutive entries (the items) share many kept blocks: a greedy walk
// takes the first block not yet paired and gives it, of the unpaired blocks
// among the next kPairWin indices, the one with the largest intersection
// (ties to the lower index); when all of those are taken it pairs it with
// the first unpaired block after it.  With a token order that keeps
// space-time neighbours close (Hilbert), the best partners are usually
// within that window.  The result is a permutation of 0..nb-1 per head; an
// odd nb leaves the last entry unpaired.
//
// pair_score_kernel  one warp per query block I: |row I AND row I + 1 + c|
//                    of the kept-block bitmaps for c < kPairWin, into a
//                    [BH, nb, kPairWin] int16 table (fully parallel)
// pair_walk_kernel   one warp per head: the greedy walk over that table,
//                    with the unpaired blocks as a bitmap in shared memory
#include "common.cuh"

namespace svsa {

constexpr int kPairWin = 32;

__global__ void __launch_bounds__(256) pair_score_kernel(const uint32_t* __restrict__ bits, int nb, int words,
                                                         int16_t* __restrict__ tab) {
  const int I = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  if (I >= nb) return;
  const uint32_t* rows = bits + bh * (long long)nb * words;
  const uint32_t* ri = rows + (long long)I * words;
  int16_t* out = tab + (bh * nb + I) * kPairWin;
  for (int c = 0; c < kPairWin; ++c) {
    const int J = I + 1 + c;
    int cnt = 0;
    if (J < nb) {
      const uint32_t* rj = rows + (long long)J * words;
      for (int w = lane; w < words; w += 32) cnt += __popc(ri[w] & rj[w]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) out[c] = (int16_t)(J < nb ? (cnt < 32767 ? cnt : 32767) : -1);
  }
}

// first unpaired block >= from (nb if none), all lanes agree
__device__ __forceinline__ int first_free(const uint32_t* used, int from, int nb) {
  const int lane = threadIdx.x & 31;
  const int words = (nb + 31) / 32;
  for (int w0 = from >> 5; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    uint32_t free_bits = 0u;
    if (w < words) {
      free_bits = ~used[w];
      if (w == (from >> 5)) free_bits &= ~0u << (from & 31);       // below `from`
      if (w == words - 1 && (nb & 31)) free_bits &= (1u << (nb & 31)) - 1u;
    }
    const uint32_t any = __ballot_sync(0xffffffffu, free_bits != 0u);
    if (any) {
      const int src = __ffs(any) - 1;
      const uint32_t fb = __shfl_sync(0xffffffffu, free_bits, src);
      return (w0 + src) * 32 + __ffs(fb) - 1;
    }
  }
  return nb;
}

__global__ void __launch_bounds__(32) pair_walk_kernel(const int16_t* __restrict__ tab, int nb,
                                                       int32_t* __restrict__ pairs) {
  extern __shared__ uint32_t used[];            // ceil(nb / 32) words, bit set = paired
  const long long bh = blockIdx.x;
  const int lane = threadIdx.x;
  const int words = (nb + 31) / 32;
  for (int w = lane; w < words; w += 32) used[w] = 0u;
  __syncwarp();
  int32_t* out = pairs + bh * nb;
  const int16_t* t = tab + bh * (long long)nb * kPairWin;
  int pos = 0, I = 0;
  while (true) {
    I = first_free(used, I, nb);
    if (I >= nb) break;
    // lane c: candidate J = I + 1 + c if it exists and is unpaired
    const int J = I + 1 + lane;
    int sc = -1;
    if (J < nb && !((used[J >> 5] >> (J & 31)) & 1u)) sc = t[(long long)I * kPairWin + lane];
    // warp argmax, ties to the lower index
    int best = sc, bj = sc >= 0 ? J : INT32_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const int ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ob > best || (ob == best && oj < bj)) {
        best = ob;
        bj = oj;
      }
    }
    if (best < 0) bj = first_free(used, I + 1, nb);     // window all taken: the next unpaired block
    __syncwarp();
    if (lane == 0) {
      out[pos] = I;
      used[I >> 5] |= 1u << (I & 31);
      if (bj < nb) {
        out[pos + 1] = bj;
        used[bj >> 5] |= 1u << (bj & 31);
      }
    }
    pos += bj < nb ? 2 : 1;
    __syncwarp();
  }
}

size_t pair_table_bytes(long long BH, int nb) { return (size_t)BH * nb * kPairWin * sizeof(int16_t); }

cudaError_t launch_pair(const uint32_t* bits, long long BH, int nb, int16_t* tab, int32_t* pairs,
                        cudaStream_t st) {
  const int words = (nb + 31) / 32;
  dim3 g1((unsigned)((nb + 7) / 8), (unsigned)BH);
  pair_score_kernel<<<g1, 256, 0, st>>>(bits, nb, words, tab);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pair_walk_kernel<<<(unsigned)BH, 32, (size_t)words * sizeof(uint32_t), st>>>(tab, nb, pairs);
  return cudaGetLastError();
}

}  // namespace svsa
