// Token order of the (T, H, W) latent grid: raster identity or 3D Hilbert.
//
// "DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
// Generation", trick 1: the tokens are threaded along a 3D Hilbert curve so
// that neighbours in the sequence are neighbours in space and time.  The grid
// is cropped from the enclosing 2^k cube; a cell's position on the curve is
// computed with Skilling's transpose method (J. Skilling, "Programming the
// Hilbert curve", AIP Conf. Proc. 707, 2004), axes (t, h, w).
//
// The sort of the N valid cells by curve index is a rank by bitmap: one bit
// per cube cell, a per-word prefix count and a per-chunk prefix count give
// each cell its rank with no comparison sort, deterministically.
#include "common.cuh"

namespace svsa {

constexpr int kChunkWords = 1024;   // bitmap words per scan chunk (one CTA)

// Curve index of cell (t, h, w) in the 2^k cube, k <= 10 (30-bit result).
__device__ __forceinline__ uint32_t hilbert_index(uint32_t t, uint32_t h, uint32_t w, int k) {
  if (k <= 0) return 0u;
  uint32_t x0 = t, x1 = h, x2 = w;
  const uint32_t top = 1u << (k - 1);
  // Stage 1: undo the rotations/reflections plane by plane, top plane first.
  for (uint32_t q = top; q > 1u; q >>= 1) {
    const uint32_t lo = q - 1u;
    if (x0 & q) x0 ^= lo;                         // axis 0 against itself: invert only
    if (x1 & q) { x0 ^= lo; } else { uint32_t s = (x0 ^ x1) & lo; x0 ^= s; x1 ^= s; }
    if (x2 & q) { x0 ^= lo; } else { uint32_t s = (x0 ^ x2) & lo; x0 ^= s; x2 ^= s; }
  }
  // Stage 2: Gray encode across the axes.
  x1 ^= x0;
  x2 ^= x1;
  uint32_t flip = 0u;
  for (uint32_t q = top; q > 1u; q >>= 1)
    if (x2 & q) flip ^= (q - 1u);
  x0 ^= flip; x1 ^= flip; x2 ^= flip;
  // Interleave: plane by plane from the top, axis 0 first.
  uint32_t key = 0u;
  for (int b = k - 1; b >= 0; --b) {
    key = (key << 1) | ((x0 >> b) & 1u);
    key = (key << 1) | ((x1 >> b) & 1u);
    key = (key << 1) | ((x2 >> b) & 1u);
  }
  return key;
}

__global__ void perm_raster_kernel(int32_t* perm, int32_t* iperm, long long N, long long Npad) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < Npad;
       i += (long long)gridDim.x * blockDim.x) {
    perm[i] = i < N ? (int32_t)i : -1;
    if (i < N) iperm[i] = (int32_t)i;
  }
}

__global__ void bitmap_clear_kernel(uint32_t* bits, long long words) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < words;
       i += (long long)gridDim.x * blockDim.x)
    bits[i] = 0u;
}

__global__ void hilbert_mark_kernel(int T, int H, int W, int k, uint32_t* bits) {
  const long long N = (long long)T * H * W;
  for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < N;
       r += (long long)gridDim.x * blockDim.x) {
    const uint32_t w = (uint32_t)(r % W);
    const uint32_t h = (uint32_t)((r / W) % H);
    const uint32_t t = (uint32_t)(r / ((long long)W * H));
    const uint32_t key = hilbert_index(t, h, w, k);
    atomicOr(&bits[key >> 5], 1u << (key & 31u));
  }
}

// One CTA of kChunkWords threads per chunk: exclusive prefix of popcounts
// within the chunk, and the chunk total.
__global__ void __launch_bounds__(kChunkWords) bitmap_scan_words_kernel(
    const uint32_t* bits, uint32_t* word_prefix, uint32_t* chunk_total, long long words) {
  __shared__ uint32_t warp_tot[kChunkWords / 32];
  const long long w = (long long)blockIdx.x * kChunkWords + threadIdx.x;
  const uint32_t c = w < words ? (uint32_t)__popc(bits[w]) : 0u;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    uint32_t v = warp_tot[lane];
    uint32_t vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += y;
    }
    warp_tot[lane] = vi - v;                      // exclusive over warps
    if (lane == 31) chunk_total[blockIdx.x] = vi;
  }
  __syncthreads();
  if (w < words) word_prefix[w] = warp_tot[wid] + incl - c;
}

// Single CTA: exclusive prefix over the chunk totals, in place.
__global__ void __launch_bounds__(1024) bitmap_scan_chunks_kernel(uint32_t* chunk_total, int nchunks) {
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t carry;
  if (threadIdx.x == 0) carry = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < nchunks; base += 1024) {
    const int i = base + threadIdx.x;
    const uint32_t c = i < nchunks ? chunk_total[i] : 0u;
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      uint32_t v = warp_tot[lane], vi = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, vi, o);
        if (lane >= o) vi += y;
      }
      warp_tot[lane] = vi - v;
    }
    __syncthreads();
    const uint32_t excl = carry + warp_tot[wid] + incl - c;
    __syncthreads();
    if (i < nchunks) chunk_total[i] = excl;
    if (threadIdx.x == 1023) carry = excl + c;
    __syncthreads();
  }
}

__global__ void hilbert_assign_kernel(int T, int H, int W, int k, const uint32_t* bits,
                                      const uint32_t* word_prefix, const uint32_t* chunk_prefix,
                                      int32_t* perm, int32_t* iperm, long long Npad) {
  const long long N = (long long)T * H * W;
  for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < Npad;
       r += (long long)gridDim.x * blockDim.x) {
    if (r >= N) { perm[r] = -1; continue; }
    const uint32_t w = (uint32_t)(r % W);
    const uint32_t h = (uint32_t)((r / W) % H);
    const uint32_t t = (uint32_t)(r / ((long long)W * H));
    const uint32_t key = hilbert_index(t, h, w, k);
    const uint32_t word = key >> 5, bit = key & 31u;
    const uint32_t below = bit ? (bits[word] & ((1u << bit) - 1u)) : 0u;
    const uint32_t rank = chunk_prefix[word / kChunkWords] + word_prefix[word] + (uint32_t)__popc(below);
    perm[rank] = (int32_t)r;
    iperm[r] = (int32_t)rank;
  }
}

int hilbert_order_bits(int T, int H, int W) {
  int m = T > H ? T : H;
  m = m > W ? m : W;
  int k = 0;
  while ((1 << k) < m) ++k;
  return k;
}

// Workspace layout for the Hilbert build: bitmap | word prefix | chunk prefix.
size_t perm_workspace_bytes(int T, int H, int W) {
  const int k = hilbert_order_bits(T, H, W);
  const long long cells = 1LL << (3 * k);
  const long long words = (cells + 31) / 32;
  const long long chunks = (words + kChunkWords - 1) / kChunkWords;
  return (size_t)(words * 4 + words * 4 + chunks * 4 + 256);
}

cudaError_t launch_build_perm(int T, int H, int W, int hilbert, int32_t* perm, int32_t* iperm,
                              void* ws, cudaStream_t st) {
  const long long N = (long long)T * H * W;
  const long long Npad = ((N + kBlock - 1) / kBlock) * kBlock;
  const int threads = 256;
  if (!hilbert) {
    const int grid = (int)std::min<long long>((Npad + threads - 1) / threads, kNumSMs * 16LL);
    perm_raster_kernel<<<grid, threads, 0, st>>>(perm, iperm, N, Npad);
    return cudaGetLastError();
  }
  const int k = hilbert_order_bits(T, H, W);
  const long long cells = 1LL << (3 * k);
  const long long words = (cells + 31) / 32;
  const long long chunks = (words + kChunkWords - 1) / kChunkWords;
  uint32_t* bits = reinterpret_cast<uint32_t*>(ws);
  uint32_t* word_prefix = bits + words;
  uint32_t* chunk_prefix = word_prefix + words;
  const int g1 = (int)std::min<long long>((words + threads - 1) / threads, kNumSMs * 16LL);
  bitmap_clear_kernel<<<g1, threads, 0, st>>>(bits, words);
  const int g2 = (int)std::min<long long>((N + threads - 1) / threads, kNumSMs * 16LL);
  hilbert_mark_kernel<<<g2, threads, 0, st>>>(T, H, W, k, bits);
  bitmap_scan_words_kernel<<<(unsigned)chunks, kChunkWords, 0, st>>>(bits, word_prefix, chunk_prefix, words);
  bitmap_scan_chunks_kernel<<<1, 1024, 0, st>>>(chunk_prefix, (int)chunks);
  const int g3 = (int)std::min<long long>((Npad + threads - 1) / threads, kNumSMs * 16LL);
  hilbert_assign_kernel<<<g3, threads, 0, st>>>(T, H, W, k, bits, word_prefix, chunk_prefix, perm, iperm, Npad);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- no-allocation variant
// Scratch of svsa_build_perm_noalloc, for callers that cannot allocate device
// memory: one file-scope array per device that loads the library, sized for
// grids whose longest side is at most 2^kNoAllocMaxBits (128).  Layout as in
// perm_workspace_bytes: bitmap | word prefix | chunk prefix.
constexpr int kNoAllocMaxBits = 7;
constexpr long long kNoAllocWords = (1LL << (3 * kNoAllocMaxBits)) / 32;
constexpr long long kNoAllocChunks = (kNoAllocWords + kChunkWords - 1) / kChunkWords;
constexpr size_t kNoAllocScratchBytes = (size_t)(kNoAllocWords * 4 * 2 + kNoAllocChunks * 4 + 256);
static __device__ __align__(256) unsigned char g_perm_scratch[kNoAllocScratchBytes];

int perm_noalloc_max_bits() { return kNoAllocMaxBits; }
size_t perm_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of g_perm_scratch in the current context.  It is looked up
// on every call (cudaGetSymbolAddress, a host-side query once the module is
// loaded) rather than cached: a cached address would go stale if the
// device's primary context were reset and the module loaded again.  The
// first call on a device loads the module, so make it before any stream
// capture.
cudaError_t perm_noalloc_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_perm_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace svsa
