// Block-sparse attention with warp-level bf16 MMAs (mma.sync m16n8k16).
//
// "SVG-EAR", problem statement: the sparse kernel computes only a subset of
// the attention blocks; 2.A: with compensation every skipped block J enters
// the same softmax as n_J copies of its centroid (kbar_J, vbar_J).
//
// Q and K are bf16, the reordered values fp16 (P is rounded to fp16 for the
// P.V product, whose 11-bit significand keeps the softmax weights 8x more
// precise than bf16 would).
//
// One CTA = one 64-row query block (the mask's granularity, so no tile is
// wasted), 4 warps x 16 query rows.  The kept key blocks are streamed through
// a double-buffered, XOR-swizzled shared-memory ring with cp.async; S = Q K^T
// and O += P V run on mma.sync with fp32 accumulators; the online softmax
// keeps a running max / sum per row in the log2 domain; P is rounded to fp16
// in registers and fed straight back as the A operand.  Compensation appends
// ceil(nb / 64) centroid tiles whose columns carry the bias log2(n_J) for
// skipped blocks and -inf for kept ones.  DENSE visits every key block.
#include <cuda_fp16.h>

#include "common.cuh"

namespace svsa {

constexpr int kMmaThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float fast_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Element offset of 16-byte chunk `c` of row `r` in a [64][D] bf16 tile.
template <int D>
__device__ __forceinline__ int swz(int r, int c) {
  return r * D + ((c ^ (r & 7)) << 3);
}

__device__ __forceinline__ int clamp_block(int J, int nb) { return J < 0 ? 0 : (J >= nb ? nb - 1 : J); }

struct AttnArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __half* v;
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  int cap;
  const float* kbar;
  const float* vbar;
  const int32_t* nvalid;
  __nv_bfloat16* o;
  float* lse;
  long long N, Npad;
  int nb;
  float scale_log2;
};

template <int D>
__device__ __forceinline__ void load_tile_async(__nv_bfloat16* dst, const __nv_bfloat16* src, int tid) {
  constexpr int CPR = D / 8;
#pragma unroll
  for (int i = 0; i < kBlock * CPR / kMmaThreads; ++i) {
    const int id = tid + i * kMmaThreads;
    const int r = id / CPR, c = id % CPR;
    cp_async16(smem_u32(dst + swz<D>(r, c)), src + (long long)r * D + c * 8);
  }
}

// Centroid rows J0 .. J0+63 (fp32) -> bf16 (keys) or fp16 (values) tile; rows past nb are zero.
template <int D, bool F16>
__device__ __forceinline__ void load_centroid_tile(__nv_bfloat16* dst, const float* src, int J0, int nb, int tid) {
  constexpr int CPR = D / 8;
#pragma unroll
  for (int i = 0; i < kBlock * CPR / kMmaThreads; ++i) {
    const int id = tid + i * kMmaThreads;
    const int r = id / CPR, c = id % CPR;
    uint4 packed = make_uint4(0u, 0u, 0u, 0u);
    if (J0 + r < nb) {
      const float4 a = *reinterpret_cast<const float4*>(src + (long long)(J0 + r) * D + c * 8);
      const float4 b = *reinterpret_cast<const float4*>(src + (long long)(J0 + r) * D + c * 8 + 4);
      if (F16) {
        packed.x = pack_f16x2(a.x, a.y); packed.y = pack_f16x2(a.z, a.w);
        packed.z = pack_f16x2(b.x, b.y); packed.w = pack_f16x2(b.z, b.w);
      } else {
        packed.x = pack_bf16x2(a.x, a.y); packed.y = pack_bf16x2(a.z, a.w);
        packed.z = pack_bf16x2(b.x, b.y); packed.w = pack_bf16x2(b.z, b.w);
      }
    }
    *reinterpret_cast<uint4*>(dst + swz<D>(r, c)) = packed;
  }
}

template <int D, bool DENSE, bool COMP>
__global__ void __launch_bounds__(kMmaThreads, 2) attn_mma_kernel(const AttnArgs a) {
  constexpr int KT = D / 16;         // k-steps over the head dim
  constexpr int DT = D / 8;          // n-tiles over the head dim
  constexpr int TILE = kBlock * D;   // elements per tile
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* Ks = Qs + TILE;          // [2][TILE]
  __nv_bfloat16* Vs = Ks + 2 * TILE;      // [2][TILE]
  uint8_t* kept = reinterpret_cast<uint8_t*>(Vs + 2 * TILE);   // [nb] (COMP)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const long long bh = blockIdx.y;
  const int I = blockIdx.x;
  const int nb = a.nb;
  const long long rowbase = bh * a.Npad;
  const __nv_bfloat16* qg = a.q + (rowbase + (long long)I * kBlock) * D;
  const __nv_bfloat16* kg = a.k + rowbase * D;
  const __nv_bfloat16* vg = reinterpret_cast<const __nv_bfloat16*>(a.v) + rowbase * D;   // fp16 bits
  const int32_t* list = DENSE ? nullptr : a.kv_idx + (bh * nb + I) * (long long)a.cap;
  // a caller-supplied list is trusted for order, not for range: the count is
  // clamped to the row capacity and entries outside [0, nb) are masked out
  const int cnt = DENSE ? nb : min(max(a.kv_cnt[bh * nb + I], 0), a.cap);
  const int ncent = COMP ? (nb + kBlock - 1) / kBlock : 0;
  const int total = cnt + ncent;
  const float* kbar_h = COMP ? a.kbar + bh * (long long)nb * D : nullptr;
  const float* vbar_h = COMP ? a.vbar + bh * (long long)nb * D : nullptr;

  if (COMP) {
    for (int j = tid; j < nb; j += kMmaThreads) kept[j] = 0;
    __syncthreads();
    for (int j = tid; j < cnt; j += kMmaThreads) {
      const int J = list[j];
      if (J >= 0 && J < nb) kept[J] = 1;
    }
  }

  auto issue = [&](int t, int buf) {
    if (t < cnt) {
      const int J = DENSE ? t : clamp_block(list[t], nb);
      load_tile_async<D>(Ks + buf * TILE, kg + (long long)J * kBlock * D, tid);
      load_tile_async<D>(Vs + buf * TILE, vg + (long long)J * kBlock * D, tid);
    } else if (COMP) {
      const int J0 = (t - cnt) * kBlock;
      load_centroid_tile<D, false>(Ks + buf * TILE, kbar_h, J0, nb, tid);
      load_centroid_tile<D, true>(Vs + buf * TILE, vbar_h, J0, nb, tid);
    }
  };

  load_tile_async<D>(Qs, qg, tid);
  if (total > 0) issue(0, 0);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  uint32_t qf[KT][4];
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
    const int r = warp * 16 + (lane & 15);
    const int c = 2 * kk + (lane >> 4);
    ldsm_x4(smem_u32(Qs + swz<D>(r, c)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
  }

  float o[DT][4];
#pragma unroll
  for (int j = 0; j < DT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale_log2;

  for (int t = 0; t < total; ++t) {
    const int buf = t & 1;
    if (t + 1 < total) issue(t + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const __nv_bfloat16* Kt = Ks + buf * TILE;
    const __nv_bfloat16* Vt = Vs + buf * TILE;
    const bool cent = COMP && t >= cnt;

    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int r = 16 * np + (lane & 7) + ((lane >> 4) << 3);
        const int c = 2 * kk + ((lane >> 3) & 1);
        ldsm_x4(smem_u32(Kt + swz<D>(r, c)), b0, b1, b2, b3);
        mma16816(s[2 * np], qf[kk], b0, b1);
        mma16816(s[2 * np + 1], qf[kk], b2, b3);
      }
    }

    // scaled logits in the log2 domain, with masking / centroid bias
    if (cent) {
      const int J0 = (t - cnt) * kBlock;
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int J = J0 + 8 * n + 2 * t4 + e;
          float bias = -INFINITY;
          if (J < nb && !kept[J]) bias = __log2f((float)a.nvalid[J]);
          s[n][e] = bias == -INFINITY ? -INFINITY : fmaf(s[n][e], sl2, bias);
          s[n][e + 2] = bias == -INFINITY ? -INFINITY : fmaf(s[n][e + 2], sl2, bias);
        }
    } else {
      const int Jraw = DENSE ? t : list[t];
      const bool in_range = DENSE || (Jraw >= 0 && Jraw < nb);
      const long long key0 = (long long)clamp_block(Jraw, nb) * kBlock;
      const bool ragged = !in_range || key0 + kBlock > a.N;
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool ok = !ragged || (in_range && key0 + 8 * n + 2 * t4 + e < a.N);
          s[n][e] = ok ? s[n][e] * sl2 : -INFINITY;
          s[n][e + 2] = ok ? s[n][e + 2] * sl2 : -INFINITY;
        }
    }

    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
      mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
    const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = fast_ex2(m0 - mu0), c1 = fast_ex2(m1 - mu1);
    m0 = mn0; m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pa[4][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float p0 = fast_ex2(s[n][0] - mu0), p1 = fast_ex2(s[n][1] - mu0);
      const float p2 = fast_ex2(s[n][2] - mu1), p3 = fast_ex2(s[n][3] - mu1);
      rs0 += p0 + p1;
      rs1 += p2 + p3;
      pa[n >> 1][(n & 1) * 2 + 0] = pack_f16x2(p0, p1);
      pa[n >> 1][(n & 1) * 2 + 1] = pack_f16x2(p2, p3);
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
#pragma unroll
    for (int j = 0; j < DT; ++j) {
      o[j][0] *= c0; o[j][1] *= c0;
      o[j][2] *= c1; o[j][3] *= c1;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dp = 0; dp < DT / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int r = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = 2 * dp + (lane >> 4);
        ldsm_x4_t(smem_u32(Vt + swz<D>(r, c)), b0, b1, b2, b3);
        mma16816_f16(o[2 * dp], pa[kk], b0, b1);
        mma16816_f16(o[2 * dp + 1], pa[kk], b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // finish: row sums across the quad, normalise, stage through shared memory
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const int r0 = warp * 16 + g, r1 = r0 + 8;
  const long long q0 = (long long)I * kBlock;
#pragma unroll
  for (int j = 0; j < DT; ++j) {
    const int col = 8 * j + 2 * t4;
    *reinterpret_cast<uint32_t*>(Qs + swz<D>(r0, j) + 2 * t4) = pack_bf16x2(o[j][0] * inv0, o[j][1] * inv0);
    *reinterpret_cast<uint32_t*>(Qs + swz<D>(r1, j) + 2 * t4) = pack_bf16x2(o[j][2] * inv1, o[j][3] * inv1);
    (void)col;
  }
  if (a.lse != nullptr && t4 == 0) {
    const float ln2 = 0.6931471805599453f;
    a.lse[rowbase + q0 + r0] = (q0 + r0 < a.N && l0 > 0.f) ? (m0 + __log2f(l0)) * ln2 : 0.f;
    a.lse[rowbase + q0 + r1] = (q0 + r1 < a.N && l1 > 0.f) ? (m1 + __log2f(l1)) * ln2 : 0.f;
  }
  __syncthreads();
  __nv_bfloat16* og = a.o + (rowbase + q0) * D;
  constexpr int CPR = D / 8;
#pragma unroll
  for (int i = 0; i < kBlock * CPR / kMmaThreads; ++i) {
    const int id = tid + i * kMmaThreads;
    const int r = id / CPR, c = id % CPR;
    uint4 v = *reinterpret_cast<const uint4*>(Qs + swz<D>(r, c));
    if (q0 + r >= a.N) v = make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(og + (long long)r * D + c * 8) = v;
  }
}

size_t attn_mma_smem_bytes(int d, int nb, bool comp) {
  return (size_t)5 * kBlock * d * sizeof(__nv_bfloat16) + (comp ? (size_t)((nb + 15) / 16) * 16 : 0);
}

template <int D, bool DENSE, bool COMP>
static cudaError_t launch_attn_mma_t(const AttnArgs& a, long long BH, cudaStream_t st) {
  const size_t smem = attn_mma_smem_bytes(D, a.nb, COMP);
  cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D, DENSE, COMP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)a.nb, (unsigned)BH);
  attn_mma_kernel<D, DENSE, COMP><<<grid, kMmaThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_attn_mma(const void* q, const void* k, const void* v, const int32_t* kv_idx,
                            const int32_t* kv_cnt, int cap, const float* kbar, const float* vbar,
                            const int32_t* nvalid, void* o, float* lse, long long BH, long long N,
                            int nb, int d, bool dense, bool comp, cudaStream_t st) {
  AttnArgs a;
  a.q = (const __nv_bfloat16*)q; a.k = (const __nv_bfloat16*)k; a.v = (const __half*)v;
  a.kv_idx = kv_idx; a.kv_cnt = kv_cnt; a.cap = cap;
  a.kbar = kbar; a.vbar = vbar; a.nvalid = nvalid;
  a.o = (__nv_bfloat16*)o; a.lse = lse;
  a.N = N; a.nb = nb; a.Npad = (long long)nb * kBlock;
  a.scale_log2 = kLog2e / sqrtf((float)d);
  if (d == 128) {
    if (dense) return launch_attn_mma_t<128, true, false>(a, BH, st);
    if (comp) return launch_attn_mma_t<128, false, true>(a, BH, st);
    return launch_attn_mma_t<128, false, false>(a, BH, st);
  }
  if (d == 64) {
    if (dense) return launch_attn_mma_t<64, true, false>(a, BH, st);
    if (comp) return launch_attn_mma_t<64, false, true>(a, BH, st);
    return launch_attn_mma_t<64, false, false>(a, BH, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace svsa
