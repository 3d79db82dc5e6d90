// W4A16 decode GEMM: Y = X * dequant(W)^T with BF16 activations at small batch
// and INT4 group-128 weights (MARLIN page, abeam.tech: "overlapping memory and
// compute" -- weights streamed asynchronously with a cache policy that keeps
// them out of L2's way, dequantization interleaved with the tensor-core MMAs,
// several warps sharing one output tile by splitting K among them).
//
// Mapping.  A warp owns one 16-row weight tile over a slice of the 128-wide
// groups.  A CTA has 4 warps = (4 / KS) row tiles x KS k-slices; the KS warps
// of a tile add their FP32 partial sums through shared memory at the end, so
// small N still fills the GPU without a global split.  For each group a lane
// loads its two 16-byte code words (1 KB per warp, coalesced, L2 evict-first)
// and its 64-byte run of activations (the offline reorder permutes K inside a
// group so that lane (g, c) of k16 step j uses k = 32c + 4j + {0,1,2,3}).
// Nibbles become bf16 (u + 128 through the exponent bits, then - 136) right in
// m16n8k16 A-fragment order; the products x * (u - 8) are exact, each group's
// FP32 sums are scaled by the group's BF16 scale in FP32.  Two independent MMA
// chains per group halve the dependent-latency path.  Batch rows beyond 8 * NT8
// are handled by further passes over the weights.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace nvq {
namespace w4a16 {

constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int PREFETCH = 8;                 // groups of weights in flight per warp

__device__ __forceinline__ uint4 ld_stream(const uint4* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 8 nibbles of one packed word -> the four bf16x2 A-fragment registers (u - 8).
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t (&a)[4]) {
  const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u;   // bf16 128 + u
    __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&v);
    h = __hsub2(h, bias);
    a[i] = *reinterpret_cast<uint32_t*>(&h);
  }
}

template <int NT8, int KS>
__global__ void __launch_bounds__(THREADS) w4a16_kernel(
    const __nv_bfloat16* __restrict__ x, const uint4* __restrict__ pcodes, const uint32_t* __restrict__ pscales,
    __nv_bfloat16* __restrict__ y, float* __restrict__ partial, uint32_t M, uint32_t N, uint32_t K,
    uint32_t groups_per_split, uint32_t splits) {
  constexpr int RT = WARPS / KS;                             // row tiles per CTA
  __shared__ float red[(KS > 1 ? (KS - 1) * RT : 1) * 32 * NT8 * 4];
  const uint32_t G = K >> 7;
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t g = lane >> 2, c = lane & 3u;
  const uint32_t rt = warp / KS, ks = warp % KS;
  const uint32_t split = blockIdx.x % splits;
  const uint32_t nt = (blockIdx.x / splits) * RT + rt;       // 16-row tile of this warp
  const uint32_t ntiles = N >> 4;
  const uint32_t gpw = groups_per_split / KS;                // groups per warp
  const uint32_t g_begin = split * groups_per_split + ks * gpw;
  const uint64_t pol = policy_evict_first();
  constexpr uint32_t MC = 8 * NT8;

  for (uint32_t m0 = 0; m0 < M; m0 += MC) {
    float acc[NT8][4];
#pragma unroll
    for (int t = 0; t < NT8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    if (nt < ntiles) {
      const uint4* up = pcodes + ((size_t)nt * G + g_begin) * 64;
      const uint32_t* sp = pscales + ((size_t)nt * G + g_begin) * 8;
      uint4 wa[PREFETCH], wb[PREFETCH];
      uint32_t sc[PREFETCH];
#pragma unroll
      for (int pf = 0; pf < PREFETCH; ++pf) {
        if ((uint32_t)pf < gpw) {
          wa[pf] = ld_stream(up + pf * 64 + lane, pol);
          wb[pf] = ld_stream(up + pf * 64 + 32 + lane, pol);
          sc[pf] = __ldg(sp + pf * 8 + g);
        }
      }
      for (uint32_t gi = 0; gi < gpw; gi += PREFETCH) {
#pragma unroll
        for (int pf = 0; pf < PREFETCH; ++pf) {
          const uint32_t gg = gi + pf;
          if (gg < gpw) {
            // Activations: lane (g, c) needs x[row, 128 gk + 32 c .. + 32) for row = m0 + 8 t + g.
            const uint32_t kbase = (g_begin + gg) * 128u + 32u * c;
            uint4 xv[NT8][4];
#pragma unroll
            for (int t = 0; t < NT8; ++t) {
              const uint32_t row = m0 + 8 * t + g;
              if (row < M) {
                const uint4* xp = reinterpret_cast<const uint4*>(x + (size_t)row * K + kbase);
#pragma unroll
                for (int v = 0; v < 4; ++v) xv[t][v] = __ldg(xp + v);
              } else {
#pragma unroll
                for (int v = 0; v < 4; ++v) xv[t][v] = make_uint4(0, 0, 0, 0);
              }
            }
            const uint32_t words[8] = {wa[pf].x, wa[pf].y, wa[pf].z, wa[pf].w,
                                       wb[pf].x, wb[pf].y, wb[pf].z, wb[pf].w};
            const uint32_t scw = sc[pf];
            if (gg + PREFETCH < gpw) {                            // refill this slot
              wa[pf] = ld_stream(up + (gg + PREFETCH) * 64 + lane, pol);
              wb[pf] = ld_stream(up + (gg + PREFETCH) * 64 + 32 + lane, pol);
              sc[pf] = __ldg(sp + (gg + PREFETCH) * 8 + g);
            }
            float t0[NT8][4], t1[NT8][4];                        // two independent chains
#pragma unroll
            for (int t = 0; t < NT8; ++t)
#pragma unroll
              for (int e = 0; e < 4; ++e) t0[t][e] = t1[t][e] = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint32_t a[4];
              dequant_word(words[j], a);
#pragma unroll
              for (int t = 0; t < NT8; ++t) {
                // k16 step j uses activation words 2j (b0) and 2j + 1 (b1) of the lane's run.
                const uint4 q = xv[t][j >> 1];
                const uint32_t b0 = (j & 1) ? q.z : q.x;
                const uint32_t b1 = (j & 1) ? q.w : q.y;
                if (j & 1) mma_bf16_16816(t1[t], a, b0, b1);
                else mma_bf16_16816(t0[t], a, b0, b1);
              }
            }
            const float s_lo = __uint_as_float(scw << 16), s_hi = __uint_as_float(scw & 0xFFFF0000u);
#pragma unroll
            for (int t = 0; t < NT8; ++t) {
              acc[t][0] = __fmaf_rn(s_lo, t0[t][0] + t1[t][0], acc[t][0]);
              acc[t][1] = __fmaf_rn(s_lo, t0[t][1] + t1[t][1], acc[t][1]);
              acc[t][2] = __fmaf_rn(s_hi, t0[t][2] + t1[t][2], acc[t][2]);
              acc[t][3] = __fmaf_rn(s_hi, t0[t][3] + t1[t][3], acc[t][3]);
            }
          }
        }
      }
    }
    if (KS > 1) {                                            // k-slices of a tile add up, fixed order
      if (ks > 0) {
#pragma unroll
        for (int t = 0; t < NT8; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) red[(((rt * (KS - 1) + ks - 1) * 32 + lane) * NT8 + t) * 4 + e] = acc[t][e];
      }
      __syncthreads();
      if (ks == 0) {
        for (int k2 = 1; k2 < KS; ++k2)
#pragma unroll
          for (int t = 0; t < NT8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[t][e] += red[(((rt * (KS - 1) + k2 - 1) * 32 + lane) * NT8 + t) * 4 + e];
      }
      __syncthreads();
    }
    if (nt < ntiles && ks == 0) {
      // C fragment: (weight row g / g+8, batch column 2c / 2c+1).
      const uint32_t n_lo = nt * 16 + g, n_hi = n_lo + 8;
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t m = m0 + t * 8 + 2 * c + (e & 1);
          const uint32_t n = (e & 2) ? n_hi : n_lo;
          if (m < M) {
            if (splits == 1) y[(size_t)m * N + n] = __float2bfloat16_rn(acc[t][e]);
            else partial[((size_t)split * M + m) * N + n] = acc[t][e];
          }
        }
      }
    }
  }
}

// Y = bf16(sum over splits of the FP32 partials), fixed summation order.
__global__ void w4a16_reduce_kernel(const float4* __restrict__ partial, uint2* __restrict__ y, uint32_t splits,
                                    uint64_t n4) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 s = __ldg(partial + i);
    for (uint32_t k = 1; k < splits; ++k) {
      const float4 v = __ldg(partial + k * n4 + i);
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&lo);
    o.y = *reinterpret_cast<uint32_t*>(&hi);
    y[i] = o;
  }
}

}  // namespace w4a16
}  // namespace nvq
