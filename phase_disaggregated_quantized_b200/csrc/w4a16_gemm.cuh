// W4A16 decode GEMM: Y = X * dequant(W)^T with BF16 activations at small batch
// and INT4 group-128 weights (MARLIN page, abeam.tech: "overlapping memory and
// compute" -- weights streamed asynchronously with a cache policy that keeps
// them out of L2's way, dequantization interleaved with the tensor-core MMAs,
// several warps sharing an output tile through a split of K).
//
// Mapping: a warp owns 16 weight rows (one packed unit column) over a range of
// 128-wide groups; a CTA of 4 warps owns 64 rows and shares one X slice in
// shared memory.  The packed layout hands each lane its m16n8k16 A fragments
// directly: per group a lane loads two 16-byte words (1 KB per warp, fully
// coalesced), turns each nibble pair into bf16x2 (u + 128 via the exponent bits,
// then - 136), and multiplies against X fragments read from shared memory.
// The products x * (u - 8) are exact; each group's FP32 partial sums are scaled
// by the group's BF16 scale in FP32, so no rounding happens on the weights.
// With a K split the FP32 partials go to workspace and a second kernel adds
// them in a fixed order.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace nvq {
namespace w4a16 {

constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int PREFETCH = 4;                 // groups in flight per warp

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

// NT8 = batch tiles of 8 rows handled per pass (M chunk = 8 * NT8).  X is
// staged in chunks of kChunkGroups(NT8) groups: 64 KB of shared memory.
template <int NT8>
__host__ __device__ constexpr uint32_t chunk_groups() { return 32u / NT8; }
template <int NT8>
__host__ __device__ constexpr uint32_t smem_bytes() { return 8u * NT8 * (chunk_groups<NT8>() * 128u + 8u) * 2u; }

template <int NT8>
__global__ void __launch_bounds__(THREADS) w4a16_kernel(
    const __nv_bfloat16* __restrict__ x, const uint4* __restrict__ pcodes, const uint32_t* __restrict__ pscales,
    __nv_bfloat16* __restrict__ y, float* __restrict__ partial, uint32_t M, uint32_t N, uint32_t K,
    uint32_t groups_per_split, uint32_t splits) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  constexpr uint32_t KCG = chunk_groups<NT8>();
  constexpr uint32_t MC = 8 * NT8;
  constexpr uint32_t ldx = KCG * 128u + 8u;                  // padded row (bank spread)
  const uint32_t G = K >> 7;
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t g = lane >> 2, c = lane & 3u;
  const uint32_t split = blockIdx.x % splits;
  const uint32_t nt = (blockIdx.x / splits) * WARPS + warp;  // 16-row tile of this warp
  const uint32_t ntiles = N >> 4;
  const uint32_t g_begin = split * groups_per_split;
  const uint32_t g_end = min(G, g_begin + groups_per_split);
  const uint64_t pol = policy_evict_first();

  for (uint32_t m0 = 0; m0 < M; m0 += MC) {
    float acc[NT8][4];
#pragma unroll
    for (int t = 0; t < NT8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    for (uint32_t c0 = g_begin; c0 < g_end; c0 += KCG) {
      const uint32_t ng = min(KCG, g_end - c0);
      // Stage X[m0 : m0 + MC, 128 c0 : 128 (c0 + ng)] (zero rows past M).
      const uint32_t vec_per_row = ng * 16u;
      for (uint32_t i = threadIdx.x; i < MC * vec_per_row; i += THREADS) {
        const uint32_t r = i / vec_per_row, cv = i % vec_per_row;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m0 + r < M) v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(m0 + r) * K + c0 * 128u) + cv);
        *reinterpret_cast<uint4*>(xs + r * ldx + cv * 8) = v;
      }
      __syncthreads();
      if (nt < ntiles) {
        const uint4* up = pcodes + ((size_t)nt * G + c0) * 64;
        const uint32_t* sp = pscales + ((size_t)nt * G + c0) * 8;
        uint4 wa[PREFETCH], wb[PREFETCH];
        uint32_t sc[PREFETCH];
#pragma unroll
        for (int pf = 0; pf < PREFETCH; ++pf) {
          if ((uint32_t)pf < ng) {
            wa[pf] = ld_stream(up + pf * 64 + lane, pol);
            wb[pf] = ld_stream(up + pf * 64 + 32 + lane, pol);
            sc[pf] = __ldg(sp + pf * 8 + g);
          }
        }
        for (uint32_t gi = 0; gi < ng; gi += PREFETCH) {
#pragma unroll
          for (int pf = 0; pf < PREFETCH; ++pf) {
            const uint32_t gg = gi + pf;
            if (gg < ng) {
              const uint32_t words[8] = {wa[pf].x, wa[pf].y, wa[pf].z, wa[pf].w,
                                         wb[pf].x, wb[pf].y, wb[pf].z, wb[pf].w};
              const uint32_t scw = sc[pf];
              if (gg + PREFETCH < ng) {                          // refill this slot
                wa[pf] = ld_stream(up + (gg + PREFETCH) * 64 + lane, pol);
                wb[pf] = ld_stream(up + (gg + PREFETCH) * 64 + 32 + lane, pol);
                sc[pf] = __ldg(sp + (gg + PREFETCH) * 8 + g);
              }
              float tmp[NT8][4];
#pragma unroll
              for (int t = 0; t < NT8; ++t) tmp[t][0] = tmp[t][1] = tmp[t][2] = tmp[t][3] = 0.f;
              const __nv_bfloat16* xg = xs + gg * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                uint32_t a[4];
                dequant_word(words[j], a);
#pragma unroll
                for (int t = 0; t < NT8; ++t) {
                  const __nv_bfloat16* xr = xg + (t * 8 + g) * ldx + 16 * j + 2 * c;
                  const uint32_t b0 = *reinterpret_cast<const uint32_t*>(xr);
                  const uint32_t b1 = *reinterpret_cast<const uint32_t*>(xr + 8);
                  mma_bf16_16816(tmp[t], a, b0, b1);
                }
              }
              const float s_lo = __uint_as_float(scw << 16), s_hi = __uint_as_float(scw & 0xFFFF0000u);
#pragma unroll
              for (int t = 0; t < NT8; ++t) {
                acc[t][0] = __fmaf_rn(s_lo, tmp[t][0], acc[t][0]);
                acc[t][1] = __fmaf_rn(s_lo, tmp[t][1], acc[t][1]);
                acc[t][2] = __fmaf_rn(s_hi, tmp[t][2], acc[t][2]);
                acc[t][3] = __fmaf_rn(s_hi, tmp[t][3], acc[t][3]);
              }
            }
          }
        }
      }
      __syncthreads();
    }
    if (nt < ntiles) {
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
