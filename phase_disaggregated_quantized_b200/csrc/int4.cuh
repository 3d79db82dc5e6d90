// INT4 group-128 weights for the decode path (MARLIN page, abeam.tech):
//   * int4_quantize_kernel: s = bf16_RNE(amax_g / 7), q = clamp(RNE(w / s), -8, 7),
//     stored offset-binary (u = q + 8), even k in the low nibble ("data handling":
//     GPTQ-style 4-bit weights with group size 128).
//   * int4_pack_kernel: the offline reorder of codes and group scales into the
//     decode kernel's fragment order ("weight layout": weights and scales are
//     rearranged ahead of time so runtime reads are regular and dequantized
//     values land directly in tensor-core fragment order).
//
// Exactness of the two fp32 roundings:
//   amax / 7 is one IEEE division; its exact value either terminates or repeats
//   with period 3 in binary, so neither the fp32 rounding nor the following bf16
//   rounding can meet a spurious tie: the bf16 result equals bf16_RNE(exact).
//   w / s: both bf16, |w / s| <= 8; a non-half-integer exact quotient is at
//   least ~2^-20 (relative) from a half-integer, far above fp32's 2^-24.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace nvq {

constexpr int kInt4QuantThreads = 256;     // 8 warps = 8 groups in flight per CTA

// One warp per (row, 128-group): lane l holds elements 4l .. 4l+3.
__global__ void __launch_bounds__(kInt4QuantThreads) int4_quantize_kernel(
    const uint2* __restrict__ w, uint32_t N, uint32_t K, uint16_t* __restrict__ codes,
    uint16_t* __restrict__ scales) {
  const uint32_t G = K >> 7;
  const uint64_t ngroups = (uint64_t)N * G;
  const uint32_t lane = threadIdx.x & 31u;
  const uint64_t warps_total = (uint64_t)gridDim.x * (blockDim.x >> 5);
  for (uint64_t grp = (uint64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); grp < ngroups;
       grp += warps_total) {
    // Groups are contiguous in memory: group grp starts at element 128 * grp.
    const uint2 v = __ldg(w + grp * 32 + lane);
    const uint32_t a = v.x & 0x7FFF7FFFu, b = v.y & 0x7FFF7FFFu;
    uint32_t m;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
    float amax = fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
    const float s = __bfloat162float(sb);
    const uint32_t words[2] = {v.x, v.y};
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t wb = (words[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
      const float x = __uint_as_float(wb << 16);
      int q = 0;
      if (s != 0.f) q = max(-8, min(7, __float2int_rn(__fdiv_rn(x, s))));
      packed |= (uint32_t)(q + 8) << (4 * i);
    }
    codes[grp * 32 + lane] = (uint16_t)packed;
    if (lane == 0) scales[grp] = __bfloat16_as_ushort(sb);
  }
}

// One thread per 32-bit word of packed codes; the first N*K/2048*8 threads also
// write one 32-bit scale word each.
__global__ void int4_pack_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                                 uint32_t N, uint32_t K, uint32_t* __restrict__ pcodes,
                                 uint32_t* __restrict__ pscales) {
  const uint32_t G = K >> 7;
  const uint64_t nwords = (uint64_t)N * K / 8;
  const uint64_t nsw = (uint64_t)(N / 16) * G * 8;
  const uint32_t half_k = K >> 1;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nwords; i += stride) {
    const uint64_t unit = i >> 8;
    const uint32_t word = (uint32_t)(i & 255u);
    const uint32_t nt = (uint32_t)(unit / G), gi = (uint32_t)(unit % G);
    const uint32_t h = word >> 7, lane = (word >> 2) & 31u, jj = word & 3u;
    const uint32_t j = 4 * h + jj, g = lane >> 2, c = lane & 3u;
    uint32_t out = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t r = 16 * nt + g + ((p & 1) ? 8u : 0u);
      const uint32_t k = 128 * gi + 32 * c + 4 * j + ((p & 2) ? 2u : 0u) + ((p & 4) ? 1u : 0u);
      const uint32_t byte = codes[(size_t)r * half_k + (k >> 1)];
      out |= ((byte >> (4 * (k & 1))) & 0xFu) << (4 * p);
    }
    pcodes[i] = out;
  }
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nsw; i += stride) {
    const uint64_t unit = i >> 3;
    const uint32_t g = (uint32_t)(i & 7u);
    const uint32_t nt = (uint32_t)(unit / G), gi = (uint32_t)(unit % G);
    const uint32_t lo = scales[(size_t)(16 * nt + g) * G + gi];
    const uint32_t hi = scales[(size_t)(16 * nt + g + 8) * G + gi];
    pscales[i] = lo | (hi << 16);
  }
}

}  // namespace nvq
