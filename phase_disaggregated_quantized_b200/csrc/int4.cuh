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

// One thread per 32-bit word of packed codes; the first (N/32)*(K/128)*16
// threads also write one 32-bit scale word each.  Dense unit = 32 rows x one
// 128-k group (two 16-row MMA tiles tt): word 128 q + 4 lane + comp holds k16
// step j = 2 q + comp / 2 of tile tt = comp % 2 for lane = 4 g + c; scale word
// 2 g + tt holds rows 16 tt + g (low half) and 16 tt + g + 8 (high half).
__global__ void int4_pack_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                                 uint32_t N, uint32_t K, uint32_t* __restrict__ pcodes,
                                 uint32_t* __restrict__ pscales) {
  const uint32_t G = K >> 7;
  const uint64_t nwords = (uint64_t)N * K / 8;
  const uint64_t nsw = (uint64_t)(N / 32) * G * 16;
  const uint32_t half_k = K >> 1;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nwords; i += stride) {
    const uint64_t unit = i >> 9;
    const uint32_t word = (uint32_t)(i & 511u);
    const uint32_t nt = (uint32_t)(unit / G), gi = (uint32_t)(unit % G);
    const uint32_t q = word >> 7, lane = (word >> 2) & 31u, comp = word & 3u;
    const uint32_t j = 2 * q + (comp >> 1), tt = comp & 1u, g = lane >> 2, c = lane & 3u;
    uint32_t out = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t r = 32 * nt + 16 * tt + g + ((p & 1) ? 8u : 0u);
      const uint32_t k = 128 * gi + 32 * c + 4 * j + ((p & 2) ? 2u : 0u) + ((p & 4) ? 1u : 0u);
      const uint32_t byte = codes[(size_t)r * half_k + (k >> 1)];
      out |= ((byte >> (4 * (k & 1))) & 0xFu) << (4 * p);
    }
    pcodes[i] = out;
  }
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nsw; i += stride) {
    const uint64_t unit = i >> 4;
    const uint32_t wi = (uint32_t)(i & 15u), g = wi >> 1, tt = wi & 1u;
    const uint32_t nt = (uint32_t)(unit / G), gi = (uint32_t)(unit % G);
    const uint32_t row = 32 * nt + 16 * tt + g;
    const uint32_t lo = scales[(size_t)row * G + gi];
    const uint32_t hi = scales[(size_t)(row + 8) * G + gi];
    pscales[i] = lo | (hi << 16);
  }
}

}  // namespace nvq

namespace nvq {

// ---------------------------------------------------------------- 2:4 sparse packing
// 2:4 magnitude pruning of the BF16 master (two largest |w| of every run of four
// k, the lower k on equal magnitudes) combined with the dense INT4 codes (a
// run's largest |w| is always kept, so the group scales and the kept codes are
// the dense ones), written in the sparse decode kernel's order: per 32-row x
// 128-k unit, two 16-row tiles tt, each 512 bytes of A-fragment code words
// (lane-major, 4 m16n8k32 steps per lane) and 256 bytes of metadata words
// (lanes c = 0, 1); the unit's 64 bytes of scales hold in word 2 g + tt rows
// 16 tt + g (low half) and 16 tt + g + 8 (high half).

// Kept positions (i0 < i1) of one run from its four bf16 values.
__device__ __forceinline__ uint32_t run_meta(uint2 w4) {
  const uint32_t a[4] = {w4.x & 0x7FFFu, (w4.x >> 16) & 0x7FFFu, w4.y & 0x7FFFu, (w4.y >> 16) & 0x7FFFu};
  uint32_t keep = 0;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t beaten = 0;                                   // runs ahead of p in the (|w| desc, k asc) order
#pragma unroll
    for (int q = 0; q < 4; ++q) beaten += (a[q] > a[p] || (a[q] == a[p] && q < p)) ? 1u : 0u;
    if (beaten < 2) keep |= 1u << p;
  }
  const uint32_t i0 = __ffs(keep) - 1, i1 = 31 - __clz(keep);
  return i0 | (i1 << 2);
}

// MMA step s, MMA run j -> run of the 128-k group.
__device__ __forceinline__ uint32_t sparse_run(uint32_t s, uint32_t j) {
  return 8 * s + ((j & 1u) ? 4 + (j >> 1) : (j >> 1));
}

// One thread per (unit, tile, lane, step): one code word, and for lanes c < 2 one metadata word.
__global__ void int4_pack_sparse24_kernel(const uint2* __restrict__ w, const uint8_t* __restrict__ codes,
                                          const uint16_t* __restrict__ scales, uint32_t N, uint32_t K,
                                          uint32_t* __restrict__ packed, uint32_t* __restrict__ pscales) {
  const uint32_t G = K >> 7;
  const uint64_t units = (uint64_t)(N >> 5) * G;
  const uint64_t total = units * 256;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t unit = i >> 8;
    const uint32_t tt = (uint32_t)(i >> 7) & 1u;
    const uint32_t lane = (uint32_t)(i >> 2) & 31u, s = (uint32_t)i & 3u;
    const uint32_t g = lane >> 2, c = lane & 3u;
    const uint32_t nt = (uint32_t)(unit / G), gi = (uint32_t)(unit - (uint64_t)nt * G);
    const uint32_t r0 = 32 * nt + 16 * tt;                  // first row of this 16-row tile
    auto kept_code = [&](uint32_t row, uint32_t run, uint32_t q) {   // q-th kept code of a run
      const uint32_t k0 = 128 * gi + 4 * run;
      const uint32_t m = run_meta(__ldg(w + ((size_t)row * K + k0) / 4));
      const uint32_t k = k0 + (q ? (m >> 2) : (m & 3u));
      return (uint32_t)(__ldg(codes + (size_t)row * (K / 2) + k / 2) >> (4 * (k & 1u))) & 0xFu;
    };
    uint32_t word = 0;
#pragma unroll
    for (int reg = 0; reg < 4; ++reg) {
      const uint32_t row = r0 + g + ((reg & 1) ? 8u : 0u);
      const uint32_t kc = 2 * c + ((reg & 2) ? 8u : 0u);   // compressed k of the register's low half
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t kk = kc + h;
        word |= kept_code(row, sparse_run(s, kk >> 1), kk & 1u) << (4 * (reg + 4 * h));
      }
    }
    uint32_t* u = packed + unit * 384 + tt * 192;            // 1536 bytes per unit, 768 per tile
    u[4 * lane + s] = word;
    if (c < 2) {
      uint32_t m = 0;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const uint32_t row = r0 + g + 8 * (n >> 2);
        const uint32_t run = sparse_run(s, 4 * c + (n & 3));
        m |= run_meta(__ldg(w + ((size_t)row * K + 128 * gi + 4 * run) / 4)) << (4 * n);
      }
      u[128 + 4 * (2 * g + c) + s] = m;
    }
    if (lane < 8 && s == 0) {                                // word 2 g + tt: rows r0 + g (low), + 8 (high)
      const uint32_t lo = __ldg(scales + (size_t)(r0 + lane) * G + gi);
      const uint32_t hi = __ldg(scales + (size_t)(r0 + lane + 8) * G + gi);
      pscales[unit * 16 + 2 * lane + tt] = lo | (hi << 16);
    }
  }
}

}  // namespace nvq
