// NVFP4 round-to-nearest quantization (Mix-Quant page, gist.science, section 2
// "hybrid precision strategy": 4-bit floats in 16-element groups with a local
// E4M3 scale plus one tensor-level FP32 scale, plain round-to-nearest).
//
// Two kernels, both HBM-streaming:
//   nvfp4_amax_kernel      max |x| over the tensor -> one partial per CTA
//   nvfp4_quantize_kernel  t from the partials (or the caller's t), then one
//                          thread per 16-element block: E4M3 block scale and
//                          sixteen E2M1 codes.
//
// Exactness.  Every rounding is decided on the exact real quotient:
//   * t = fp32_RN(amax / 2688): one correctly rounded IEEE division.
//   * s = E4M3_RNE(amax_b / (6t)): a fast estimate from an fp32 quotient is
//     within one code of the exact answer; the two neighbouring midpoints are
//     then tested exactly with the sign of fma(-(6 mu), t, amax_b), an exact
//     product minus an exact value rounded once.
//   * codes: q = |x| * (1/(S t)) in fp32 is within 3.01 ulp (relative 2^-24)
//     of the exact quotient, so cvt.rn.satfinite.e2m1x2 on q decides like the
//     exact quotient unless some bf16 value lies within 4.03 fp32 ulps of a
//     threshold mu_i S t.  For each E4M3 scale code the kernel precomputes
//     (once per CTA) whether that can happen; blocks with such a scale take an
//     exact path that compares |x| against mu_i S t through its rounded value
//     h = fl(P t) and the exact residual e = fma(P, t, -h), P = mu_i S exact.
#pragma once
#include "ptx.cuh"

namespace nvq {

constexpr int kAmaxThreads = 512;
constexpr int kAmaxMaxBlocks = 592;       // 4 per SM on 148 SMs
constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  // For non-negative bf16 the bit patterns order like the values.
  const uint32_t x = a & 0x7FFF7FFFu, y = b & 0x7FFF7FFFu;
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
  return r;
}

__device__ __forceinline__ float bf16x2_hmax_to_f32(uint32_t v) {
  const uint32_t lo = v << 16, hi = v & 0xFFFF0000u;
  return fmaxf(__uint_as_float(lo), __uint_as_float(hi));
}

__global__ void __launch_bounds__(kAmaxThreads) nvfp4_amax_kernel(const uint4* __restrict__ x, size_t nvec,
                                                                  float* __restrict__ partial) {
  uint32_t m = 0;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 v0 = __ldg(x + i), v1 = __ldg(x + i + stride), v2 = __ldg(x + i + 2 * stride),
          v3 = __ldg(x + i + 3 * stride);
    m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(v0.x, v0.y), bf16x2_absmax(v0.z, v0.w)));
    m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(v1.x, v1.y), bf16x2_absmax(v1.z, v1.w)));
    m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(v2.x, v2.y), bf16x2_absmax(v2.z, v2.w)));
    m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(v3.x, v3.y), bf16x2_absmax(v3.z, v3.w)));
  }
  for (; i < nvec; i += stride) {
    uint4 v = __ldg(x + i);
    m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(v.x, v.y), bf16x2_absmax(v.z, v.w)));
  }
  float f = bf16x2_hmax_to_f32(m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
  __shared__ float red[kAmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = f;
  __syncthreads();
  if (threadIdx.x < 32) {
    f = threadIdx.x < kAmaxThreads / 32 ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) f = fmaxf(f, __shfl_xor_sync(0xFFFFFFFFu, f, o));
    if (threadIdx.x == 0) partial[blockIdx.x] = f;
  }
}

// Value of a non-negative E4M3 (FN) code 0..126: bias 7, 3 mantissa bits.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  return e == 0 ? __int2float_rn((int)m) * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(v));
  return r & 0xFFu;
}

// Two E2M1 codes in one byte: `lo` in bits 0..3, `hi` in bits 4..7 (inputs >= 0).
__device__ __forceinline__ uint32_t e2m1x2_rn_satfinite(float hi, float lo) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__constant__ float c_e2m1_mid[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};

// amax_b > 6 mu t, or equal with the tie going up (upper code even)?
__device__ __forceinline__ bool scale_passes(float amax, float mu, float t, uint32_t upper_code) {
  const float r = __fmaf_rn(-__fmul_rn(mu, 6.0f), t, amax);   // exact sign
  return r > 0.f || (r == 0.f && (upper_code & 1u) == 0u);
}

__device__ __forceinline__ uint32_t block_scale_code(float amax, float t, float t6) {
  uint32_t s = e4m3_rn_satfinite(__fdiv_rn(amax, t6));
  if (s < 126u && scale_passes(amax, 0.5f * (e4m3_value(s) + e4m3_value(s + 1)), t, s + 1))
    s += 1;
  else if (s > 0u && !scale_passes(amax, 0.5f * (e4m3_value(s - 1) + e4m3_value(s)), t, s))
    s -= 1;
  return s;
}

// Exact E2M1 magnitude of |x| (fp32 value of a bf16) for block scale S, tensor scale t.
__device__ __noinline__ uint32_t e2m1_exact_pair(float ax_hi, float ax_lo, float S, float t) {
  uint32_t mh = 0, ml = 0;
  if (S > 0.f) {
#pragma unroll
    for (int i = 0; i < 7; ++i) {
      const float P = __fmul_rn(c_e2m1_mid[i], S);         // exact: <= 7 significant bits
      const float h = __fmul_rn(P, t);
      const float e = __fmaf_rn(P, t, -h);                 // exact residual: threshold = h + e
      const bool up_on_tie = (i & 1);
      mh += (ax_hi > h || (ax_hi == h && (e < 0.f || (e == 0.f && up_on_tie)))) ? 1u : 0u;
      ml += (ax_lo > h || (ax_lo == h && (e < 0.f || (e == 0.f && up_on_tie)))) ? 1u : 0u;
    }
  }
  return (mh << 4) | ml;
}

// Codes for 4 bf16x2 words (8 elements) -> 32 bits of packed codes.
template <bool kExact>
__device__ __forceinline__ uint32_t codes8(const uint32_t (&w)[4], float inv_d, float S, float t) {
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float alo = __uint_as_float((w[i] & 0x7FFFu) << 16);
    const float ahi = __uint_as_float(w[i] & 0x7FFF0000u);
    uint32_t byte;
    if (kExact) byte = e2m1_exact_pair(ahi, alo, S, t);
    else byte = e2m1x2_rn_satfinite(__fmul_rn(ahi, inv_d), __fmul_rn(alo, inv_d));
    byte |= ((w[i] >> 12) & 0x8u) | ((w[i] >> 24) & 0x80u);       // signs of x
    out |= byte << (8 * i);
  }
  return out;
}

__device__ __forceinline__ float resolve_tensor_scale(const float* t_in, const float* partial, int npartial) {
  if (t_in != nullptr) return __ldg(t_in);
  float m = 0.f;
  for (int i = 0; i < npartial; ++i) m = fmaxf(m, __ldg(partial + i));
  return m == 0.f ? 1.0f : __fdiv_rn(m, 2688.0f);
}

// rows x K bf16 -> codes [rows, K/2], tiled scales, t.
__global__ void __launch_bounds__(kQuantThreads) nvfp4_quantize_kernel(
    const uint4* __restrict__ x, uint32_t rows, uint32_t K, const float* __restrict__ t_in,
    const float* __restrict__ partial, int npartial, uint2* __restrict__ codes,
    uint8_t* __restrict__ scales, float* __restrict__ t_out) {
  __shared__ float s_inv_d[128];
  __shared__ uint8_t s_danger[128];
  __shared__ float s_t;
  if (threadIdx.x < 32) {
    // Every warp-0 lane reduces a slice of the partial maxima.
    float m = 0.f;
    if (t_in == nullptr)
      for (int i = threadIdx.x; i < npartial; i += 32) m = fmaxf(m, __ldg(partial + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0) {
      const float t = t_in != nullptr ? __ldg(t_in) : (m == 0.f ? 1.0f : __fdiv_rn(m, 2688.0f));
      s_t = t;
      if (blockIdx.x == 0) *t_out = t;
    }
  }
  __syncthreads();
  const float t = s_t;
  if (threadIdx.x < 127) {
    const float S = e4m3_value(threadIdx.x);
    const float d = __fmul_rn(S, t);
    float inv = 0.f;
    uint32_t danger = 0;
    if (threadIdx.x != 0) {
      inv = __frcp_rn(d);
      if (!(d >= 1.17549435e-38f) || isinf(inv)) {
        danger = 0x7F;                                      // tiny / huge: exact path
      } else {
#pragma unroll
        for (int i = 0; i < 7; ++i) {
          const float h = __fmul_rn(__fmul_rn(c_e2m1_mid[i], S), t);
          const uint32_t f = __float_as_uint(h) & 0xFFFFu;
          const uint32_t dist = min(f, 0x10000u - f);        // fp32 ulps to the nearest bf16
          if (dist <= 16u || !(h >= 1e-30f) || isinf(h)) danger |= 1u << i;
        }
      }
    }
    s_inv_d[threadIdx.x] = inv;
    s_danger[threadIdx.x] = (uint8_t)danger;
  }
  __syncthreads();

  const float t6 = __fmul_rn(6.0f, t);
  const uint32_t nbk = K >> 4;                               // 16-element blocks per row
  const uint32_t atoms_per_rowtile = K >> 6;
  const uint64_t nblocks = (uint64_t)rows * nbk;
  const uint32_t lane = threadIdx.x & 31u;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t base = (uint64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31u); base < nblocks;
       base += stride) {
    const uint64_t b = base + lane;
    const bool valid = b < nblocks;                          // nblocks % 4 == 0: groups of 4 agree
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (valid) {
      const uint4 v0 = __ldg(x + 2 * b), v1 = __ldg(x + 2 * b + 1);
      w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
      w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    }
    uint32_t m2 = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(w[0], w[1]), bf16x2_absmax(w[2], w[3])),
                                bf16x2_absmax(bf16x2_absmax(w[4], w[5]), bf16x2_absmax(w[6], w[7])));
    const float amax = bf16x2_hmax_to_f32(m2);
    const uint32_t s = block_scale_code(amax, t, t6);
    const float inv_d = s_inv_d[s];
    uint2 c;
    const uint32_t wa[4] = {w[0], w[1], w[2], w[3]}, wb[4] = {w[4], w[5], w[6], w[7]};
    if (s_danger[s] == 0) {
      c.x = codes8<false>(wa, inv_d, 0.f, t);
      c.y = codes8<false>(wb, inv_d, 0.f, t);
    } else {
      const float S = e4m3_value(s);
      c.x = codes8<true>(wa, inv_d, S, t);
      c.y = codes8<true>(wb, inv_d, S, t);
    }
    // Gather the 4 scale bytes of an aligned group of 4 blocks (same row, same atom).
    uint32_t sv = s << (8 * (lane & 3u));
    sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 1);
    sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 2);
    if (valid) {
      codes[b] = c;
      if ((lane & 3u) == 0u) {
        const uint32_t r = (uint32_t)(b / nbk), kb = (uint32_t)(b - (uint64_t)r * nbk);
        const uint64_t off = ((uint64_t)(r >> 7) * atoms_per_rowtile + (kb >> 2)) * 512u +
                             (r & 31u) * 16u + ((r & 127u) >> 5) * 4u;
        *reinterpret_cast<uint32_t*>(scales + off) = sv;
      }
    }
  }
  // Zero the scales of the padding rows up to the next multiple of 128.
  const uint32_t rows_pad = (rows + 127u) & ~127u;
  const uint64_t npad = (uint64_t)(rows_pad - rows) * atoms_per_rowtile;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < npad; i += stride) {
    const uint32_t r = rows + (uint32_t)(i / atoms_per_rowtile);
    const uint32_t kt = (uint32_t)(i % atoms_per_rowtile);
    const uint64_t off = ((uint64_t)(r >> 7) * atoms_per_rowtile + kt) * 512u + (r & 31u) * 16u +
                         ((r & 127u) >> 5) * 4u;
    *reinterpret_cast<uint32_t*>(scales + off) = 0u;
  }
}

}  // namespace nvq
