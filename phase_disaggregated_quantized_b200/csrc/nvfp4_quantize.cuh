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
//   * codes: for each of the 127 E4M3 scale codes S the kernel derives, once
//     per CTA, the exact decision thresholds as bf16 values: the smallest bf16
//     that lies above mu_i S t (or on it, when the tie goes up), found from
//     h = fl(P t) and the exact residual e = fma(P, t, -h), P = mu_i S exact.
//     The fast path (q = |x| * r, r = fl(1/fl(S t)) or that value moved by
//     2^-20 relative, cvt.rn.satfinite.e2m1x2) is exact for a scale code if it
//     gives the exact code on both sides of every threshold; both maps are
//     monotone in |x|, so it is then exact for every bf16 input.  A warp takes
//     it when it is exact for all 32 of its blocks' scale codes; otherwise the
//     warp counts thresholds with packed bf16x2 compares, which is exact by
//     construction.
#pragma once
#include "ptx.cuh"

namespace nvq {

constexpr int kAmaxThreads = 512;
constexpr int kAmaxMaxBlocks = 592;       // 4 per SM on 148 SMs
constexpr int kQuantThreads = 1024;   // one CTA per SM (64 registers): the per-CTA tables are built 148 times

__device__ __forceinline__ uint32_t bf16x2_max(uint32_t x, uint32_t y) {   // inputs already >= 0
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
  auto vmax = [](const uint4 v) {            // max |x| of 8 bf16, still packed in two halves
    return bf16x2_max(bf16x2_max(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                      bf16x2_max(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  };
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    const uint4 v0 = __ldg(x + i), v1 = __ldg(x + i + stride), v2 = __ldg(x + i + 2 * stride),
                v3 = __ldg(x + i + 3 * stride);
    m = bf16x2_max(m, bf16x2_max(bf16x2_max(vmax(v0), vmax(v1)), bf16x2_max(vmax(v2), vmax(v3))));
  }
  for (; i < nvec; i += stride) m = bf16x2_max(m, vmax(__ldg(x + i)));
  // The quantize pass may start launching now (it waits for this grid before it
  // reads the partials).
  grid_launch_dependents();
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

// The tensor scale of a tensor whose max |x| is `amax`: 1 for an all-zero
// tensor, else fp32_RNE(amax / 2688), 2688 = 6 (largest E2M1) x 448 (largest E4M3).
__device__ __forceinline__ float tensor_scale_of(float amax) {
  return amax == 0.f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// Max of the amax kernel's per-CTA partials (0 for none): the tensor's max |x|.
__global__ void __launch_bounds__(32) nvfp4_amax_finish_kernel(const float* __restrict__ partial, int npartial,
                                                                float* __restrict__ amax_out) {
  float m = 0.f;
  for (int i = threadIdx.x; i < npartial; i += 32) m = fmaxf(m, __ldg(partial + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (threadIdx.x == 0) *amax_out = m;
}

// t from a max |x| computed elsewhere (for instance combined over the row
// shards of one tensor held by several processes).
__global__ void nvfp4_scale_from_amax_kernel(const float* amax, float* t_out) {   // may alias
  *t_out = tensor_scale_of(*amax);
}

// Value of a non-negative E4M3 (FN) code 0..126: bias 7, 3 mantissa bits.
// Subnormals (exponent field 0) are m * 2^-9 = (1 + m/8) 2^-6 - 2^-6, exact.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  const float nrm = __uint_as_float(((e + 120u) << 23) | (m << 20));
  const float sub = __fadd_rn(__uint_as_float((121u << 23) | (m << 20)), -0.015625f);
  return e == 0 ? sub : nrm;
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

// The fast map's multiplier r: fl(1/fl(S t)), or that value moved down or up
// by 2^-20 relative when the plain one fails the exactness check.  With a
// computed t = fl(amax / 2688), amax a bf16 value and 2688 = 2^7 * 21, every
// threshold mu_i S t with mu_i S divisible by 21 lies within t's own rounding
// error (<= 2^-24 relative) of a bf16 value, and on the same side of it for
// every such threshold; the three roundings of the fast map (<= 3 * 2^-24)
// then decide those inputs at random.  A 2^-20 move outweighs all of that and
// puts every such input on one side, which is right for all of them in one of
// the two directions, while thresholds that are not near a bf16 value keep
// margins far above 2^-20.  The check decides in every case.
constexpr float kNudgeDown = 1.0f - 0x1p-20f;
constexpr float kNudgeUp = 1.0f + 0x1p-20f;

// E4M3_RNE_satfinite(amax / (6 t)) decided on the exact quotient.  The estimate
// amax * fl(1/fl(6t)) is within ~2 ulp, so the answer is s0 or a neighbour.
// mid6[c] = 6 * (value(c) + value(c + 1)) / 2, exact in FP32 (at most 7
// significant bits).
__device__ __forceinline__ uint32_t block_scale_code(float amax, float t, float inv6t, const float* mid6) {
  uint32_t s = e4m3_rn_satfinite(__fmul_rn(amax, inv6t));
  const float r_up = __fmaf_rn(-mid6[s], t, amax);                      // exact sign (s <= 126)
  if (s < 126u && (r_up > 0.f || (r_up == 0.f && ((s + 1u) & 1u) == 0u))) return s + 1u;
  if (s > 0u) {
    const float r_dn = __fmaf_rn(-mid6[s - 1u], t, amax);
    if (!(r_dn > 0.f || (r_dn == 0.f && (s & 1u) == 0u))) return s - 1u;
  }
  return s;
}

// Smallest bf16 (as bits) whose value passes E2M1 midpoint i of a block with
// decode scale S t: value > mu_i S t, or equal with the tie going up (odd i).
// h = fl(P t) with P = mu_i S exact, e = fma(P, t, -h) the exact residual.
__device__ __forceinline__ uint32_t e2m1_threshold_bits(float P, float t, int i) {
  const float h = __fmul_rn(P, t);
  const float e = __fmaf_rn(P, t, -h);
  const uint32_t hb = __float_as_uint(h);
  if (isinf(h)) return 0x7F80u;
  if (h == 0.f) return 1u;                                  // any positive value passes
  if ((hb & 0xFFFFu) != 0u) return (hb >> 16) + 1u;         // next bf16 above h (and above h + e)
  const uint32_t v0 = hb >> 16;                             // h is itself a bf16 value
  if (e > 0.f) return v0 + 1u;
  if (e < 0.f) return v0;
  return (i & 1) ? v0 : v0 + 1u;                            // exact tie
}

__device__ __forceinline__ uint32_t e2m1_fast_code(uint32_t bf16_bits, float inv_d) {
  const float v = __uint_as_float(bf16_bits << 16);
  return e2m1x2_rn_satfinite(0.f, __fmul_rn(v, inv_d)) & 0xFu;
}

// Packed codes for 4 bf16x2 words (8 elements) -> 32 bits, fast path.  The
// signed product goes straight into the conversion: fl(-a * r) = -fl(a * r) and
// round-to-nearest-even is symmetric, so the code of -a is the code of a with
// the sign bit set -- also for a product that rounds to zero (R6).
__device__ __forceinline__ uint32_t codes8_fast(const uint32_t* w, float inv_d) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), inv_d);            // even k (low half)
    v[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv_d); // odd k (high half)
  }
  uint32_t out;
  asm("{ .reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3}; }"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// Exact path: count the thresholds each |x| reaches, two elements at a time
// with packed bf16x2 compares (1.0 / 0.0) accumulated on top of 128.0, which
// keeps the count in the low mantissa bits.
__device__ __forceinline__ uint32_t codes8_exact(const uint32_t* w, const uint32_t (&B)[7]) {
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t a = w[i] & 0x7FFF7FFFu;
    uint32_t acc = 0x43004300u;
#pragma unroll
    for (int k = 0; k < 7; ++k) {
      uint32_t ge;
      asm("set.ge.bf16x2.bf16x2 %0, %1, %2;" : "=r"(ge) : "r"(a), "r"(B[k]));
      asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(acc) : "r"(acc), "r"(ge));
    }
    uint32_t byte = (acc & 0x7u) | ((acc >> 12) & 0x70u);
    byte |= ((w[i] >> 12) & 0x8u) | ((w[i] >> 24) & 0x80u);
    out |= byte << (8 * i);
  }
  return out;
}

// rows x K bf16 -> codes [rows, K/2], tiled scales, t.
__global__ void __launch_bounds__(kQuantThreads, 1) nvfp4_quantize_kernel(
    const uint4* __restrict__ x, uint32_t rows, uint32_t K, const float* __restrict__ t_in,
    const float* __restrict__ partial, int npartial, uint2* __restrict__ codes,
    uint8_t* __restrict__ scales, float* __restrict__ t_out) {
  __shared__ float s_inv_d[128];
  __shared__ uint32_t s_fast_ok[128];
  __shared__ uint4 s_thr[128];                               // 7 thresholds (bf16 bits) + pad
  __shared__ float s_mid6[128];                              // 6 x midpoints between E4M3 codes
  __shared__ uint16_t s_b[127][8];                           // thresholds while the tables are built
  __shared__ uint8_t s_ck[127][8];                           // per threshold: which candidate multipliers pass
  __shared__ float s_t;
  const uint32_t nblocks = rows * (K >> 4);                  // 16-element blocks, < 2^31 (checked on the host)
  const uint32_t stride = gridDim.x * blockDim.x;
  // Two blocks per thread stay in flight (this one and the next): their 64
  // bytes are requested before t is known and the tables are built, so the
  // first loads overlap that set-up and HBM latency overlaps the conversions.
  uint4 p0 = make_uint4(0, 0, 0, 0), p1 = p0, q0 = p0, q1 = p0;
  {
    const uint32_t b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < nblocks) { p0 = __ldg(x + 2 * (size_t)b); p1 = __ldg(x + 2 * (size_t)b + 1); }
    if (b + stride < nblocks) { q0 = __ldg(x + 2 * (size_t)(b + stride)); q1 = __ldg(x + 2 * (size_t)(b + stride) + 1); }
  }
  // After the amax pass this kernel is launched early (programmatic dependent
  // launch): x is only read by that pass, so the loads above may start during
  // its tail, but its partials are read only after this wait (a no-op otherwise).
  grid_dependency_wait();
  if (threadIdx.x < 32) {
    float m = 0.f;
    if (t_in == nullptr)
      for (int i = threadIdx.x; i < npartial; i += 32) m = fmaxf(m, __ldcg(partial + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0) {
      const float t = t_in != nullptr ? __ldcg(t_in) : tensor_scale_of(m);
      s_t = t;
      if (blockIdx.x == 0) *t_out = t;
    }
  }
  __syncthreads();
  const float t = s_t;
  // Per E4M3 scale code: the exact thresholds, and whether the fast path
  // (fp32 quotient + cvt) provably agrees with them for every bf16 input: both
  // are monotone in |x|, so agreeing on both sides of every exact threshold
  // means agreeing everywhere.
  // One (code, midpoint) pair per thread: the exact threshold, and for each of
  // the three candidate multipliers whether the fast map gives the exact code on
  // both sides of it ...
  for (uint32_t i = threadIdx.x; i < 127u * 7u; i += blockDim.x) {
    const uint32_t c = i / 7u, j = i - 7u * c;
    uint32_t bits = 0x7F80u, pass = 0u;
    if (c != 0) {
      const float S = e4m3_value(c);
      bits = e2m1_threshold_bits(__fmul_rn(c_e2m1_mid[j], S), t, (int)j);
      const float inv0 = __frcp_rn(__fmul_rn(S, t));
      const float cand[3] = {inv0, __fmul_rn(inv0, kNudgeDown), __fmul_rn(inv0, kNudgeUp)};
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        bool g = !isinf(cand[k]);
        if (bits >= 0x7F80u) {
          g = g && e2m1_fast_code(0x7F7Fu, cand[k]) == j;
        } else {
          g = g && e2m1_fast_code(bits, cand[k]) == j + 1u;
          if (bits > 0u) g = g && e2m1_fast_code(bits - 1u, cand[k]) == j;
        }
        pass |= (g ? 1u : 0u) << k;
      }
    }
    s_b[c][j] = (uint16_t)bits;
    s_ck[c][j] = (uint8_t)pass;
  }
  __syncthreads();
  // ... then one thread per code takes the first candidate that passes all seven
  // (the fast map is then exact for every bf16 input: both maps are monotone in |x|).
  if (threadIdx.x < 127) {
    const uint32_t c = threadIdx.x;
    const float S = e4m3_value(c);
    uint32_t b[7], all = 7u;
#pragma unroll
    for (int i = 0; i < 7; ++i) {
      b[i] = s_b[c][i];
      all &= s_ck[c][i];
    }
    const float d = __fmul_rn(S, t);
    const float inv0 = (c == 0) ? 0.f : __frcp_rn(d);
    float inv = inv0;
    bool ok = (c == 0) || (d >= 1.17549435e-38f && !isinf(inv0));
    if (c != 0 && ok) {
      ok = all != 0u;
      if (all & 1u) inv = inv0;
      else if (all & 2u) inv = __fmul_rn(inv0, kNudgeDown);
      else if (all & 4u) inv = __fmul_rn(inv0, kNudgeUp);
    }
    s_inv_d[c] = inv;
    s_fast_ok[c] = ok ? 1u : 0u;
    s_mid6[c] = c < 126 ? __fmul_rn(6.0f, 0.5f * (S + e4m3_value(c + 1))) : 0.f;
    s_thr[c] = make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16), b[6] | (0x7F80u << 16));
  }
  __syncthreads();

  const float inv6t = __frcp_rn(__fmul_rn(6.0f, t));
  const uint32_t nbk = K >> 4;                               // 16-element blocks per row
  const uint32_t atoms_per_rowtile = K >> 6;
  const uint32_t lane = threadIdx.x & 31u;
  // (row, block-in-row) of this thread's block, advanced without a division.
  const uint32_t b0 = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t row = b0 / nbk, kb = b0 - row * nbk;
  const uint32_t step_r = stride / nbk, step_kb = stride - step_r * nbk;
  for (uint32_t base = blockIdx.x * blockDim.x + (threadIdx.x & ~31u); base < nblocks; base += stride) {
    const uint32_t b = base + lane;
    const bool valid = b < nblocks;                          // nblocks % 4 == 0: groups of 4 agree
    uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    p0 = q0;
    p1 = q1;
    {
      const uint32_t bn = b + 2 * stride;                    // < 2^31 + two grids: no wrap
      if (bn < nblocks) { q0 = __ldg(x + 2 * (size_t)bn); q1 = __ldg(x + 2 * (size_t)bn + 1); }
      else { q0 = make_uint4(0, 0, 0, 0); q1 = q0; }
    }
    uint32_t a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = w[i] & 0x7FFF7FFFu;
    const uint32_t m2 = bf16x2_max(bf16x2_max(bf16x2_max(a[0], a[1]), bf16x2_max(a[2], a[3])),
                                   bf16x2_max(bf16x2_max(a[4], a[5]), bf16x2_max(a[6], a[7])));
    const float amax = bf16x2_hmax_to_f32(m2);
    const uint32_t s = block_scale_code(amax, t, inv6t, s_mid6);
    uint2 c;
    // Warp-uniform choice: the fast path only when it is exact for every
    // block of the warp.  (Per-thread choice made nearly every warp run both
    // paths, since a quarter to a third of the scale codes fail the fast check.)
    if (__all_sync(0xFFFFFFFFu, s_fast_ok[s] != 0u)) {
      const float inv_d = s_inv_d[s];
      c.x = codes8_fast(w, inv_d);
      c.y = codes8_fast(w + 4, inv_d);
    } else {
      const uint4 T = s_thr[s];
      const uint32_t B[7] = {__byte_perm(T.x, 0, 0x1010), __byte_perm(T.x, 0, 0x3232),
                             __byte_perm(T.y, 0, 0x1010), __byte_perm(T.y, 0, 0x3232),
                             __byte_perm(T.z, 0, 0x1010), __byte_perm(T.z, 0, 0x3232),
                             __byte_perm(T.w, 0, 0x1010)};
      c.x = codes8_exact(w, B);
      c.y = codes8_exact(w + 4, B);
    }
    // Gather the 4 scale bytes of an aligned group of 4 blocks (same row, same atom).
    uint32_t sv = s << (8 * (lane & 3u));
    sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 1);
    sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 2);
    if (valid) {
      codes[b] = c;
      if ((lane & 3u) == 0u) {
        const size_t off = ((size_t)(row >> 7) * atoms_per_rowtile + (kb >> 2)) * 512u + (row & 31u) * 16u +
                           ((row & 127u) >> 5) * 4u;
        *reinterpret_cast<uint32_t*>(scales + off) = sv;
      }
    }
    row += step_r;
    kb += step_kb;
    if (kb >= nbk) {
      kb -= nbk;
      ++row;
    }
  }
  // Zero the scales of the padding rows up to the next multiple of 128.
  const uint32_t rows_pad = (rows + 127u) & ~127u;
  const uint32_t npad = (rows_pad - rows) * atoms_per_rowtile;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < npad; i += stride) {
    const uint32_t r = rows + i / atoms_per_rowtile;
    const uint32_t kt = i % atoms_per_rowtile;
    const size_t off = ((size_t)(r >> 7) * atoms_per_rowtile + kt) * 512u + (r & 31u) * 16u + ((r & 127u) >> 5) * 4u;
    *reinterpret_cast<uint32_t*>(scales + off) = 0u;
  }
}

}  // namespace nvq
