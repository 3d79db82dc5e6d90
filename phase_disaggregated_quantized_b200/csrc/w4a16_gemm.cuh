// W4A16 decode GEMM: Y = X * dequant(W)^T with BF16 activations at small batch
// and INT4 group-128 weights (MARLIN page, abeam.tech, the sections on the
// offline weight reorder and on running the pipeline stages concurrently:
// weights streamed asynchronously past L2 with an evict-first policy,
// dequantization interleaved with tensor-core MMAs, several warps and CTAs
// sharing one output tile by splitting K, partial sums added on chip).
//
// Work split.  The packed weights are a sequence of "groups": 1 KB of codes +
// 32 B of scales for one 16-row tile and 128 consecutive k, tile-major.  Each
// cluster of CS CTAs owns a contiguous run of whole 16-row tiles; inside the
// cluster the run's groups are split evenly over CS CTAs x W warps, so every
// warp streams the same number of bytes whatever N and K are.
//
// Streaming.  Each warp owns a ring of D stages of SG groups in shared memory;
// lane 0 refills a stage with two bulk copies (codes, scales) that complete on
// the stage's mbarrier, so D * SG KB per warp are in flight without holding
// registers.  Activations (a few KB, L1-resident) are read with plain loads one
// group ahead.
//
// Math.  The offline reorder permutes K inside a group so that lane (g, c) of
// k16 step j uses k = 32c + 4j + {0..3}: its 64-byte activation run feeds all
// eight steps.  Nibbles become bf16 (128 + u) through the exponent bits; the
// -136 offset (u - 8 = (128 + u) - 136) is either subtracted in bf16 (exact) or,
// for one batch tile, added by a second MMA of -136 * x into the same FP32
// chain, which costs one tensor-core op instead of four ALU ops.  Each group's
// FP32 sum is scaled by the group's BF16 scale in FP32.
//
// Reduction.  A warp writes tiles it covered entirely straight to Y; the tiles
// at the ends of its range stay in registers, are summed by warp order in
// shared memory, and tiles shared by CTAs of the cluster are summed by rank
// order through distributed shared memory between two cluster barriers.  The
// summation order depends only on the shapes and the grid, so results are
// reproducible run to run.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace nvq {
namespace w4a16 {

constexpr int SG = 4;                        // groups per ring stage
constexpr int CS = 2;                        // CTAs per cluster (74 such pairs fill 148 SMs)
// Bytes of one 16-row x 128-k group: codes (dense 1024; 2:4 sparse 512 of kept
// codes + 256 of metadata) and 32 of scales.
template <bool SPARSE>
struct Unit {
  static constexpr uint32_t CODE = SPARSE ? 768u : 1024u;
  static constexpr uint32_t BYTES = CODE + 32u;
};

template <int NT8, bool SPARSE = false>
struct Cfg {
  static constexpr int W = NT8 == 1 ? 16 : 8;          // warps per CTA (register budget)
  static constexpr int D = NT8 == 1 ? 3 : 6;           // ring stages per warp
  static constexpr int THREADS = W * 32;
  static constexpr int STAGE = SG * Unit<SPARSE>::BYTES;
  static constexpr int RING = W * D * STAGE;
  static constexpr int TILEF = 128 * NT8;               // floats of one 16 x (8 NT8) partial tile
  static constexpr int BARS = RING;                      // W * D stage barriers
  static constexpr int CTA_SLOTS = BARS + W * D * 8;     // 2 CTA partial tiles, read by the cluster
  static constexpr int SMEM = CTA_SLOTS + 2 * TILEF * 4;
  static constexpr bool ONES = NT8 == 1;                 // -136 x through the tensor core
  static_assert(W * 2 * TILEF * 4 <= RING, "warp partial tiles overlay the ring");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// ---------------------------------------------------------------- small PTX helpers
__device__ __forceinline__ void bulk_load_l2hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                                 uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(pol) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(cluster_addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// d (+)= a * b for one m16n8k16 bf16 step; the _z form starts a chain at zero.
__device__ __forceinline__ void mma_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// (v & 0x000F000F) | 0x43004300: two nibbles -> bf16x2 (128 + u).
__device__ __forceinline__ uint32_t nibbles_to_bf16x2(uint32_t v) {
  uint32_t r;
  asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(v));
  return r;
}
__device__ __forceinline__ uint32_t shr32(uint32_t v, uint32_t s) {
  uint32_t r;
  asm("shr.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(s));
  return r;
}
// The eight nibbles of one packed word as A-fragment registers of (128 + u).
__device__ __forceinline__ void word_to_frag(uint32_t w, uint32_t (&a)[4]) {
  a[0] = nibbles_to_bf16x2(w);
  a[1] = nibbles_to_bf16x2(shr32(w, 4));
  a[2] = nibbles_to_bf16x2(shr32(w, 8));
  a[3] = nibbles_to_bf16x2(shr32(w, 12));
}
__device__ __forceinline__ uint32_t bf16x2_sub136(uint32_t v) {
  const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
  __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&v);
  h = __hsub2(h, bias);                                  // exact: (128 + u) - 136 = u - 8
  return *reinterpret_cast<uint32_t*>(&h);
}

// Even split of [0, len) into 2^LOG2P parts: part i starts at len * i / 2^LOG2P.
template <int LOG2P>
__device__ __forceinline__ uint32_t split_at(uint32_t len, uint32_t i) {
  return (uint32_t)(((uint64_t)len * i) >> LOG2P);
}
// The part holding x < len: the largest i with split_at(len, i) <= x (a
// non-empty part, since the next one starts after x).
template <int LOG2P>
__device__ __forceinline__ uint32_t part_of(uint32_t len, uint32_t x) {
  uint32_t i = 0;
#pragma unroll
  for (int b = LOG2P - 1; b >= 0; --b)
    if (split_at<LOG2P>(len, i | (1u << b)) <= x) i |= 1u << b;
  return i;
}
__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

template <int NT8>
__device__ __forceinline__ void zero_tile(float (&a)[NT8][4]) {
#pragma unroll
  for (int t = 0; t < NT8; ++t) a[t][0] = a[t][1] = a[t][2] = a[t][3] = 0.f;
}
template <int NT8>
__device__ __forceinline__ void add_tile(float (&a)[NT8][4], const float* p) {   // p: this lane's 4 NT8 floats
#pragma unroll
  for (int t = 0; t < NT8; ++t) {
    const float4 v = *reinterpret_cast<const float4*>(p + 4 * t);
    a[t][0] += v.x; a[t][1] += v.y; a[t][2] += v.z; a[t][3] += v.w;
  }
}
template <int NT8>
__device__ __forceinline__ void put_tile(float* p, const float (&a)[NT8][4]) {
#pragma unroll
  for (int t = 0; t < NT8; ++t) *reinterpret_cast<float4*>(p + 4 * t) = make_float4(a[t][0], a[t][1], a[t][2], a[t][3]);
}
// C fragment of tile `tn` (weight rows 16 tn + g / + 8, batch columns m0 + 8t + 2c / + 1) -> Y bf16.
template <int NT8>
__device__ __forceinline__ void store_tile(__nv_bfloat16* __restrict__ y, const float (&acc)[NT8][4], uint32_t tn,
                                           uint32_t m0, uint32_t M, uint32_t N, uint32_t lane) {
  const uint32_t n_lo = tn * 16 + (lane >> 2), n_hi = n_lo + 8;
#pragma unroll
  for (int t = 0; t < NT8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t m = m0 + t * 8 + 2 * (lane & 3u) + (e & 1);
      if (m < M) y[(size_t)m * N + ((e & 2) ? n_hi : n_lo)] = __float2bfloat16_rn(acc[t][e]);
    }
}

// Dequantize one group (two 16-byte code vectors of this lane) and run the
// eight k16 steps for every batch tile; t0 / t1 receive the even / odd steps.
template <int NT8, bool ONES>
__device__ __forceinline__ void group_mma(const uint4 wa, const uint4 wb, const uint4 (&xv)[NT8][4],
                                          float (&t0)[NT8][4], float (&t1)[NT8][4]) {
  const uint32_t words[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
  constexpr uint32_t kNeg136 = 0xC308C308u;              // bf16x2 (-136, -136)
  const uint32_t neg[4] = {kNeg136, kNeg136, kNeg136, kNeg136};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t a[4];
    word_to_frag(words[j], a);
    if (!ONES) {
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = bf16x2_sub136(a[i]);
    }
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      // k16 step j reads activation words 2j (b0) and 2j + 1 (b1) of the lane's run.
      const uint4 q = xv[t][j >> 1];
      const uint32_t b0 = (j & 1) ? q.z : q.x;
      const uint32_t b1 = (j & 1) ? q.w : q.y;
      float (&d)[4] = (j & 1) ? t1[t] : t0[t];
      if (j < 2) mma_z(d, a, b0, b1);
      else mma_acc(d, a, b0, b1);
      if (ONES) mma_acc(d, neg, b0, b1);
    }
  }
}

// d += A * B for one m16n8k32 step with a 2:4-sparse A (compressed 16 x 16
// values, metadata e from lanes c = 0, 1 of each quad).
__device__ __forceinline__ void mma_sp_acc(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[4], uint32_t e) {
  asm volatile(
      "mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9,%10,%11}, {%0,%1,%2,%3}, %12, 0x0;"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(e));
}

// One 2:4-sparse unit (16 rows x 128 k, 64 kept codes per row): four m16n8k32
// steps; step s reads runs 8 s .. 8 s + 7 of the group, so lane (g, c) needs
// activations k = 32 s + 16 (c / 2) + {0 .. 15}, of which words c % 2, 2 + c % 2,
// 4 + c % 2, 6 + c % 2 feed its B fragment.  t0 / t1 receive the even / odd steps.
template <int NT8, bool ONES>
__device__ __forceinline__ void sparse_group(uint32_t unit, uint32_t lane, const uint4* const (&xrow)[NT8],
                                             const bool (&live)[NT8], uint32_t gk, float (&t0)[NT8][4],
                                             float (&t1)[NT8][4]) {
  const uint32_t g = lane >> 2, c = lane & 3u, odd = c & 1u;
  const uint4 wq = lds128(unit + lane * 16);
  const uint4 mq = lds128(unit + 512 + (2 * g + odd) * 16);   // lanes c >= 2 load a copy the MMA ignores
  const uint32_t wsw[4] = {wq.x, wq.y, wq.z, wq.w};
  const uint32_t msw[4] = {mq.x, mq.y, mq.z, mq.w};
  constexpr uint32_t kNeg136 = 0xC308C308u;
  const uint32_t neg[4] = {kNeg136, kNeg136, kNeg136, kNeg136};
#pragma unroll
  for (int t = 0; t < NT8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) t0[t][e] = t1[t][e] = 0.f;
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    uint32_t a[4];
    word_to_frag(wsw[st], a);
    if (!ONES) {
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = bf16x2_sub136(a[i]);
    }
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
      if (live[t]) {
        const uint4* px = xrow[t] + gk * 16u + 4u * st + 2u * (c >> 1);
        x0 = __ldg(px);
        x1 = __ldg(px + 1);
      }
      const uint32_t b[4] = {odd ? x0.y : x0.x, odd ? x0.w : x0.z, odd ? x1.y : x1.x, odd ? x1.w : x1.z};
      float (&d)[4] = (st & 1) ? t1[t] : t0[t];
      mma_sp_acc(d, a, b, msw[st]);
      if (ONES) mma_sp_acc(d, neg, b, msw[st]);
    }
  }
}

template <int NT8, bool SPARSE>
__global__ void __launch_bounds__(Cfg<NT8, SPARSE>::THREADS, 1) w4a16_kernel(
    const __nv_bfloat16* __restrict__ x, const uint8_t* __restrict__ pcodes, const uint8_t* __restrict__ pscales,
    __nv_bfloat16* __restrict__ y, uint32_t M, uint32_t N, uint32_t K) {
  using C = Cfg<NT8, SPARSE>;
  constexpr uint32_t UC = Unit<SPARSE>::CODE;
  constexpr int W = C::W, D = C::D;
  constexpr uint32_t MC = 8 * NT8, TILEF = C::TILEF;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t G = K >> 7, ntiles = N >> 4;
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t gl = lane >> 2;
  const uint32_t rank = cluster_rank();
  // This cluster's run of whole tiles, as flat groups [A, A + L).
  // Flat group indices fit in 32 bits (the host rejects N * K / 2048 >= 2^32).
  constexpr int LW = ilog2(W), LCS = ilog2(CS);
  static_assert((1 << LW) == W && (1 << LCS) == CS, "powers of two");
  const uint32_t nclu = cluster_count(), cid = cluster_id();
  const uint32_t tq = ntiles / nclu, tr = ntiles % nclu;
  const uint32_t A = (tq * cid + tr * cid / nclu) * G;
  const uint32_t L = (tq * (cid + 1) + tr * (cid + 1) / nclu) * G - A;
  const uint32_t F0 = A + split_at<LCS>(L, rank), F1 = A + split_at<LCS>(L, rank + 1), FL = F1 - F0;   // this CTA
  const uint32_t f0 = F0 + split_at<LW>(FL, warp), f1 = F0 + split_at<LW>(FL, warp + 1);               // this warp
  const uint32_t nf = (uint32_t)(f1 - f0);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t ring = sbase + warp * D * C::STAGE;
  const uint32_t bars = sbase + C::BARS + warp * D * 8;
  float* wslots = reinterpret_cast<float*>(smem);                       // overlays the ring
  float* cslots = reinterpret_cast<float*>(smem + C::CTA_SLOTS);
  const uint64_t pol = policy_evict_first();
  const uint32_t npass = (M + MC - 1) / MC;
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();
  grid_dependency_wait();                      // before any global access (launched back to back)
  uint32_t cs = 0, phase = 0;                  // ring position of the next stage to consume
  uint32_t in_flight = 0;                      // lane 0: stages issued and not consumed
  bool ok = true;
  const uint32_t wt_first = f0 / G;            // first tile of this warp's range
  const uint32_t g_first = (uint32_t)(f0 - wt_first * G);

  for (uint32_t pass = 0; pass < npass; ++pass) {
    const uint32_t m0 = pass * MC;
    float p0[NT8][4], p1[NT8][4];             // partial tiles at the ends of the warp's range
    zero_tile<NT8>(p0);
    zero_tile<NT8>(p1);
    bool has0 = false, has1 = false;
    if (nf > 0 && ok) {
      // Stages hold up to SG groups and never straddle a tile, so a stage's
      // groups share one tile and consecutive k-groups.
      const uint8_t* wnext = pcodes + (size_t)f0 * UC;
      const uint8_t* snext = pscales + (size_t)f0 * 32;
      uint32_t irem = nf, ig = g_first, islot = cs;
      auto issue = [&]() {                    // lane 0: the next stage of this warp's range
        const uint32_t n = min(min(irem, (uint32_t)SG), G - ig);
        const uint32_t bar = bars + 8 * islot;
        const uint32_t dst = ring + islot * C::STAGE;
        mbar_arrive_expect_tx(bar, n * Unit<SPARSE>::BYTES);
        bulk_load_l2hint(dst, wnext, n * UC, bar, pol);
        bulk_load_l2hint(dst + SG * UC, snext, n * 32u, bar, pol);
        wnext += n * UC;
        snext += n * 32;
        irem -= n;
        ig = ig + n == G ? 0u : ig + n;
        islot = islot + 1 == (uint32_t)D ? 0u : islot + 1;
        ++in_flight;
      };
      if (lane == 0) {
        if (pass > 0) fence_proxy_async_smem();   // ring bytes were partial-tile slots last pass
        for (int s = 0; s < D && irem > 0; ++s) issue();
      }
      // Activation rows of this lane (zero beyond M); two register sets
      // alternate between the group being multiplied and the next one.
      const uint4* xrow[NT8];
      bool live[NT8];
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
        const uint32_t m = m0 + 8 * t + gl;
        live[t] = m < M;
        xrow[t] = reinterpret_cast<const uint4*>(x + (size_t)(live[t] ? m : 0) * K + (SPARSE ? 0u : 32u * (lane & 3u)));
      }
      uint4 xa[NT8][4], xb[NT8][4];
#pragma unroll
      for (int t = 0; t < NT8; ++t)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          xa[t][v] = live[t] ? __ldg(xrow[t] + g_first * 16u + v) : make_uint4(0, 0, 0, 0);
          xb[t][v] = make_uint4(0, 0, 0, 0);
        }
      float acc[NT8][4];
      zero_tile<NT8>(acc);
      uint32_t nt = wt_first, g = g_first, left = nf;
      while (left > 0) {
        if (!mbar_wait(bars + 8 * cs, phase)) { ok = false; break; }
        const uint32_t n = min(min(left, (uint32_t)SG), G - g);
        const uint32_t w_addr = ring + cs * C::STAGE + lane * 16;
        const uint32_t s_addr = ring + cs * C::STAGE + SG * UC + gl * 4;
#pragma unroll
        for (int i = 0; i < SG; ++i) {
          if ((uint32_t)i < n) {
            float t0[NT8][4], t1[NT8][4];
            if constexpr (SPARSE) {
              sparse_group<NT8, C::ONES>(ring + cs * C::STAGE + i * UC, lane, xrow, live, g + i, t0, t1);
            } else {
              uint4 (&cur)[NT8][4] = (i & 1) ? xb : xa;
              uint4 (&nxt)[NT8][4] = (i & 1) ? xa : xb;
              const uint32_t gn = g + i + 1 == G ? 0u : g + i + 1;     // next group's k-block
#pragma unroll
              for (int t = 0; t < NT8; ++t)
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  if (live[t]) nxt[t][v] = __ldg(xrow[t] + gn * 16u + v);
              const uint4 wa = lds128(w_addr + i * UC);
              const uint4 wb = lds128(w_addr + i * UC + 512);
              group_mma<NT8, C::ONES>(wa, wb, cur, t0, t1);
            }
            const uint32_t scw = lds32(s_addr + i * 32);
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
        if (!SPARSE && (n & 1)) {             // the next group's activations sit in xb
#pragma unroll
          for (int t = 0; t < NT8; ++t)
#pragma unroll
            for (int v = 0; v < 4; ++v) xa[t][v] = xb[t][v];
        }
        __syncwarp();                         // every lane has read the stage
        if (lane == 0) {
          --in_flight;
          if (irem > 0) issue();
        }
        cs = cs + 1 == (uint32_t)D ? 0u : cs + 1;
        phase ^= cs == 0 ? 1u : 0u;
        g += n;
        left -= n;
        if (g == G) {                         // tile nt ends inside this warp's range
          if (nt == wt_first && g_first != 0) {
#pragma unroll
            for (int t = 0; t < NT8; ++t)
#pragma unroll
              for (int e = 0; e < 4; ++e) p0[t][e] = acc[t][e];
            has0 = true;
          } else {
            store_tile<NT8>(y, acc, nt, m0, M, N, lane);
          }
          zero_tile<NT8>(acc);
          g = 0;
          ++nt;
        }
      }
      if (ok && g != 0) {                     // range ends inside tile nt
        if (nt == wt_first) {
#pragma unroll
          for (int t = 0; t < NT8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) p0[t][e] = acc[t][e];
          has0 = true;
        } else {
#pragma unroll
          for (int t = 0; t < NT8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) p1[t][e] = acc[t][e];
          has1 = true;
        }
      }
    }

    if (pass + 1 == npass) grid_launch_dependents();   // the next kernel may start launching
    // ---- warps -> CTA: partial tiles summed in warp order through shared memory
    __syncthreads();                          // all rings idle: the slots may overlay them
    if (has0) put_tile<NT8>(wslots + (warp * 2 + 0) * TILEF + lane * 4 * NT8, p0);
    if (has1) put_tile<NT8>(wslots + (warp * 2 + 1) * TILEF + lane * 4 * NT8, p1);
    __syncthreads();
    const uint32_t t_lo = F0 / G;
    if (FL > 0) {
      const uint32_t t_hi = (F1 - 1) / G;
      for (uint32_t tt = t_lo + warp; tt <= t_hi; tt += W) {
        const uint32_t lo = tt * G > F0 ? tt * G : F0;
        const uint32_t hi = (tt + 1) * G < F1 ? (tt + 1) * G : F1;
        const uint32_t wa = part_of<LW>(FL, lo - F0), wb = part_of<LW>(FL, hi - 1 - F0);
        const uint32_t f0a = F0 + split_at<LW>(FL, wa), f1a = F0 + split_at<LW>(FL, wa + 1);
        if (wa == wb && f0a <= tt * G && f1a >= (tt + 1) * G) continue;   // its warp stored it
        float s[NT8][4];
        zero_tile<NT8>(s);
        for (uint32_t w2 = wa; w2 <= wb; ++w2) {
          const uint32_t f0w = F0 + split_at<LW>(FL, w2);
          if (f0w == F0 + split_at<LW>(FL, w2 + 1)) continue;              // empty range
          add_tile<NT8>(s, wslots + (w2 * 2 + ((f0w / G == tt) ? 0 : 1)) * TILEF + lane * 4 * NT8);
        }
        if (lo == tt * G && hi == (tt + 1) * G) store_tile<NT8>(y, s, tt, m0, M, N, lane);
        else put_tile<NT8>(cslots + ((tt == t_lo) ? 0 : 1) * TILEF + lane * 4 * NT8, s);
      }
    }
    // ---- CTAs -> cluster: a tile cut by a CTA boundary is finished by the CTA
    // holding its last group (for which it is the first tile), summing the
    // ranks' partials in rank order through distributed shared memory.
    cluster_sync();
    if (FL > 0 && warp == 0 && t_lo * G < F0 && (t_lo + 1) * G <= F1) {
      const uint32_t r_first = part_of<LCS>(L, t_lo * G - A);
      float s[NT8][4];
      zero_tile<NT8>(s);
      for (uint32_t r = r_first; r <= rank; ++r) {
        const uint32_t F0r = A + split_at<LCS>(L, r);
        if (F0r == A + split_at<LCS>(L, r + 1)) continue;                 // empty rank
        const uint32_t off = C::CTA_SLOTS + ((F0r / G == t_lo) ? 0u : 1u) * TILEF * 4 + lane * 16 * NT8;
        if (r == rank) {
          add_tile<NT8>(s, reinterpret_cast<const float*>(smem + off));
        } else {
          const uint32_t ra = map_to_rank(sbase + off, r);
#pragma unroll
          for (int t = 0; t < NT8; ++t) {
            const float4 v = ld_dsmem_f4(ra + 16 * t);
            s[t][0] += v.x; s[t][1] += v.y; s[t][2] += v.z; s[t][3] += v.w;
          }
        }
      }
      store_tile<NT8>(y, s, t_lo, m0, M, N, lane);
    }
    cluster_sync();                           // partials stay readable until every rank is done
  }
  if (!ok && lane == 0) {                     // let copies already in flight land before exit
    for (uint32_t r = 0; r < in_flight; ++r) {
      mbar_wait_drain(bars + 8 * cs, phase, 200000000ull);
      cs = cs + 1 == (uint32_t)D ? 0u : cs + 1;
      phase ^= cs == 0 ? 1u : 0u;
    }
  }
}

}  // namespace w4a16
}  // namespace nvq
