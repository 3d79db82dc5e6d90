// W4A16 decode GEMM: Y = X * dequant(W)^T with BF16 activations at small batch
// and INT4 group-128 weights (MARLIN page, abeam.tech, the sections on the
// offline weight reorder and on running the pipeline stages concurrently:
// weights streamed asynchronously past L2 with an evict-first policy,
// dequantization interleaved with tensor-core MMAs, several warps and CTAs
// sharing one output tile by splitting K, partial sums added on chip).
//
// Work split.  The packed weights are a sequence of "units": one 128-wide
// k-group of a tile of weight rows, tile-major.  Units hold 32 rows (two 16-row
// MMA tiles): dense 2 KB of codes + 64 B of scales, 2:4-sparse 1536 B of codes
// and metadata + 64 B of scales.  Each cluster of CS CTAs
// owns a contiguous run of whole tiles; inside the cluster the run's units are
// split evenly over CS CTAs x W warps, so every warp streams the same number of
// bytes whatever N and K are.
//
// Streaming.  Each warp owns a ring of D stages of SG units in shared memory;
// lane 0 refills a stage with two bulk copies (codes, scales) that complete on
// the stage's mbarrier, so a few KB per warp are in flight without holding
// registers.  Activations (a few KB, L1-resident) are read with plain loads one
// unit ahead.
//
// Math.  The offline reorder permutes K inside a group so that lane (g, c) of
// k16 step j uses k = 32c + 4j + {0..3}: its 64-byte activation run feeds all
// eight steps of both tiles of a dense unit.  Nibbles become bf16 (128 + u)
// through the exponent bits.  The -136 offset (u - 8 = (128 + u) - 136) is
// either subtracted in bf16 (exact; always so for 2:4-sparse units) or, for
// dense units with up to two batch tiles, formed once per unit as the chain
// -136 * sum(x) on the tensor core: with two batch tiles passed as the C input
// of both tiles' first MMA; with one, run independently of the weight chains
// and added to their sums at the end (a shorter dependent path per unit).
// Either way it costs no dequantization work.  Each group's FP32
// sum is scaled by the group's BF16 scale in FP32.
//
// Reduction.  A warp writes tiles it covered entirely straight to Y; the tiles
// at the ends of its range stay in registers and are summed by warp order in
// shared memory.  The one tile a cluster's two CTAs share (cut by their
// boundary) is finished by rank 1: rank 0 pushes its partial into rank 1's
// shared memory with st.async, which completes on rank 1's mbarrier, and rank 1
// adds it before its own (rank order).  No cluster-wide barrier sits on the
// exit path.  The summation order depends only on the shapes and the grid, so
// results are reproducible run to run.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace nvq {
namespace w4a16 {

constexpr int CS = 2;                        // CTAs per cluster (74 such pairs fill 148 SMs)

template <bool SPARSE>
struct Unit {
  static constexpr uint32_t TILES = 2u;                   // 16-row MMA tiles per unit
  static constexpr uint32_t ROWS = 16u * TILES;           // weight rows of one output tile
  static constexpr uint32_t TILE_CODE = SPARSE ? 768u : 1024u;
  static constexpr uint32_t CODE = TILES * TILE_CODE;
  static constexpr uint32_t SCALE = 32u * TILES;
  static constexpr uint32_t BYTES = CODE + SCALE;
};

template <int NT8, bool SPARSE = false>
struct Cfg {
  using U = Unit<SPARSE>;
  static constexpr int W = 8;                          // warps per CTA (two CTAs per SM)
  static constexpr int SG = 3;                         // units per ring stage
  static constexpr int D = NT8 == 1 ? 2 : 3;           // ring stages per warp (more shared memory leaves less L1 for x)
  static constexpr int THREADS = W * 32;
  static constexpr int MIN_CTAS = NT8 == 1 ? 2 : 1;     // CTAs per SM the register budget must allow
  static constexpr int STAGE = SG * U::BYTES;           // codes first, then the scales
  static constexpr int RING = W * D * STAGE;
  static constexpr int NTT = (int)U::TILES * NT8;       // 16 x 8 accumulator fragments per lane
  static constexpr int TILEF = 128 * NTT;               // floats of one partial output tile
  static constexpr int BARS = RING;                      // W * D stage barriers
  static constexpr int XSLOT = (BARS + W * D * 8 + 15) / 16 * 16;   // 2 receive slots (pass parity)
  static constexpr int XBARS = XSLOT + 2 * TILEF * 4;    // receive-full [2], slot-free [2] barriers
  static constexpr int SMEM = XBARS + 32;
  static constexpr bool ONES = NT8 <= 2;                 // dense units: -136 x through the tensor core
  static constexpr bool XDB = NT8 <= 2;                  // activations double-buffered one unit ahead
  static constexpr bool LATE = NT8 == 1;                  // -136 chain summed after the weight chains
  static_assert(STAGE % 16 == 0 && (SG * U::CODE) % 16 == 0, "bulk-copy alignment");
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
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16 bytes into the shared memory of another CTA of the cluster; the bytes
// count toward the transaction count of that CTA's mbarrier `rbar`.
__device__ __forceinline__ void st_async_f4(uint32_t raddr, const float (&v)[4], uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
               ::"r"(raddr), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "r"(rbar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t rbar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(rbar) : "memory");
}
// Bounded wait (cluster-scope acquire: the data came from another CTA).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    if (ok) return true;
    if ((it & 255u) == 255u) {
      if (error_raised()) return false;
      if (globaltimer() - t0 > kWaitLimitNs) { flag_error(kErrTimeout); return false; }
    }
  }
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

// d = a * b + c for one m16n8k16 bf16 step (register-only: the compiler may
// schedule these freely); the _acc form accumulates, the _z form starts at 0.
__device__ __forceinline__ void mma_c(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                      const float (&c)[4]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}
__device__ __forceinline__ void mma_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
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
__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

// Accumulator of one output tile: NTT = (16-row tiles) x (8-column batch tiles)
// m16n8 fragments, fragment index tt * NT8 + t.
template <int NTT>
__device__ __forceinline__ void zero_tile(float (&a)[NTT][4]) {
#pragma unroll
  for (int t = 0; t < NTT; ++t) a[t][0] = a[t][1] = a[t][2] = a[t][3] = 0.f;
}
template <int NTT>
__device__ __forceinline__ void copy_tile(float (&d)[NTT][4], const float (&a)[NTT][4]) {
#pragma unroll
  for (int t = 0; t < NTT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) d[t][e] = a[t][e];
}
template <int NTT>
__device__ __forceinline__ void add_tile(float (&a)[NTT][4], const float* p) {   // p: this lane's 4 NTT floats
#pragma unroll
  for (int t = 0; t < NTT; ++t) {
    const float4 v = *reinterpret_cast<const float4*>(p + 4 * t);
    a[t][0] += v.x; a[t][1] += v.y; a[t][2] += v.z; a[t][3] += v.w;
  }
}
template <int NTT>
__device__ __forceinline__ void put_tile(float* p, const float (&a)[NTT][4]) {
#pragma unroll
  for (int t = 0; t < NTT; ++t) *reinterpret_cast<float4*>(p + 4 * t) = make_float4(a[t][0], a[t][1], a[t][2], a[t][3]);
}
// C fragments of output tile `tn` (16-row MMA tile tt: weight rows ROWS tn + 16 tt + g / + 8;
// batch columns m0 + 8t + 2c / + 1) -> Y bf16.
template <int TILES, int NT8>
__device__ __forceinline__ void store_tile(__nv_bfloat16* __restrict__ y, const float (&acc)[TILES * NT8][4],
                                           uint32_t tn, uint32_t m0, uint32_t M, uint32_t N, uint32_t lane) {
#pragma unroll
  for (int tt = 0; tt < TILES; ++tt) {
    const uint32_t n_lo = (tn * TILES + tt) * 16 + (lane >> 2), n_hi = n_lo + 8;
#pragma unroll
    for (int t = 0; t < NT8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t m = m0 + t * 8 + 2 * (lane & 3u) + (e & 1);
        if (m < M) y[(size_t)m * N + ((e & 2) ? n_hi : n_lo)] = __float2bfloat16_rn(acc[tt * NT8 + t][e]);
      }
  }
}

// One dense unit: 32 rows x 128 k, lane-major words.  LDS q (q = 0..3) of a
// lane holds k16 steps 2q and 2q + 1 of MMA tiles 0 and 1: component
// 2 (j & 1) + tt.  d[tt * NT8 + t] receives the group sum of tile tt, batch tile t.
// LATE: the weight chains start from zero, independent of the -136 chain, and
// its sum is added at the end (a shorter dependent path per unit).
template <int NT8, bool ONES, bool LATE>
__device__ __forceinline__ void dense_unit(uint32_t addr, const uint4 (&xv)[NT8][4], float (&d)[2 * NT8][4]) {
  uint4 wq[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) wq[q] = lds128(addr + 512 * q);
  float offs[NT8][4];
  if constexpr (ONES) {                       // offs = -136 * sum_k x, the same for every weight row
    constexpr uint32_t kNeg136 = 0xC308C308u;              // bf16x2 (-136, -136)
    const uint32_t neg[4] = {kNeg136, kNeg136, kNeg136, kNeg136};
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
        const uint4 q = xv[t][j >> 1];
        const uint32_t b0 = (j & 1) ? q.z : q.x, b1 = (j & 1) ? q.w : q.y;
        if (j == 0) mma_z(offs[t], neg, b0, b1);
        else mma_acc(offs[t], neg, b0, b1);
      }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 v = wq[j >> 1];
    uint32_t a0[4], a1[4];
    word_to_frag((j & 1) ? v.z : v.x, a0);
    word_to_frag((j & 1) ? v.w : v.y, a1);
    if constexpr (!ONES) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a0[i] = bf16x2_sub136(a0[i]);
        a1[i] = bf16x2_sub136(a1[i]);
      }
    }
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      // k16 step j reads activation words 2j (b0) and 2j + 1 (b1) of the lane's run.
      const uint4 q = xv[t][j >> 1];
      const uint32_t b0 = (j & 1) ? q.z : q.x, b1 = (j & 1) ? q.w : q.y;
      if (j == 0) {
        if constexpr (ONES && !LATE) {
          mma_c(d[t], a0, b0, b1, offs[t]);
          mma_c(d[NT8 + t], a1, b0, b1, offs[t]);
        } else {
          mma_z(d[t], a0, b0, b1);
          mma_z(d[NT8 + t], a1, b0, b1);
        }
      } else {
        mma_acc(d[t], a0, b0, b1);
        mma_acc(d[NT8 + t], a1, b0, b1);
      }
    }
  }
  if constexpr (ONES && LATE) {
#pragma unroll
    for (int f = 0; f < 2 * NT8; ++f)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[f][e] += offs[f % NT8][e];
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

// One 2:4-sparse unit: two 16-row tiles x 128 k (64 kept codes per row), each
// 512 bytes of code words and 256 of metadata words; four m16n8k32 steps per
// tile.  Step s reads runs 8 s .. 8 s + 7 of the group, so lane (g, c) needs
// activations k = 32 s + 16 (c / 2) + {0 .. 15}, of which words c % 2,
// 2 + c % 2, 4 + c % 2, 6 + c % 2 feed its B fragment; the activations of a
// step are loaded once for both tiles.  d[tt * NT8 + t] receives the group sum.
// The -136 offset is taken off each kept weight before the MMA (bf16x2
// subtract, exact): the offset a dense unit gets from one -136 * sum(x) chain
// would here need a second sparse MMA per step, since which activations meet
// a kept weight depends on the row's metadata.
template <int NT8>
__device__ __forceinline__ void sparse_unit(uint32_t unit, uint32_t lane, const uint4* const (&xrow)[NT8],
                                            uint32_t gk, float (&d)[2 * NT8][4]) {
  const uint32_t g = lane >> 2, c = lane & 3u, odd = c & 1u;
  uint32_t wsw[2][4], msw[2][4];
#pragma unroll
  for (int tt = 0; tt < 2; ++tt) {
    const uint4 wq = lds128(unit + tt * 768u + lane * 16);
    const uint4 mq = lds128(unit + tt * 768u + 512 + (2 * g + odd) * 16);   // lanes c >= 2: a copy the MMA ignores
    wsw[tt][0] = wq.x; wsw[tt][1] = wq.y; wsw[tt][2] = wq.z; wsw[tt][3] = wq.w;
    msw[tt][0] = mq.x; msw[tt][1] = mq.y; msw[tt][2] = mq.z; msw[tt][3] = mq.w;
  }
#pragma unroll
  for (int t = 0; t < 2 * NT8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) d[t][e] = 0.f;
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    uint32_t b[NT8][4];
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      const uint4* px = xrow[t] + gk * 16u + 4u * st + 2u * (c >> 1);   // rows >= M read row 0 (discarded)
      const uint4 x0 = __ldg(px), x1 = __ldg(px + 1);
      b[t][0] = odd ? x0.y : x0.x;
      b[t][1] = odd ? x0.w : x0.z;
      b[t][2] = odd ? x1.y : x1.x;
      b[t][3] = odd ? x1.w : x1.z;
    }
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      uint32_t a[4];
      word_to_frag(wsw[tt][st], a);
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = bf16x2_sub136(a[i]);
#pragma unroll
      for (int t = 0; t < NT8; ++t) mma_sp_acc(d[tt * NT8 + t], a, b[t], msw[tt][st]);
    }
  }
}

template <int NT8, bool SPARSE>
__global__ void __launch_bounds__(Cfg<NT8, SPARSE>::THREADS, Cfg<NT8, SPARSE>::MIN_CTAS) w4a16_kernel(
    const __nv_bfloat16* __restrict__ x, const uint8_t* __restrict__ pcodes, const uint8_t* __restrict__ pscales,
    __nv_bfloat16* __restrict__ y, uint32_t M, uint32_t N, uint32_t K) {
  using C = Cfg<NT8, SPARSE>;
  using U = typename C::U;
  constexpr uint32_t UC = U::CODE, USC = U::SCALE;
  constexpr int W = C::W, D = C::D, SG = C::SG, NTT = C::NTT, TILES = (int)U::TILES;
  constexpr uint32_t MC = 8 * NT8, TILEF = C::TILEF;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t G = K >> 7, ntiles = N / U::ROWS;
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t gl = lane >> 2;
  const uint32_t rank = cluster_rank();
  // This cluster's run of whole tiles, as flat units [A, A + L).
  // Flat unit indices fit in 32 bits (the host rejects larger N * K).
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
  const float* xslots = reinterpret_cast<const float*>(smem + C::XSLOT);
  const uint32_t rbar = sbase + C::XBARS, fbar = rbar + 16;   // [2] each, indexed by pass parity
  const uint64_t pol = policy_evict_first();
  const uint32_t npass = (M + MC - 1) / MC;
  static_assert(CS == 2, "the cross-CTA exchange is written for CTA pairs");
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(bars + 8 * s, 1);
    if (warp == 0)
      for (int i = 0; i < 2; ++i) {
        mbar_init(rbar + 8 * i, 1);
        mbar_init(fbar + 8 * i, 1);
      }
    fence_mbar_init();
  }
  __syncwarp();
  cluster_arrive();                            // the partner may use this CTA's barriers after its wait
  uint32_t cs = 0, phase = 0;                  // ring position of the next stage to consume
  uint32_t in_flight = 0;                      // lane 0: stages issued and not consumed
  bool ok = true;
  const uint32_t wt_first = f0 / G;            // first tile of this warp's range
  const uint32_t g_first = (uint32_t)(f0 - wt_first * G);
  // Stages hold up to SG units and never straddle a tile, so a stage's units
  // share one tile and consecutive k-groups.  Issue state of the current pass:
  const uint8_t* wnext = pcodes + (size_t)f0 * UC;
  const uint8_t* snext = pscales + (size_t)f0 * USC;
  uint32_t irem = nf, ig = g_first, islot = cs;
  auto issue = [&]() {                        // lane 0: the next stage of this warp's range
    const uint32_t n = min(min(irem, (uint32_t)SG), G - ig);
    const uint32_t bar = bars + 8 * islot;
    const uint32_t dst = ring + islot * C::STAGE;
    mbar_arrive_expect_tx(bar, n * U::BYTES);
    bulk_load_l2hint(dst, wnext, n * UC, bar, pol);
    bulk_load_l2hint(dst + SG * UC, snext, n * USC, bar, pol);
    wnext += n * UC;
    snext += n * USC;
    irem -= n;
    ig = ig + n == G ? 0u : ig + n;
    islot = islot + 1 == (uint32_t)D ? 0u : islot + 1;
    ++in_flight;
  };
  // The packed weights are constant inputs: the first stages are requested
  // before waiting for the preceding kernel (programmatic dependent launch),
  // so their latency overlaps its tail.  Activations and Y wait.
  if (lane == 0)
    for (int s = 0; s < D && irem > 0; ++s) issue();
  grid_dependency_wait();                      // before any access to x or y
  // Let the next kernel launch now: its CTAs take each SM slot that a CTA of
  // this grid frees and request their own first weight stages during this
  // grid's tail.  (Its own wait still holds its x and y until this grid is done.)
  grid_launch_dependents();

  for (uint32_t pass = 0; pass < npass; ++pass) {
    const uint32_t m0 = pass * MC;
    float p0[NTT][4];                         // partial tile at the start of the warp's range
    float acc[NTT][4];                        // the tile being accumulated (partial at the end)
    zero_tile<NTT>(p0);
    zero_tile<NTT>(acc);
    bool has0 = false, has1 = false;
    if (nf > 0 && ok) {
      if (pass > 0) {                         // the same weights again for the next batch rows
        wnext = pcodes + (size_t)f0 * UC;
        snext = pscales + (size_t)f0 * USC;
        irem = nf;
        ig = g_first;
        islot = cs;
        if (lane == 0) {
          fence_proxy_async_smem();           // ring bytes were partial-tile slots last pass
          for (int s = 0; s < D && irem > 0; ++s) issue();
        }
      }
      // Activation rows of this lane (row 0 beyond M: read, then discarded); for XDB two register
      // sets alternate between the unit being multiplied and the next one,
      // otherwise (the register budget of 4 batch tiles) each unit loads its own.
      const uint4* xrow[NT8];
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
        const uint32_t m = m0 + 8 * t + gl;
        xrow[t] = reinterpret_cast<const uint4*>(x + (size_t)(m < M ? m : 0) * K + (SPARSE ? 0u : 32u * (lane & 3u)));
      }
      uint4 xa[NT8][4], xb[NT8][4];
#pragma unroll
      for (int t = 0; t < NT8; ++t)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          xa[t][v] = (!SPARSE && C::XDB) ? __ldg(xrow[t] + g_first * 16u + v) : make_uint4(0, 0, 0, 0);
          xb[t][v] = make_uint4(0, 0, 0, 0);
        }
      uint32_t nt = wt_first, g = g_first, left = nf;
      while (left > 0) {
        if (!mbar_wait(bars + 8 * cs, phase)) { ok = false; break; }
        const uint32_t n = min(min(left, (uint32_t)SG), G - g);
        const uint32_t stage = ring + cs * C::STAGE;
        const uint32_t s_addr = stage + SG * UC + gl * (4u * TILES);
#pragma unroll
        for (int i = 0; i < SG; ++i) {
          if ((uint32_t)i < n) {
            float d[NTT][4];
            if constexpr (SPARSE) {
              sparse_unit<NT8>(stage + i * UC, lane, xrow, g + i, d);
            } else if constexpr (C::XDB) {
              uint4 (&cur)[NT8][4] = (i & 1) ? xb : xa;
              uint4 (&nxt)[NT8][4] = (i & 1) ? xa : xb;
              const uint32_t gn = g + i + 1 == G ? 0u : g + i + 1;     // next unit's k-group
#pragma unroll
              for (int t = 0; t < NT8; ++t)
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  nxt[t][v] = __ldg(xrow[t] + gn * 16u + v);      // rows >= M read row 0 (discarded)
              dense_unit<NT8, C::ONES, C::LATE>(stage + i * UC + lane * 16, cur, d);
            } else {
#pragma unroll
              for (int t = 0; t < NT8; ++t)
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  xa[t][v] = __ldg(xrow[t] + (g + i) * 16u + v);
              dense_unit<NT8, C::ONES, C::LATE>(stage + i * UC + lane * 16, xa, d);
            }
            // Scale word tt of this lane: rows 16 tt + g (low half) and 16 tt + g + 8 (high half).
            uint32_t scw[TILES];
            if constexpr (TILES == 2) {
              const uint2 v = lds64(s_addr + i * USC);
              scw[0] = v.x;
              scw[TILES - 1] = v.y;
            } else {
              scw[0] = lds32(s_addr + i * USC);
            }
#pragma unroll
            for (int tt = 0; tt < TILES; ++tt) {
              const float s_lo = __uint_as_float(scw[tt] << 16), s_hi = __uint_as_float(scw[tt] & 0xFFFF0000u);
#pragma unroll
              for (int t = 0; t < NT8; ++t) {
                float (&a)[4] = acc[tt * NT8 + t];
                const float (&dd)[4] = d[tt * NT8 + t];
                a[0] = __fmaf_rn(s_lo, dd[0], a[0]);
                a[1] = __fmaf_rn(s_lo, dd[1], a[1]);
                a[2] = __fmaf_rn(s_hi, dd[2], a[2]);
                a[3] = __fmaf_rn(s_hi, dd[3], a[3]);
              }
            }
          }
        }
        if (!SPARSE && C::XDB && (n & 1)) {   // the next unit's activations sit in xb
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
            copy_tile<NTT>(p0, acc);
            has0 = true;
          } else {
            store_tile<TILES, NT8>(y, acc, nt, m0, M, N, lane);
          }
          zero_tile<NTT>(acc);
          g = 0;
          ++nt;
        }
      }
      if (ok && g != 0) {                     // range ends inside tile nt
        if (nt == wt_first) {
          copy_tile<NTT>(p0, acc);
          has0 = true;
        } else {
          has1 = true;                        // acc holds it
        }
      }
    }

    // ---- warps -> CTA: partial tiles summed in warp order through shared memory
    __syncthreads();                          // all rings idle: the slots may overlay them
    if (has0) put_tile<NTT>(wslots + (warp * 2 + 0) * TILEF + lane * 4 * NTT, p0);
    if (has1) put_tile<NTT>(wslots + (warp * 2 + 1) * TILEF + lane * 4 * NTT, acc);
    __syncthreads();
    if (pass == 0) cluster_wait();            // the partner's barriers are initialised
    if (FL > 0) {
      const uint32_t t_lo = F0 / G, t_hi = (F1 - 1) / G;
      const uint32_t par = pass & 1u, use = (pass >> 1) & 1u;
      for (uint32_t tt = t_lo + warp; tt <= t_hi; tt += W) {
        const uint32_t tb = tt * G, te = tb + G;
        const bool whole = tb >= F0 && te <= F1;          // the tile lies inside this CTA's range
        // Warp w2's slot for this tile: 0 if the tile is the first of its range, else 1.
        // A tile that one warp covered whole was stored by that warp.  All
        // loads are issued (slots always hold readable bytes), the sum keeps
        // the warps that meet the tile, in warp order.
        float s[NTT][4];
        zero_tile<NTT>(s);
        bool any = false;
#pragma unroll
        for (int w2 = 0; w2 < W; ++w2) {
          const uint32_t a = F0 + split_at<LW>(FL, w2), b = F0 + split_at<LW>(FL, w2 + 1);
          const bool take = a < b && a < te && b > tb && !(a <= tb && b >= te);
          const float* q = wslots + (w2 * 2 + (a >= tb ? 0 : 1)) * TILEF + lane * 4 * NTT;
#pragma unroll
          for (int t = 0; t < NTT; ++t) {
            const float4 v = *reinterpret_cast<const float4*>(q + 4 * t);
            if (take) { s[t][0] += v.x; s[t][1] += v.y; s[t][2] += v.z; s[t][3] += v.w; }
          }
          any |= take;
        }
        if (whole) {
          if (any) store_tile<TILES, NT8>(y, s, tt, m0, M, N, lane);
        } else if (te > F1) {
          // Rank 0's last tile continues in rank 1: push the partial there.
          if (pass >= 2 && !mbar_wait_cluster(fbar + 8 * par, use ^ 1u)) { ok = false; continue; }
          const uint32_t dst = map_to_rank(sbase + C::XSLOT + par * TILEF * 4 + lane * 16 * NTT, 1);
          const uint32_t rb = map_to_rank(rbar + 8 * par, 1);
#pragma unroll
          for (int t = 0; t < NTT; ++t) st_async_f4(dst + 16 * t, s[t], rb);
        } else {
          // Rank 1's first tile began in rank 0: its partial comes first.
          if (lane == 0) mbar_arrive_expect_tx(rbar + 8 * par, TILEF * 4);
          if (!mbar_wait_cluster(rbar + 8 * par, use)) { ok = false; continue; }
          float r[NTT][4];
          zero_tile<NTT>(r);
          add_tile<NTT>(r, xslots + par * TILEF + lane * 4 * NTT);
#pragma unroll
          for (int t = 0; t < NTT; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) r[t][e] += s[t][e];
          store_tile<TILES, NT8>(y, r, tt, m0, M, N, lane);
          __syncwarp();                        // every lane has read the slot
          if (lane == 0 && pass + 2 < npass) mbar_arrive_remote(map_to_rank(fbar + 8 * par, 0));
        }
      }
    }
    if (pass + 1 < npass) __syncthreads();    // slots read before the ring is refilled
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
