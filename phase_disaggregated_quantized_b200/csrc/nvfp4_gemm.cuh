// NVFP4 W4A4 block-scaled GEMM on the sm_100a tensor cores (Mix-Quant page,
// gist.science, section 2.3: the prefill worker runs the W4A4 NVFP4 path; the
// page names Blackwell's microscaling FP4 format, section 2).
//
//   Y[m, n] = bf16( t_x t_w sum_k sx[m, k/16] e2m1(cx[m, k]) * sw[n, k/16] e2m1(cw[n, k]) )
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: per k-stage of 256 elements it loads the A tile
//               (128 rows x 128 bytes, 128B-swizzled), the B tile (256 x 128 B)
//               and the matching 512-byte scale atoms with plain bulk copies.
//   warp 1      MMA issuer: copies the stage's scales into TMEM
//               (tcgen05.cp 32x128b.warpx4) and issues four
//               tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (128 x 256 x 64),
//               accumulating in a 256-column FP32 TMEM accumulator; a
//               tcgen05.commit frees each smem stage when its MMAs are done.
//   warps 2..5  epilogue: drain the accumulator with tcgen05.ld into registers
//               (scaled by t_x t_w, rounded to bf16), release TMEM at once so the
//               next tile's MMAs start, then stage 64-column chunks in 128B-
//               swizzled smem and TMA-store them.
// TMEM: columns [0, 256) accumulator, [256, 256 + 48 * stages) scales
// (per stage: A scales 4 MMAs x 4 columns, B scales 4 MMAs x 8 columns).
#pragma once
#include "ptx.cuh"

namespace nvq {
namespace w4a4 {

constexpr int BM = 128, BN = 256;
constexpr int BKB = 128;                      // k-stage width in bytes (256 FP4 elements)
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BKB;             // 16 KB
constexpr int B_BYTES = BN * BKB;             // 32 KB
constexpr int SFA_BYTES = 4 * 512;            // 4 atoms (128 rows x 4 blocks) per stage
constexpr int SFB_BYTES = 2 * 4 * 512;        // two 128-row halves
constexpr int C_CHUNK_COLS = 64;              // 64 bf16 = 128 bytes per staged row
constexpr int C_BYTES = BM * C_CHUNK_COLS * 2;  // 16 KB per staging buffer
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 256;
constexpr uint32_t SF_COLS_PER_STAGE = 48;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
constexpr int OFF_SFA = OFF_C + 2 * C_BYTES;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 3;
constexpr int OFF_TMEM_PTR = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;   // + slack for 1024-byte alignment

// Instruction descriptor, kind::mxf4nvf4: A/B E2M1 (format 1), K-major,
// UE4M3 scales, N = 256 (bits 17..22 hold N >> 3), M = 128 (bits 24..28 hold M >> 4).
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct Params {
  const uint8_t* x_scales;
  const uint8_t* w_scales;
  const float* t_x;
  const float* t_w;
  uint32_t M, N, K;
  uint32_t num_m_tiles, num_n_tiles, num_k_stages;
  uint32_t k_atoms;        // K / 64: scale atoms per 128-row tile
  uint32_t n_row_atoms;    // padded N / 128
};

__global__ void __launch_bounds__(THREADS, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                  const __grid_constant__ CUtensorMap tmap_y, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t bar_full = sbase + OFF_BAR;                 // + 8 s
  const uint32_t bar_empty = bar_full + 8 * STAGES;         // + 8 s
  const uint32_t bar_acc_full = bar_empty + 8 * STAGES;
  const uint32_t bar_acc_empty = bar_acc_full + 8;
  const uint32_t bar_drain = bar_acc_empty + 8;
  uint32_t* tmem_ptr_smem = reinterpret_cast<uint32_t*>(smem + OFF_TMEM_PTR);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_empty, 4);                             // one arrive per epilogue warp
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tensormap(&tmap_a);
    prefetch_tensormap(&tmap_b);
    prefetch_tensormap(&tmap_y);
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_ptr_smem), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr_smem;

  const uint32_t num_tiles = p.num_m_tiles * p.num_n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      uint32_t stage = 0, phase = 0;
      uint32_t pending = 0, pending_parity = 0;              // per-stage bit masks
      bool ok = true;
      for (uint32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const uint32_t mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
        const uint32_t nb_atoms = min(2u, p.n_row_atoms - 2 * nt);
        for (uint32_t ks = 0; ks < p.num_k_stages; ++ks) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t natoms = min(4u, p.k_atoms - 4 * ks);
          const uint32_t bytes = A_BYTES + B_BYTES + natoms * 512u * (1u + nb_atoms);
          const uint32_t fb = bar_full + 8 * stage;
          mbar_arrive_expect_tx(fb, bytes);
          tma_load_2d(sbase + OFF_A + stage * A_BYTES, &tmap_a, fb, (int)(ks * BKB), (int)(mt * BM), pol);
          tma_load_2d(sbase + OFF_B + stage * B_BYTES, &tmap_b, fb, (int)(ks * BKB), (int)(nt * BN), pol);
          bulk_load(sbase + OFF_SFA + stage * SFA_BYTES,
                    p.x_scales + ((size_t)mt * p.k_atoms + 4 * ks) * 512u, natoms * 512u, fb);
          for (uint32_t a = 0; a < nb_atoms; ++a)
            bulk_load(sbase + OFF_SFB + stage * SFB_BYTES + a * 2048u,
                      p.w_scales + ((size_t)(2 * nt + a) * p.k_atoms + 4 * ks) * 512u, natoms * 512u, fb);
          pending |= 1u << stage;
          pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // Let every copy issued into shared memory land before the CTA exits.
      for (int s2 = 0; s2 < STAGES; ++s2)
        if (pending & (1u << s2)) mbar_wait_drain(bar_full + 8 * s2, (pending_parity >> s2) & 1u, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0, acc_phase = 0;
    bool ok = true;
    for (uint32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      if (!(ok = warp_mbar_wait(bar_acc_empty, acc_phase ^ 1))) break;
      tc_fence_after();
      for (uint32_t ks = 0; ks < p.num_k_stages; ++ks) {
        if (!(ok = warp_mbar_wait(bar_full + 8 * stage, phase))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t natoms = min(4u, p.k_atoms - 4 * ks);
          const uint32_t sf_col = tmem_base + SF_COL0 + stage * SF_COLS_PER_STAGE;
          const uint32_t sfa_smem = sbase + OFF_SFA + stage * SFA_BYTES;
          const uint32_t sfb_smem = sbase + OFF_SFB + stage * SFB_BYTES;
          for (uint32_t j = 0; j < natoms; ++j) {
            tc_cp_32x128b_warpx4(sf_col + 4 * j, smem_desc(sfa_smem + 512 * j, 0, 128, kSwizzleNone));
            tc_cp_32x128b_warpx4(sf_col + 16 + 8 * j, smem_desc(sfb_smem + 512 * j, 0, 128, kSwizzleNone));
            tc_cp_32x128b_warpx4(sf_col + 16 + 8 * j + 4,
                                 smem_desc(sfb_smem + 2048 + 512 * j, 0, 128, kSwizzleNone));
          }
          const uint64_t adesc = smem_desc(sbase + OFF_A + stage * A_BYTES, 0, 1024, kSwizzle128B);
          const uint64_t bdesc = smem_desc(sbase + OFF_B + stage * B_BYTES, 0, 1024, kSwizzle128B);
          for (uint32_t j = 0; j < natoms; ++j) {
            // Advance 32 bytes (64 FP4 elements) along K inside the swizzle atom.
            tc_mma_nvf4(tmem_base, adesc + 2 * j, bdesc + 2 * j, IDESC, sf_col + 4 * j, sf_col + 16 + 8 * j,
                        (ks | j) != 0u);
          }
          tc_commit(bar_empty + 8 * stage);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(bar_acc_full);
      __syncwarp();
      acc_phase ^= 1;
    }
    // Every MMA this thread issued has finished before TMEM is released.
    if (lane == 0) {
      tc_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, 200000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3u;                            // TMEM sub-partition of this warp
    const uint32_t row = q * 32 + lane;                      // row of the tile held by this thread
    const bool issuer = (warp == 2 && lane == 0);
    const float alpha = __ldg(p.t_x) * __ldg(p.t_w);
    uint32_t acc_phase = 0;
    uint32_t chunk_count = 0;
    bool dead = false;                                       // a wait ran out: keep the barrier
    for (uint32_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {  // sequence, skip work
      const uint32_t mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
      if (!dead && !warp_mbar_wait(bar_acc_full, acc_phase)) dead = true;
      uint32_t packed[BN / 2];
      if (!dead) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tc_ld_32x32b_x32(tmem_base + ((q * 32u) << 16) + 32u * c, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float lo = __uint_as_float(v[2 * i]) * alpha, hi = __uint_as_float(v[2 * i + 1]) * alpha;
            uint32_t r;
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
            packed[c * 16 + i] = r;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_acc_empty);
      } else {
#pragma unroll
        for (int i = 0; i < BN / 2; ++i) packed[i] = 0u;
      }
      acc_phase ^= 1;
      // Store 4 chunks of 64 columns through the two swizzled staging buffers.
#pragma unroll
      for (int ch = 0; ch < BN / C_CHUNK_COLS; ++ch) {
        const uint32_t col0 = nt * BN + ch * C_CHUNK_COLS;
        const uint32_t buf = chunk_count & 1u;
        if (issuer) bulk_wait_read<1>();
        named_barrier_sync(1, 128);
        uint8_t* cbuf = smem + OFF_C + buf * C_BYTES;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t sw = ((uint32_t)i ^ (row & 7u)) * 16u;
          uint4 val = make_uint4(packed[ch * 32 + 4 * i], packed[ch * 32 + 4 * i + 1],
                                 packed[ch * 32 + 4 * i + 2], packed[ch * 32 + 4 * i + 3]);
          *reinterpret_cast<uint4*>(cbuf + row * 128u + sw) = val;
        }
        fence_proxy_async_smem();
        named_barrier_sync(1, 128);
        if (issuer && !dead && col0 < p.N) {
          tma_store_2d(&tmap_y, sbase + OFF_C + buf * C_BYTES, (int)col0, (int)(mt * BM));
          bulk_commit();
        }
        ++chunk_count;
      }
    }
    if (issuer) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace w4a4
}  // namespace nvq
