// NVFP4 W4A4 block-scaled GEMM on the sm_100a tensor cores (Mix-Quant page,
// gist.science, section 2.3: the prefill worker runs the W4A4 NVFP4 path; the
// page names Blackwell's microscaling FP4 format, section 2).
//
//   Y[m, n] = bf16( t_x t_w sum_k sx[m, k/16] e2m1(cx[m, k]) * sw[n, k/16] e2m1(cw[n, k]) )
//
// Design (one CTA per SM, persistent over 128 x BN output tiles, BN = 192):
//   warp 0      TMA producer: per k-stage of 256 elements it loads the A tile
//               (128 rows x 128 bytes, 128B-swizzled), the B tile (BN x 128 B)
//               and the 512-byte scale atoms covering those rows (plain bulk copies).
//   warp 1      MMA issuer: for each 64-wide k step copies that step's scales
//               into TMEM (tcgen05.cp 32x128b.warpx4, two alternating regions)
//               and issues one tcgen05.mma.kind::mxf4nvf4.block_scale.block16
//               (128 x BN x 64) into one of two FP32 TMEM accumulators; a
//               tcgen05.commit frees each smem stage when its MMAs are done and
//               marks an accumulator full after a tile's last k step.
//   warps 2..5  epilogue: per accumulator, 32-column chunks are read with
//               tcgen05.ld, scaled by t_x t_w, rounded to bf16, staged in 64B-
//               swizzled smem and TMA-stored; the accumulator is released after
//               the last chunk is read, so the next-but-one tile can reuse it
//               while this tile's stores drain.  Two accumulators let the MMAs
//               of tile i+1 run during the epilogue of tile i.
// TMEM (512 columns): accumulators [0, BN) and [BN, 2 BN); the rest is a ring of
// 12-column scale slots, one per MMA (A scales 4 columns, B scales 2 atoms x 4),
// so a slot is rewritten only several MMAs after the MMA that read it.
// The B-scale address is shifted by (n0 % 128) / 32 columns so that column j
// holds tile rows 32 j .. 32 j + 31.  That shift must be even (a 224-wide tile,
// whose shifts include 1 and 3, raised a misaligned-address error), so BN is a
// multiple of 64.
#pragma once
#include "ptx.cuh"

namespace nvq {
namespace w4a4 {

constexpr int BM = 128;
constexpr int BKB = 128;                      // k-stage width in bytes (256 FP4 elements)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BKB;             // 16 KB
constexpr int SFA_BYTES = 4 * 512;            // 4 k-atoms of 128 rows
constexpr int SFB_ATOMS = 2;                  // 128-row scale atoms a 192-row B tile can touch
constexpr uint32_t SF_SLOT_COLS = 12;         // A: 4 columns, B: 2 atoms x 4 columns
constexpr int SFB_BYTES = SFB_ATOMS * 4 * 512;
constexpr int C_COLS = 32;                    // epilogue chunk: 32 bf16 = 64-byte rows
constexpr int C_BYTES = BM * C_COLS * 2;      // 8 KB per staging buffer
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;

template <int BN>
struct Cfg {
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 192, "BN: multiple of 64, two accumulators in TMEM");
  static constexpr int B_BYTES = BN * BKB;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFA = OFF_C + 2 * C_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
  static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 5;   // full, empty, acc_full x2, acc_empty x2, drain
  static constexpr int OFF_TMEM_PTR = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;    // + slack for 1024-byte alignment
  static constexpr uint32_t SF_COL0 = 2 * BN;
  static constexpr uint32_t SF_SLOTS = (TMEM_COLS - SF_COL0) / SF_SLOT_COLS;
  // Instruction descriptor, kind::mxf4nvf4: A/B E2M1 (format 1), K-major,
  // UE4M3 scales, N >> 3 in bits 17..22, M >> 4 in bits 24..28.
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
  static_assert(SF_SLOTS >= 4, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "smem budget");
};

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

template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                  const __grid_constant__ CUtensorMap tmap_y, const Params p) {
  using C = Cfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t bar_full = sbase + C::OFF_BAR;              // + 8 s
  const uint32_t bar_empty = bar_full + 8 * STAGES;          // + 8 s
  const uint32_t bar_acc_full = bar_empty + 8 * STAGES;      // + 8 b
  const uint32_t bar_acc_empty = bar_acc_full + 16;          // + 8 b
  const uint32_t bar_drain = bar_acc_empty + 16;
  uint32_t* tmem_ptr_smem = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_PTR);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, 4);                   // one arrive per epilogue warp
    }
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
        const uint32_t n0 = nt * BN;
        const uint32_t atom0 = n0 / 128;
        const uint32_t nb_atoms = min((uint32_t)SFB_ATOMS, min(p.n_row_atoms, (n0 + BN - 1) / 128 + 1) - atom0);
        for (uint32_t ks = 0; ks < p.num_k_stages; ++ks) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t natoms = min(4u, p.k_atoms - 4 * ks);
          const uint32_t bytes = A_BYTES + C::B_BYTES + natoms * 512u * (1u + nb_atoms);
          const uint32_t fb = bar_full + 8 * stage;
          mbar_arrive_expect_tx(fb, bytes);
          tma_load_2d(sbase + C::OFF_A + stage * A_BYTES, &tmap_a, fb, (int)(ks * BKB), (int)(mt * BM), pol);
          tma_load_2d(sbase + C::OFF_B + stage * C::B_BYTES, &tmap_b, fb, (int)(ks * BKB), (int)n0, pol);
          bulk_load(sbase + C::OFF_SFA + stage * SFA_BYTES,
                    p.x_scales + ((size_t)mt * p.k_atoms + 4 * ks) * 512u, natoms * 512u, fb);
          for (uint32_t a = 0; a < nb_atoms; ++a)
            bulk_load(sbase + C::OFF_SFB + stage * SFB_BYTES + a * 2048u,
                      p.w_scales + ((size_t)(atom0 + a) * p.k_atoms + 4 * ks) * 512u, natoms * 512u, fb);
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
    // Kept lean: a single thread issues every tcgen05 instruction, so its
    // instruction count per 64-wide K step bounds the tensor-pipe rate.  All
    // descriptors are built once; per stage and step only the start-address
    // field (low word, in 16-byte units) moves.
    const uint64_t adesc0 = smem_desc(sbase + C::OFF_A, 0, 1024, kSwizzle128B);
    const uint64_t bdesc0 = smem_desc(sbase + C::OFF_B, 0, 1024, kSwizzle128B);
    const uint64_t sfadesc0 = smem_desc(sbase + C::OFF_SFA, 0, 128, kSwizzleNone);
    const uint64_t sfbdesc0 = smem_desc(sbase + C::OFF_SFB, 0, 128, kSwizzleNone);
    const uint32_t sf_begin = tmem_base + C::SF_COL0;
    const uint32_t sf_end = sf_begin + C::SF_SLOTS * SF_SLOT_COLS;
    uint32_t sf = sf_begin;                                  // next scale slot (ring)
    uint32_t stage = 0, phase = 0, acc_par = 0;              // acc_par: parity bit per buffer
    uint32_t local = 0;
    bool ok = true;
    for (uint32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
      const uint32_t buf = local & 1u;
      const uint32_t n0 = (tile / p.num_m_tiles) * BN;
      const uint32_t sfb_shift = 4u + (n0 % 128) / 32;       // B scales start 4 columns into a slot
      if (!(ok = warp_mbar_wait(bar_acc_empty + 8 * buf, ((acc_par >> buf) & 1u) ^ 1u))) break;
      acc_par ^= 1u << buf;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + buf * BN;
      for (uint32_t ks = 0; ks < p.num_k_stages; ++ks) {
        if (!(ok = warp_mbar_wait(bar_full + 8 * stage, phase))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t ad = adesc0 + stage * (A_BYTES >> 4);
          const uint64_t bd = bdesc0 + stage * (C::B_BYTES >> 4);
          const uint64_t sad = sfadesc0 + stage * (SFA_BYTES >> 4);
          const uint64_t sbd = sfbdesc0 + stage * (SFB_BYTES >> 4);
          const uint32_t natoms = min(4u, p.k_atoms - 4 * ks);
          // B-scale atoms past the last row tile are not loaded; their slot
          // columns then hold stale values that only reach output columns >= N.
          if (natoms == 4) {
#pragma unroll
            for (uint32_t j = 0; j < 4; ++j) {
              tc_cp_32x128b_warpx4(sf, sad + 32 * j);                  // 512-byte atoms: 32 x 16 B
              tc_cp_32x128b_warpx4(sf + 4, sbd + 32 * j);
              tc_cp_32x128b_warpx4(sf + 8, sbd + 128 + 32 * j);       // second atom, 2048 B further
              tc_mma_nvf4(d_tmem, ad + 2 * j, bd + 2 * j, C::IDESC, sf, sf + sfb_shift, (ks | j) != 0u);
              sf += SF_SLOT_COLS;
              if (sf == sf_end) sf = sf_begin;
            }
          } else {
            for (uint32_t j = 0; j < natoms; ++j) {
              tc_cp_32x128b_warpx4(sf, sad + 32 * j);
              tc_cp_32x128b_warpx4(sf + 4, sbd + 32 * j);
              tc_cp_32x128b_warpx4(sf + 8, sbd + 128 + 32 * j);
              tc_mma_nvf4(d_tmem, ad + 2 * j, bd + 2 * j, C::IDESC, sf, sf + sfb_shift, (ks | j) != 0u);
              sf += SF_SLOT_COLS;
              if (sf == sf_end) sf = sf_begin;
            }
          }
          tc_commit(bar_empty + 8 * stage);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(bar_acc_full + 8 * buf);
      __syncwarp();
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
    uint32_t acc_par = 0;                                    // parity bit per accumulator buffer
    uint32_t chunk_count = 0, local = 0;
    bool dead = false;                                       // a wait ran out: keep the barrier
    for (uint32_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {  // sequence, skip work
      const uint32_t mt = tile % p.num_m_tiles, nt = tile / p.num_m_tiles;
      const uint32_t buf = local & 1u;
      if (!dead && !warp_mbar_wait(bar_acc_full + 8 * buf, (acc_par >> buf) & 1u)) dead = true;
      acc_par ^= 1u << buf;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((q * 32u) << 16) + buf * BN;
      uint32_t v[32];
      if (!dead) tc_ld_32x32b_x32(taddr, v);
#pragma unroll 1
      for (int ch = 0; ch < BN / C_COLS; ++ch) {
        uint32_t packed[16];
        if (!dead) {
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float lo = __uint_as_float(v[2 * i]) * alpha, hi = __uint_as_float(v[2 * i + 1]) * alpha;
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(packed[i]) : "f"(hi), "f"(lo));
          }
          if (ch + 1 < BN / C_COLS) {
            tc_ld_32x32b_x32(taddr + (uint32_t)(ch + 1) * C_COLS, v);   // next chunk in flight
          } else {
            tc_fence_before();                               // all TMEM reads of this tile issued
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_acc_empty + 8 * buf);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) packed[i] = 0u;
        }
        const uint32_t col0 = nt * BN + ch * C_COLS;
        const uint32_t cb = chunk_count & 1u;
        if (issuer) bulk_wait_read<1>();
        named_barrier_sync(1, 128);
        uint8_t* cbuf = smem + C::OFF_C + cb * C_BYTES;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          // 64-byte swizzle: 16-byte chunk i of row r sits at chunk i ^ ((r >> 1) & 3).
          const uint32_t sw = ((uint32_t)i ^ ((row >> 1) & 3u)) * 16u;
          *reinterpret_cast<uint4*>(cbuf + row * 64u + sw) =
              make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
        fence_proxy_async_smem();
        named_barrier_sync(1, 128);
        if (issuer && !dead && col0 < p.N) {
          tma_store_2d(&tmap_y, sbase + C::OFF_C + cb * C_BYTES, (int)col0, (int)(mt * BM));
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
