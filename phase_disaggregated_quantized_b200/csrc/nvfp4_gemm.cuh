// NVFP4 W4A4 block-scaled GEMM on the sm_100a tensor cores (Mix-Quant page,
// gist.science, section 2.3: the prefill worker runs the W4A4 NVFP4 path; the
// page names Blackwell's microscaling FP4 format, section 2).
//
//   Y[m, n] = bf16( t_x t_w sum_k sx[m, k/16] e2m1(cx[m, k]) * sw[n, k/16] e2m1(cw[n, k]) )
//
// Measured on B200: a block-scaled MMA instruction (M = 128, K = 64) takes about
// the same issue time for N = 64 ... 256, a tcgen05.cp of scales placed in the
// MMA thread's stream costs about a third of an MMA, and so does a per-MMA
// handshake with another warp.  So the kernel uses the widest tile (128 x 256
// per MMA) and keeps the MMA thread to waits, MMAs and commits:
//
//   warp 0       TMA producer: per 256-element k-stage, A (128 rows x 128 B) and
//                B (256 rows x 128 B) with 128-byte swizzle, plus the 512-byte
//                scale atoms (A: 4, B: 2 row-atoms x 4) as plain bulk copies.
//   warp 1       MMA issuer: per k-stage one wait for the stage's data and one
//                for its scales in TMEM, four tcgen05.mma.kind::mxf4nvf4
//                .block_scale.block16 (128 x 256 x 64), one commit (it frees the
//                stage's operands and, two stages later, its scale slot).
//   warps 2..9   epilogue, two warps per TMEM sub-partition, each draining one
//                64-column chunk after another (tcgen05.ld), scaling by t_x t_w,
//                rounding to bf16 and TMA-storing its own 32 rows x 64 columns
//                from its own 128-byte-swizzled staging buffer.
//   warps 10..13 scale writers: per k-stage, read the stage's scales from shared
//                memory and write them into a TMEM scale slot with tcgen05.st
//                (each warp its own 32 lanes), then signal the MMA warp once.
//
// TMEM (512 columns): accumulator 0 = [0, 256), accumulator 1 = [128, 384); the
// two overlap in [128, 256).  For each tile the epilogue reads the overlapping
// 128 columns first and releases them before converting anything, so the next
// tile's MMAs (other accumulator) wait only for that read; the rest of the
// drain overlaps them.  [384, 480) holds two 48-column scale slots, one per
// k-stage in flight: k step j uses A scales at columns 4j..4j+3 (column c: rows
// 32c + lane) and B scales at 16 + 8j .. 16 + 8j + 7 (column c: rows 32c + lane),
// the same in all four sub-partitions.
#pragma once
#include "nvfp4_quantize.cuh"
#include "ptx.cuh"

namespace nvq {
namespace w4a4 {

constexpr int BM = 128, BN = 256;
constexpr int BKB = 128;                      // k-stage width in bytes (256 FP4 elements)
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BKB;             // 16 KB
constexpr int B_BYTES = BN * BKB;             // 32 KB
constexpr int SFA_BYTES = 4 * 512;            // 4 k-atoms of the 128 A rows
constexpr int SFB_BYTES = 2 * 4 * 512;        // 2 row-atoms x 4 k-atoms of the 256 B rows
constexpr int EPI_WARPS = 8;
constexpr int C_COLS = 64;                    // epilogue chunk: 64 bf16 = 128-byte rows
constexpr int C_BYTES = 32 * C_COLS * 2;      // 4 KB staging per epilogue warp (32 rows)
constexpr int THREADS = (2 + EPI_WARPS + 4) * 32;   // 14 warps
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC1_COL = 128;            // accumulator 1 starts here (overlaps 0 by 128)
constexpr uint32_t SF_COL0 = 384;
constexpr uint32_t SF_SLOT_COLS = 48;         // one k-stage: 4 x (4 A + 8 B) columns
constexpr uint32_t SF_SLOTS = 2;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
constexpr int OFF_SFA = OFF_C + EPI_WARPS * C_BYTES;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
// full[S], empty[S], acc_full[2], acc_empty[2], overlap_free, sf_full[2], drain, scales_in[S]
constexpr int NUM_BARS = 2 * STAGES + 2 + 2 + 1 + SF_SLOTS + 1 + STAGES;
constexpr int OFF_TMEM_PTR = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;    // + slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "smem budget");
static_assert(SF_COL0 + SF_SLOTS * SF_SLOT_COLS <= TMEM_COLS && ACC1_COL + BN <= SF_COL0, "TMEM budget");

// Instruction descriptor, kind::mxf4nvf4: A/B E2M1 (format 1), K-major,
// UE4M3 scales, N >> 3 in bits 17..22, M >> 4 in bits 24..28.
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
  uint32_t m_fastest;      // 1: tile index runs over row blocks first (A re-read per wave)
  // SiLU * mul epilogue only (B rows interleaved in blocks of 128: gate, up, gate, up, ...)
  uint8_t* h_codes;        // [M, N/2 / 2] E2M1 codes of H = silu(gate) * up
  uint8_t* h_scales;       // tiled E4M3 scales of H, padded rows zero
  const float* t_h;        // static tensor scale of H
  uint32_t h_katoms;       // (N / 2) / 64
};

// Tile order: the tiles in flight at once (one per SM) cover a band of tiles
// that re-reads one operand every wave.  The host picks the smaller operand for
// that role (A_fastest: row blocks fastest, all of A swept per wave), so the
// swept operand stays in L2 next to the output stream and each byte of the
// other operand is read from HBM once.
__device__ __forceinline__ void tile_coords(uint32_t tile, const Params& p, uint32_t& mt, uint32_t& nt) {
  if (p.m_fastest) {
    mt = tile % p.num_m_tiles;
    nt = tile / p.num_m_tiles;
  } else {
    nt = tile % p.num_n_tiles;
    mt = tile / p.num_n_tiles;
  }
}

// ---------------------------------------------------------------- SiLU * mul -> NVFP4 epilogue
// Per-CTA tables for the static tensor scale t_h of H, one entry per E4M3 block
// scale code S: the multiplier of the fast map (1 / fl(S t_h), or that value
// moved by 2^-20 relative, as for the activations), whether the fast map (fp32
// product + cvt) gives the exact RTN code for every fp32 input, and 6 x the
// midpoint to the next code.
struct HTables {
  float inv_d[128];
  uint32_t fast_ok[128];
  float mid6[128];
};

__device__ __forceinline__ uint32_t e2m1_code_f32(float x, float inv_d) {   // x >= 0
  return e2m1x2_rn_satfinite(0.f, __fmul_rn(x, inv_d)) & 0xFu;
}

// Built by 127 threads.  The fast map is monotone in x, so it is exact for all
// fp32 inputs once it is exact at the last fp32 below and the first fp32 at or
// above every exact threshold mu_i S t (located with h = fl(P t) and the exact
// residual fma(P, t, -h), P = mu_i S exact).
__device__ __forceinline__ void build_h_table(HTables& tb, uint32_t c, float t) {
  const float S = e4m3_value(c);
  const float d = __fmul_rn(S, t);
  const float inv0 = (c == 0) ? 0.f : __frcp_rn(d);
  float inv = inv0;
  bool ok = (c == 0) || (d >= 1.17549435e-38f && !isinf(inv0));
  auto exact_with = [&](float r) {
    bool g = true;
    for (int i = 0; i < 7 && g; ++i) {
      const float P = __fmul_rn(c_e2m1_mid[i], S);
      const float h = __fmul_rn(P, t);
      const float e = __fmaf_rn(P, t, -h);
      if (isinf(h)) {
        g = e2m1_code_f32(3.40282347e38f, r) == (uint32_t)i;
        continue;
      }
      const bool pass_h = e < 0.f || (e == 0.f && ((i + 1) & 1) == 0);   // h above the threshold, or on a tie that goes up
      const uint32_t hb = __float_as_uint(h);
      const float x1 = pass_h ? h : __uint_as_float(hb + 1u);
      if (e2m1_code_f32(x1, r) != (uint32_t)(i + 1)) g = false;
      if (hb != 0u || !pass_h) {
        const float x0 = pass_h ? __uint_as_float(hb - 1u) : h;
        if (e2m1_code_f32(x0, r) != (uint32_t)i) g = false;
      }
    }
    return g;
  };
  if (c != 0 && ok) {                 // the multiplier candidates of the activation quantizer
    const float cand[3] = {inv0, __fmul_rn(inv0, kNudgeDown), __fmul_rn(inv0, kNudgeUp)};
    ok = false;
    for (int j = 0; j < 3 && !ok; ++j)
      if (!isinf(cand[j]) && exact_with(cand[j])) {
        ok = true;
        inv = cand[j];
      }
  }
  tb.inv_d[c] = inv;
  tb.fast_ok[c] = ok ? 1u : 0u;
  tb.mid6[c] = c < 126 ? __fmul_rn(6.0f, 0.5f * (S + e4m3_value(c + 1))) : 0.f;
}

// 16 fp32 values of one block -> 8 bytes of codes (even k in the low nibble)
// and its E4M3 scale code.
__device__ __forceinline__ uint32_t quantize_block16(const float (&v)[16], float t, float inv6t, const HTables& tb,
                                                     uint2& out) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t s = block_scale_code(amax, t, inv6t, tb.mid6);
  uint32_t w[2] = {0u, 0u};
  if (__all_sync(0xFFFFFFFFu, tb.fast_ok[s] != 0u)) {        // warp-uniform: no warp runs both paths
    const float inv = tb.inv_d[s];
#pragma unroll
    for (int i = 0; i < 8; ++i) {                          // signed product: the sign lands on the code
      const uint32_t byte = e2m1x2_rn_satfinite(__fmul_rn(v[2 * i + 1], inv), __fmul_rn(v[2 * i], inv));
      w[i >> 2] |= byte << (8 * (i & 3));
    }
  } else {
    const float S = e4m3_value(s);
#pragma unroll
    for (int i = 0; i < 16; ++i) {                         // unrolled: v stays in registers
      const float ax = fabsf(v[i]);
      uint32_t mag = 0;
      if (s != 0) {
#pragma unroll
        for (int j = 0; j < 7; ++j) {
          const float r = __fmaf_rn(-__fmul_rn(c_e2m1_mid[j], S), t, ax);   // exact sign
          mag += (r > 0.f || (r == 0.f && ((j + 1) & 1) == 0)) ? 1u : 0u;
        }
      }
      const uint32_t code = mag | ((__float_as_uint(v[i]) >> 28) & 8u);
      w[i >> 3] |= code << (4 * (i & 7));
    }
  }
  out = make_uint2(w[0], w[1]);
  return s;
}

// silu(g) * u in fp32.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ uint32_t acc_col(uint32_t buf) { return buf ? ACC1_COL : 0u; }

// EPI 0: Y = BF16(alpha acc).  EPI 1: B rows interleaved in blocks of 128 (gate,
// up, gate, up, ...); H = silu(gate) * up quantized to NVFP4 with a static t_h.
template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                  const __grid_constant__ CUtensorMap tmap_y, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t bar_full = sbase + OFF_BAR;                  // + 8 s
  const uint32_t bar_empty = bar_full + 8 * STAGES;           // + 8 s
  const uint32_t bar_acc_full = bar_empty + 8 * STAGES;       // + 8 b
  const uint32_t bar_acc_empty = bar_acc_full + 16;           // + 8 b
  const uint32_t bar_overlap = bar_acc_empty + 16;
  const uint32_t bar_sf_full = bar_overlap + 8;               // + 8 slot
  const uint32_t bar_drain = bar_sf_full + 8 * SF_SLOTS;
  const uint32_t bar_sc_in = bar_drain + 8;                   // + 8 s: the stage's scale atoms landed
  uint32_t* tmem_ptr_smem = reinterpret_cast<uint32_t*>(smem + OFF_TMEM_PTR);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
      mbar_init(bar_sc_in + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, EPI_WARPS);            // one arrive per epilogue warp
    }
    mbar_init(bar_overlap, EPI_WARPS);
    for (uint32_t k = 0; k < SF_SLOTS; ++k) {
      mbar_init(bar_sf_full + 8 * k, 4);                      // one arrive per scale-writer warp
    }
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tensormap(&tmap_a);
    prefetch_tensormap(&tmap_b);
    if (EPI == 0) prefetch_tensormap(&tmap_y);
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
      uint32_t pending = 0, pending_parity = 0;               // per-stage bit masks
      bool ok = true;
      for (uint32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        uint32_t mt, nt;
        tile_coords(tile, p, mt, nt);
        const uint32_t nb_atoms = min(2u, p.n_row_atoms - 2 * nt);
        for (uint32_t ks = 0; ks < p.num_k_stages; ++ks) {
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1)) { ok = false; break; }
          const uint32_t natoms = min(4u, p.k_atoms - 4 * ks);
          // The scale atoms complete on a barrier of their own and go first, so
          // the scale writers can move them into TMEM while the operands land.
          const uint32_t sb = bar_sc_in + 8 * stage;
          mbar_arrive_expect_tx(sb, natoms * 512u * (1u + nb_atoms));
          bulk_load(sbase + OFF_SFA + stage * SFA_BYTES,
                    p.x_scales + ((size_t)mt * p.k_atoms + 4 * ks) * 512u, natoms * 512u, sb);
          for (uint32_t a = 0; a < nb_atoms; ++a)
            bulk_load(sbase + OFF_SFB + stage * SFB_BYTES + a * 2048u,
                      p.w_scales + ((size_t)(2 * nt + a) * p.k_atoms + 4 * ks) * 512u, natoms * 512u, sb);
          const uint32_t fb = bar_full + 8 * stage;
          mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
          tma_load_2d(sbase + OFF_A + stage * A_BYTES, &tmap_a, fb, (int)(ks * BKB), (int)(mt * BM), pol);
          tma_load_2d(sbase + OFF_B + stage * B_BYTES, &tmap_b, fb, (int)(ks * BKB), (int)(nt * BN), pol);
          pending |= 1u << stage;
          pending_parity = (pending_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // Let every copy issued into shared memory land before the CTA exits.
      for (int s2 = 0; s2 < STAGES; ++s2)
        if (pending & (1u << s2)) {
          mbar_wait_drain(bar_sc_in + 8 * s2, (pending_parity >> s2) & 1u, 200000000ull);
          mbar_wait_drain(bar_full + 8 * s2, (pending_parity >> s2) & 1u, 200000000ull);
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t adesc0 = smem_desc(sbase + OFF_A, 0, 1024, kSwizzle128B);
    const uint64_t bdesc0 = smem_desc(sbase + OFF_B, 0, 1024, kSwizzle128B);
    uint32_t stage = 0, phase = 0, acc_par = 0, local = 0;
    uint32_t slot = 0, slot_phase = 0;
    bool ok = true;
    for (uint32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
      const uint32_t buf = local & 1u;
      // This accumulator was drained (tile - 2), and the columns it shares with
      // the other accumulator were read for the previous tile.
      if (!(ok = warp_mbar_wait(bar_acc_empty + 8 * buf, ((acc_par >> buf) & 1u) ^ 1u))) break;
      acc_par ^= 1u << buf;
      if (local > 0 && !(ok = warp_mbar_wait(bar_overlap, (local - 1) & 1u))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc_col(buf);
      for (uint32_t ks = 0; ks < p.num_k_stages; ++ks) {
        if (!(ok = warp_mbar_wait(bar_full + 8 * stage, phase))) break;
        if (!(ok = warp_mbar_wait(bar_sf_full + 8 * slot, slot_phase))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t ad = adesc0 + stage * (A_BYTES >> 4);
          const uint64_t bd = bdesc0 + stage * (B_BYTES >> 4);
          const uint32_t sf = tmem_base + SF_COL0 + SF_SLOT_COLS * slot;
          const uint32_t natoms = min(4u, p.k_atoms - 4 * ks);
          for (uint32_t j = 0; j < natoms; ++j)     // 32 bytes (64 FP4 elements) per k step
            tc_mma_nvf4(d_tmem, ad + 2 * j, bd + 2 * j, IDESC, sf + 4 * j, sf + 16 + 8 * j, (ks | j) != 0u);
          tc_commit(bar_empty + 8 * stage);                    // also frees this stage's scale slot
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
        if (++slot == SF_SLOTS) { slot = 0; slot_phase ^= 1; }
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
  } else if (warp >= 2 + EPI_WARPS) {
    // ------------------------------------------------------------ scale writers
    const uint32_t q = warp & 3u;                             // TMEM sub-partition of this warp
    const uint32_t lane_base = (q * 32u) << 16;
    uint32_t stage = 0, phase = 0, slot = 0;
    // A scale slot is free once the MMAs of the k-stage that used it (SF_SLOTS
    // k-stages back) have completed, i.e. once that stage's empty barrier has
    // fired: one commit per k-stage serves the TMA producer and these warps
    // (so the MMA thread commits once per k-stage, for both).
    uint32_t lag_stage = 0, lag_phase = 0, kg = 0;
    bool ok = true;
    for (uint32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (uint32_t ks = 0; ks < p.num_k_stages; ++ks, ++kg) {
        if (kg >= SF_SLOTS) {
          if (!(ok = warp_mbar_wait(bar_empty + 8 * lag_stage, lag_phase))) break;
          if (++lag_stage == STAGES) { lag_stage = 0; lag_phase ^= 1; }
        }
        if (!(ok = warp_mbar_wait(bar_sc_in + 8 * stage, phase))) break;   // this stage's scale atoms
        tc_fence_after();
        const uint8_t* sfa = smem + OFF_SFA + stage * SFA_BYTES + 16 * lane;
        const uint8_t* sfb = smem + OFF_SFB + stage * SFB_BYTES + 16 * lane;
        const uint32_t col = lane_base + tmem_base + SF_COL0 + SF_SLOT_COLS * slot;
        const uint32_t natoms = min(4u, p.k_atoms - 4 * ks);
        // Atom row `lane` holds rows lane, lane+32, lane+64, lane+96 (4 bytes each);
        // column c gets rows 32c + lane, as tcgen05.cp .32x128b.warpx4 would place them.
        if (natoms == 4u) {                   // whole stage: two wide TMEM stores
          uint32_t aw[16], bw[32];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 a = *reinterpret_cast<const uint4*>(sfa + 512 * j);
            const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + 512 * j);
            const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + 2048 + 512 * j);
            aw[4 * j] = a.x; aw[4 * j + 1] = a.y; aw[4 * j + 2] = a.z; aw[4 * j + 3] = a.w;
            bw[8 * j] = b0.x; bw[8 * j + 1] = b0.y; bw[8 * j + 2] = b0.z; bw[8 * j + 3] = b0.w;
            bw[8 * j + 4] = b1.x; bw[8 * j + 5] = b1.y; bw[8 * j + 6] = b1.z; bw[8 * j + 7] = b1.w;
          }
          tc_st_32x32b_x16(col, aw);
          tc_st_32x32b_x32(col + 16, bw);
        } else {
          for (uint32_t j = 0; j < natoms; ++j) {
            const uint4 a = *reinterpret_cast<const uint4*>(sfa + 512 * j);
            const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + 512 * j);
            const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + 2048 + 512 * j);
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
            const uint32_t bw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            tc_st_32x32b_x4(col + 4 * j, aw);
            tc_st_32x32b_x8(col + 16 + 8 * j, bw);
          }
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sf_full + 8 * slot);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
        if (++slot == SF_SLOTS) slot = 0;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3u;                             // TMEM sub-partition of this warp
    const uint32_t h = (warp - 2) >> 2;                       // which 64-column chunk of each pair
    const uint32_t row = q * 32 + lane;                       // row of the tile held by this thread
    const float alpha = __ldg(p.t_x) * __ldg(p.t_w);
    if constexpr (EPI == 0) {
    uint8_t* cbuf = smem + OFF_C + (warp - 2) * C_BYTES;      // this warp's 32 x 128 B staging
    const uint32_t cbuf_s = smem_addr(cbuf);
    uint32_t acc_par = 0, local = 0;
    bool dead = false;                                        // a wait ran out: skip work
    for (uint32_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      uint32_t mt, nt;
      tile_coords(tile, p, mt, nt);
      const uint32_t buf = local & 1u;
      if (!dead && !warp_mbar_wait(bar_acc_full + 8 * buf, (acc_par >> buf) & 1u)) dead = true;
      acc_par ^= 1u << buf;
      if (dead) continue;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((q * 32u) << 16) + acc_col(buf);
      // Chunk (64 columns) in the region shared with the other accumulator first:
      // chunks 2, 3 of accumulator 0 and 0, 1 of accumulator 1.
      const uint32_t ch_first = (buf ? 0u : 2u) + h, ch_second = (buf ? 2u : 0u) + h;
      uint32_t v[64];
      tc_ld_32x32b_x64(taddr + ch_first * C_COLS, v);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_overlap);
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        const uint32_t ch = part ? ch_second : ch_first;
        uint32_t packed[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float lo = __uint_as_float(v[2 * e]) * alpha, hi = __uint_as_float(v[2 * e + 1]) * alpha;
          asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(packed[e]) : "f"(hi), "f"(lo));
        }
        if (part == 0) tc_ld_32x32b_x64(taddr + ch_second * C_COLS, v);   // in flight during the store
        if (lane == 0) bulk_wait_read<0>();                     // previous store done reading staging
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          // 128-byte swizzle: 16-byte chunk e of row r sits at chunk e ^ (r & 7).
          const uint32_t sw = ((uint32_t)e ^ (lane & 7u)) * 16u;
          *reinterpret_cast<uint4*>(cbuf + lane * 128u + sw) =
              make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        const uint32_t col0 = nt * BN + ch * C_COLS;
        if (lane == 0 && col0 < p.N) {
          tma_store_2d(&tmap_y, cbuf_s, (int)col0, (int)(mt * BM + q * 32));
          bulk_commit();
        }
        if (part == 0) {
          tc_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_acc_empty + 8 * buf);   // all of this tile's TMEM read
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
    (void)row;
    } else {
      // SiLU * mul -> NVFP4.  Tile columns [0, 128) are gate rows of B, [128, 256)
      // the matching up rows; this warp owns H columns 64 h .. 64 h + 63 of the
      // tile (its gate chunk h and up chunk 2 + h) for rows 32 q .. 32 q + 31.
      HTables& tb = *reinterpret_cast<HTables*>(smem + OFF_C);   // staging unused here
      const float t_h = __ldg(p.t_h);
      const uint32_t etid = threadIdx.x - 64u;                  // 0 .. 255 over the epilogue warps
      if (etid < 127u) build_h_table(tb, etid, t_h);
      named_barrier_sync(1, EPI_WARPS * 32);
      const float inv6t = __frcp_rn(__fmul_rn(6.0f, t_h));
      const uint32_t hrow_bytes = p.N >> 2;                     // (N / 2) codes, two per byte
      uint32_t acc_par = 0, local = 0;
      bool dead = false;
      for (uint32_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
        uint32_t mt, nt;
        tile_coords(tile, p, mt, nt);
        const uint32_t buf = local & 1u;
        if (!dead && !warp_mbar_wait(bar_acc_full + 8 * buf, (acc_par >> buf) & 1u)) dead = true;
        acc_par ^= 1u << buf;
        if (dead) continue;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((q * 32u) << 16) + acc_col(buf);
        // The chunk in the region shared with the other accumulator first (up
        // for accumulator 0, gate for accumulator 1), then the other in halves.
        const uint32_t ch_first = (buf ? 0u : 2u) + h, ch_second = (buf ? 2u : 0u) + h;
        uint32_t vf[64];
        tc_ld_32x32b_x64(taddr + ch_first * C_COLS, vf);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_overlap);
        const uint32_t grow = mt * BM + row;
        uint32_t sword = 0;
#pragma unroll
        for (int part = 0; part < 2; ++part) {              // unrolled: vf is indexed at compile time
          uint32_t vs[32];
          tc_ld_32x32b_x32(taddr + ch_second * C_COLS + 32u * part, vs);
          tc_wait_ld();
          if (part == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_acc_empty + 8 * buf);   // all of this tile's TMEM read
          }
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float hv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float a = __uint_as_float(vf[32 * part + 16 * b + i]) * alpha;
              const float c2 = __uint_as_float(vs[16 * b + i]) * alpha;
              hv[i] = buf ? silu_mul(a, c2) : silu_mul(c2, a);
            }
            uint2 codes;
            const uint32_t sc = quantize_block16(hv, t_h, inv6t, tb, codes);
            sword |= sc << (8 * (2 * part + b));
            const uint32_t col = nt * 128u + h * 64u + 32u * part + 16u * b;   // H column of the block
            if (grow < p.M) *reinterpret_cast<uint2*>(p.h_codes + (size_t)grow * hrow_bytes + (col >> 1)) = codes;
          }
        }
        // The row's four scale bytes of blocks kb .. kb + 3: one aligned word of its atom.
        const uint32_t kb = (nt * 128u + h * 64u) >> 4;
        const size_t off = ((size_t)(grow >> 7) * p.h_katoms + (kb >> 2)) * 512u + (grow & 31u) * 16u +
                           ((grow & 127u) >> 5) * 4u;
        *reinterpret_cast<uint32_t*>(p.h_scales + off) = sword;
      }
    }
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
