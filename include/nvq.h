/*
 * nvq.h -- C ABI of the phase-specialised quantized linear layers for B200 (sm_100a).
 *
 * Prefill: NVFP4 W4A4.  Activations and weights are quantized to NVFP4 by
 * round-to-nearest: E2M1 4-bit codes in 16-element blocks along K, one E4M3
 * scale per block and one FP32 scale per tensor (Mix-Quant page, gist.science,
 * section 2 "hybrid precision strategy"; section 2.3: the prefill worker runs
 * the NVFP4 W4A4 path).  The quantized operands feed a block-scaled GEMM on the
 * tcgen05 tensor cores.
 *
 * Decode: W4A16.  BF16 activations at small batch multiply INT4 weights that
 * carry one BF16 scale per group of 128 weights; the weights are reordered
 * offline into the kernel's fragment order (MARLIN page, abeam.tech, sections
 * "weight layout" and "overlapping memory and compute").
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory and frees nothing.  Outputs are written in place.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream; no call synchronises the host
 *     except nvq_check_device_error().
 *   - Matrices are row-major.  BF16 is IEEE bfloat16 stored as 16-bit words.
 *   - Packed 4-bit codes: two per byte, the even-k element in the low nibble.
 *   - The return value reports host-side validation and launch errors
 *     (cudaGetLastError after launch).  Errors found on the device (a bounded
 *     wait that ran out) set a library-wide device error word that
 *     nvq_check_device_error() reads and clears.  No kernel traps.
 *   - Pointers must be 16-byte aligned (NVQ_ERR_MISALIGNED otherwise).
 *   - Size limits common to all calls (NVQ_ERR_UNSUPPORTED_SHAPE beyond them):
 *     every dimension < 2^31; a quantize call holds < 2^31 16-element blocks
 *     (rows * K / 16); a GEMM has < 2^31 128 x 128 output blocks.
 */
#ifndef NVQ_H_
#define NVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVQ_OK = 0,
  NVQ_ERR_INVALID_ARG = 1,        /* null pointer, negative size */
  NVQ_ERR_UNSUPPORTED_SHAPE = 2,  /* shape outside the documented rules */
  NVQ_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
  NVQ_ERR_WORKSPACE = 4,          /* workspace missing or too small */
  NVQ_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
  NVQ_ERR_DEVICE_TIMEOUT = 6      /* a kernel's bounded wait ran out */
} nvq_status;

/* Version of this ABI; bumped on any incompatible change. */
int nvq_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* nvq_status_string(nvq_status s);

/* Text describing the last failed call on this host thread (argument or CUDA
 * error), or "" if none; owned by the library, valid until the next call. */
const char* nvq_last_error_detail(void);

/* Workspace bytes of one call, by operation (the per-operation *_workspace_bytes
 * functions give the same numbers): NVQ_OP_NVFP4_QUANTIZE (rows = M, K; also
 * nvfp4_amax), NVQ_OP_NVFP4_GEMM (0: none), NVQ_OP_W4A16_GEMM (0: partial sums
 * stay on chip), NVQ_OP_LINEAR (nvq_linear at the default crossover).
 * SIZE_MAX for an unknown op. */
typedef enum {
  NVQ_OP_NVFP4_QUANTIZE = 0,
  NVQ_OP_NVFP4_GEMM = 1,
  NVQ_OP_W4A16_GEMM = 2,
  NVQ_OP_LINEAR = 3
} nvq_op;
size_t nvq_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns NVQ_ERR_DEVICE_TIMEOUT if any kernel since the last check gave up on
 * a bounded wait, NVQ_ERR_CUDA if the synchronisation failed, else NVQ_OK.
 * The error word is one per device and per loaded library, shared by every
 * stream and every caller on that device: a timeout in a kernel on one stream
 * is reported to whichever caller checks first (on any stream), and that
 * check clears it for everyone.  Kernels still running on other streams are
 * not waited for; a timeout they raise later is seen by a later check. */
nvq_status nvq_check_device_error(void* stream);

/* Diagnostic of the timeout path: launches one thread on `stream` that waits,
 * with the bounded wait every pipeline of this library uses, on an mbarrier
 * that nothing ever completes.  After limit_ns of device time (1 us .. 100 ms,
 * else NVQ_ERR_INVALID_ARG and nothing is launched) the wait gives up, raises
 * the device error word and the kernel returns normally: no trap, no hang, the
 * context stays usable.  The next nvq_check_device_error() then returns
 * NVQ_ERR_DEVICE_TIMEOUT and clears the word.  Run it only while no other
 * kernel of this library is in flight: a kernel that is waiting while the word
 * is raised gives up too. */
nvq_status nvq_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* ------------------------------------------------------------------------ *
 * NVFP4 round-to-nearest quantization (Mix-Quant page, section 2: 16-element
 * groups with a local scale plus a tensor-level scale, plain RTN).
 *
 *   t   = *tensor_scale_in if tensor_scale_in != NULL, else
 *         1.0f if max|x| == 0, else fp32_RNE(max|x| / 2688)   (2688 = 6 * 448)
 *   s_b = E4M3_RNE_satfinite(amax_b / (6 t))   for each 16-element block b
 *   c   = sign(x) | E2M1_RNE_satfinite(|x| / (e4m3(s_b) t)), ties to the even
 *         code; a block with s_b == 0 stores magnitude 0 (sign kept)
 * Every rounding is decided on the exact real quotient (the same result as
 * infinitely precise division followed by one rounding).
 *
 * x_bf16            [rows, K] BF16, row stride K elements.  Inputs are finite;
 *                   non-finite values are outside the contract.
 * rows              >= 0 (0 is a no-op that still writes tensor_scale_out = 1
 *                   when tensor_scale_in == NULL).
 * K                 > 0, K % 64 == 0.
 * tensor_scale_in   NULL, or a device pointer to a caller-fixed positive finite
 *                   FP32 t (a static activation scale).
 * codes             [rows, K/2] bytes, written.
 * scales            nvfp4_scales_bytes(rows, K) bytes, written in the tiled
 *                   layout that the block-scaled MMA reads: 512-byte atoms of
 *                   128 rows x 4 blocks, row r / block c of an atom at byte
 *                   16*(r%32) + 4*((r%128)/32) + c, atoms K-fastest
 *                   (atom index = (r/128)*(K/64) + kb/4).  Padding rows (rows
 *                   up to the next multiple of 128) get zero scales.
 * tensor_scale_out  device pointer, receives t (may alias tensor_scale_in).
 * workspace         device scratch of nvfp4_quantize_workspace_bytes(rows, K)
 *                   bytes (may be NULL when that is 0).
 * ------------------------------------------------------------------------ */
size_t nvfp4_scales_bytes(int64_t rows, int64_t K);
/* Host-side map of the tiled scale layout: byte offset, inside the scales
 * buffer of a [rows, K] tensor, of the E4M3 scale of row `row`, 16-element
 * block `kblock`; -1 if an argument is out of range.  The layout is 512-byte
 * atoms of 128 rows x 4 blocks, row-tile major, each atom the 32 x 16-byte
 * matrix the block-scaled tensor-core MMA takes its scales from. */
int64_t nvfp4_scale_offset(int64_t row, int64_t kblock, int64_t rows, int64_t K);
size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t K);
nvq_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t K,
                          const float* tensor_scale_in, uint8_t* codes, uint8_t* scales,
                          float* tensor_scale_out, void* workspace, size_t workspace_bytes,
                          void* stream);

/* ------------------------------------------------------------------------ *
 * One tensor's rows split over several processes (an M split of a prefill
 * linear): the tensor-level scale of the Mix-Quant page, section 2, must come
 * from the max |x| of the whole tensor, so each rank
 *   1. nvfp4_amax            its rows' max |x| -> *amax_out (FP32, exact;
 *                            0 for rows == 0);
 *   2. all-reduces that FP32 value with MAX over the ranks (4 bytes);
 *   3. nvfp4_scale_from_amax the combined value -> t, the same t that
 *                            nvfp4_quantize computes for a tensor with that
 *                            amax (1 if it is 0, else fp32_RNE(amax / 2688));
 *   4. nvfp4_quantize        its rows with tensor_scale_in = that t.
 * Every rank then holds exactly the codes and scales that one nvfp4_quantize
 * call over the whole tensor would give for its rows (scales compared in the
 * logical [rows, K/16] order; they tile identically when each shard starts on a
 * multiple of 128 rows).
 * nvfp4_amax: x_bf16, rows, K as for nvfp4_quantize; amax_out a 4-byte aligned
 * device float; workspace of nvfp4_quantize_workspace_bytes(rows, K) bytes
 * (may be NULL when rows == 0).  nvfp4_scale_from_amax: two 4-byte aligned
 * device floats (may alias).  Both asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
nvq_status nvfp4_amax(const void* x_bf16, int64_t rows, int64_t K, float* amax_out, void* workspace,
                      size_t workspace_bytes, void* stream);
nvq_status nvfp4_scale_from_amax(const float* amax, float* tensor_scale_out, void* stream);

/* ------------------------------------------------------------------------ *
 * nvfp4_quantize without any device allocation or workspace (no counterpart
 * on the pages; an addition of this library).  For callers that cannot call
 * cudaMalloc or lend scratch memory: for example an engine whose device memory
 * is all owned by its own pool once serving starts, or a plugin that must not
 * allocate behind its host's back.  Same arguments, same results (bit for bit)
 * as nvfp4_quantize, minus the workspace.
 *
 * The tensor-amax partials live in a fixed 4 KiB file-scope device array
 * inside the library (1024 floats; the amax pre-pass uses the same grid as
 * nvfp4_quantize, at most 592 partials), held on every GPU that loads the
 * library until the process exits.  Limit: rows * K <= 2^30 elements; larger
 * calls return NVQ_ERR_UNSUPPORTED_SHAPE before any pointer is examined.
 * The first call on each device resolves the array's device address with
 * cudaGetSymbolAddress (that device must be current) and caches it for the
 * life of the process; make that first call before any stream capture.  The
 * cached address does not survive cudaDeviceReset() or a reset of the primary
 * context: do not call this entry point after either.  All calls on a device
 * share the array: calls that overlap on the GPU (different streams, no
 * ordering) race and give wrong results.  Each call overwrites every partial
 * it later reads, so nothing needs clearing between calls.  Calls no
 * cudaMalloc/cudaFree.
 * ------------------------------------------------------------------------ */
nvq_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t K,
                                  const float* tensor_scale_in, uint8_t* codes, uint8_t* scales,
                                  float* tensor_scale_out, void* stream);

/* ------------------------------------------------------------------------ *
 * NVFP4 W4A4 GEMM (Mix-Quant page, section 2.3: the prefill worker's W4A4 path).
 *
 *   Y[m, n] = bf16_RNE( t_x * t_w * sum_k (e4m3(sx[m, k/16]) e2m1(cx[m, k]))
 *                                        * (e4m3(sw[n, k/16]) e2m1(cw[n, k])) )
 * accumulated in FP32 on the tensor cores (tcgen05 block-scaled MMA, TMEM
 * accumulators).  Operands are the outputs of nvfp4_quantize: X [M, K] and
 * W [N, K] (nn.Linear layout), so Y = X W^T.
 *
 * x_codes [M, K/2], x_scales (tiled, nvfp4_scales_bytes(M, K)), t_x (device FP32)
 * w_codes [N, K/2], w_scales (tiled, nvfp4_scales_bytes(N, K)), t_w (device FP32)
 * y_bf16  [M, N] BF16, row stride N, written.
 * Shape rules: M >= 0, N >= 8, N % 8 == 0, K >= 64, K % 64 == 0.
 * ------------------------------------------------------------------------ */
nvq_status nvfp4_gemm_w4a4(const uint8_t* x_codes, const uint8_t* x_scales, const float* t_x,
                           const uint8_t* w_codes, const uint8_t* w_scales, const float* t_w,
                           void* y_bf16, int64_t M, int64_t N, int64_t K, void* stream);

/* ------------------------------------------------------------------------ *
 * gate_up W4A4 GEMM whose epilogue applies SiLU * mul and writes NVFP4 for the
 * down projection (Mix-Quant page, gist.science, section 2: NVFP4 activations
 * with 16-element E4M3 scales and a tensor scale for the prefill linears; the
 * Qwen3 gated MLP feeds down_proj with silu(x Wg^T) * (x Wu^T)).  The BF16
 * [M, N] gate_up output never reaches memory.
 *
 *   G, U  = t_x t_w sum (NVFP4 products), FP32, as nvfp4_gemm_w4a4 computes Y
 *   H     = silu(G) * U in FP32, silu(g) = g / (1 + exp(-g)) (relative error
 *           about 1e-6 from the fast exponential and division)
 *   codes, scales = NVFP4 RTN of H with the caller's static tensor scale *t_h
 *           (the epilogue cannot see max|H| over the tensor before it writes),
 *           the same exact rounding rules as nvfp4_quantize.
 *
 * w_codes / w_scales / t_w: nvfp4_quantize of the gate_up weight with its rows
 * interleaved in blocks of 128: rows 256 b .. 256 b + 127 are gate rows
 * 128 b .. 128 b + 127, the next 128 rows the same up rows (I = N / 2 gate and
 * up rows each).  h_codes [M, I/2] bytes (even column in the low nibble);
 * h_scales nvfp4_scales_bytes(M, I) bytes, tiled as nvfp4_quantize writes them
 * (padding rows zero): the input nvfp4_gemm_w4a4 takes for down_proj, with
 * t_x = *t_h.  Shape rules: N % 256 == 0, K % 64 == 0.
 * ------------------------------------------------------------------------ */
nvq_status nvfp4_gemm_w4a4_swiglu(const uint8_t* x_codes, const uint8_t* x_scales, const float* t_x,
                                  const uint8_t* w_codes, const uint8_t* w_scales, const float* t_w,
                                  const float* t_h, uint8_t* h_codes, uint8_t* h_scales, int64_t M, int64_t N,
                                  int64_t K, void* stream);

/* ------------------------------------------------------------------------ *
 * INT4 group-128 round-to-nearest weight quantization (MARLIN page: 4-bit
 * weights with one scale per 128-weight group).
 *
 *   s[n, g] = bf16_RNE(amax(w[n, 128g : 128g+128]) / 7)
 *   q       = clamp(RNE_half_even(w / s), -8, 7)   (0 when s == 0)
 *   u       = q + 8, stored as nibbles, even k in the low nibble
 * w_bf16 [N, K]; codes [N, K/2] bytes; scales_bf16 [N, K/128] BF16.
 * Shape rules: N >= 0, K > 0, K % 128 == 0.
 * ------------------------------------------------------------------------ */
nvq_status int4_quantize(const void* w_bf16, int64_t N, int64_t K, uint8_t* codes,
                         void* scales_bf16, void* stream);

/* ------------------------------------------------------------------------ *
 * Offline reorder of INT4 codes and group scales into the decode kernel's
 * fragment order (MARLIN page, abeam.tech, the section on the offline weight
 * reorder: codes and scales are permuted ahead of time so each thread's loads
 * are regular and dequantize straight into tensor-core fragment order).  A
 * bijection: no byte is added or lost.
 *
 * Unit = 32 weight rows x one 128-wide group: 2048 code bytes at unit index
 * (n/32)*(K/128) + k/128; its rows are two 16-row tensor-core tiles tt = 0, 1.
 * Inside a unit, 32-bit word 128q + 4lane + comp (q in [0,4), lane = 4g + c in
 * [0,32), comp in [0,4)) holds k16-step j = 2q + comp/2 of tile tt = comp%2,
 * with nibble p (bits 4p..4p+3) at (row in tile, k-in-group); K is permuted
 * inside the group so that lane (g, c) covers k = 32c .. 32c+31:
 *   p=0 (g, 32c+4j)   p=4 (g, 32c+4j+1)   p=1 (g+8, 32c+4j)   p=5 (g+8, 32c+4j+1)
 *   p=2 (g, 32c+4j+2) p=6 (g, 32c+4j+3)   p=3 (g+8, 32c+4j+2) p=7 (g+8, 32c+4j+3)
 * Scales: 64 bytes per unit; 32-bit word 2g + tt holds rows 16tt + g (low half)
 * and 16tt + g + 8 (high half).
 *
 * codes [N, K/2] (as written by int4_quantize), scales_bf16 [N, K/128]
 * packed_codes N*K/2 bytes, packed_scales N*(K/128)*2 bytes, written.
 * Shape rules: N % 32 == 0, K % 128 == 0.
 * ------------------------------------------------------------------------ */
nvq_status int4_pack_weights(const uint8_t* codes, const void* scales_bf16, int64_t N, int64_t K,
                             uint8_t* packed_codes, void* packed_scales, void* stream);

/* ------------------------------------------------------------------------ *
 * W4A16 decode GEMM (MARLIN page, abeam.tech: FP16/BF16 activations x INT4
 * weights with group-128 scales, streaming the weights asynchronously with an
 * L2-sparing cache policy, dequantizing in registers next to the tensor-core
 * MMAs, several warps sharing one output tile).
 *
 *   Y[m, n] = bf16_RNE( sum_g s[n, g] * sum_{k in g} x[m, k] * (u[n, k] - 8) )
 * with the inner sums accumulated in FP32 by the tensor cores and the group
 * scale applied in FP32.  All products are exact; for M <= 16 the inner sum is
 * formed as sum x * (128 + u) + sum x * (-136), equal up to FP32 rounding.
 * Group sums are added in an order fixed by the shapes and the GPU's SM count,
 * so repeated calls give identical results.
 *
 * x_bf16 [M, K] BF16; packed_codes / packed_scales from int4_pack_weights;
 * y_bf16 [M, N] BF16, row stride N, written.
 * workspace / workspace_bytes: unused (w4a16_workspace_bytes returns 0, the
 * partial sums stay on chip); kept so callers need not change.
 * Runs best for M <= 16; larger M is processed 32 rows per pass over W.
 * Launched with programmatic dependent launch: the call may begin while the
 * preceding kernel on the stream is still finishing, and it starts streaming
 * the packed weights before waiting for that kernel (x and y are touched only
 * after the wait).  So the packed weights must not be written by the kernel
 * immediately before it when that kernel lets dependents launch early; no
 * kernel of this library that writes them does, nor does an ordinary copy.
 * It also lets the next kernel on the stream launch early (once its own wait
 * is over, before it computes), so that kernel's CTAs fill the SMs this call
 * frees: a kernel launched after it with programmatic dependent launch must
 * execute griddepcontrol.wait before it reads y (ordinary launches are
 * ordered as usual).
 * Shape rules: M >= 0, N % 32 == 0, K % 128 == 0.
 * ------------------------------------------------------------------------ */
size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K);
nvq_status w4a16_gemm(const void* x_bf16, const uint8_t* packed_codes, const void* packed_scales,
                      void* y_bf16, int64_t M, int64_t N, int64_t K,
                      void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------ *
 * 2:4-sparse INT4 decode (MARLIN page, abeam.tech: its official implementation
 * also combines the group-128 INT4 weights with 2:4 structured sparsity).
 *
 * int4_pack_sparse24 prunes the BF16 master W [N, K] 2:4 (in every run of 4
 * consecutive k of a row the 2 entries of largest |w| stay, the lower k winning
 * among equal magnitudes) and writes the kept INT4 codes in the order of the
 * m16n8k32 sparse MMA, with their 2-bit positions as MMA metadata.  codes and
 * scales_bf16 are int4_quantize of the same W (a run's largest |w| is always
 * kept, so the group scales and the kept codes equal the dense ones).
 * packed: N*K*3/8 bytes (per 32-row x 128-k unit, unit index
 * (n/32)*(K/128) + k/128: two 16-row tiles tt, each 512 bytes of codes then
 * 256 of metadata); packed_scales: N*(K/128)*2 bytes, 64 per unit, 32-bit word
 * 2g + tt holding rows 16tt + g (low half) and 16tt + g + 8 (high half).
 *
 * w4a16_sparse24_gemm: Y = X (s (u - 8) at the kept positions, 0 elsewhere)^T,
 * with the arithmetic of w4a16_gemm (exact products, FP32 sums, group scale in
 * FP32, BF16 RNE out) and its streaming kernel on 24% fewer weight bytes.
 * Shape rules for both: N % 32 == 0, K % 128 == 0; pointers 16-byte aligned.
 * ------------------------------------------------------------------------ */
nvq_status int4_pack_sparse24(const void* w_bf16, const uint8_t* codes, const void* scales_bf16, int64_t N,
                              int64_t K, uint8_t* packed, void* packed_scales, void* stream);
nvq_status w4a16_sparse24_gemm(const void* x_bf16, const uint8_t* packed, const void* packed_scales,
                               void* y_bf16, int64_t M, int64_t N, int64_t K, void* stream);

/* ------------------------------------------------------------------------ *
 * Phase dispatch over one master weight held in both formats (Disaggregated
 * Quantization page, singularity-lens.com, the section on format
 * disaggregation; Mix-Quant page, gist.science, section 2: NVFP4 W4A4 where
 * the layer is compute-bound, weight-only INT4 where it streams weights):
 *
 *   M <= crossover_m:  Y = w4a16_gemm(X, packed INT4 W)
 *   M >  crossover_m:  (codes, scales, t) = nvfp4_quantize(X), then
 *                      Y = nvfp4_gemm_w4a4(X as NVFP4, NVFP4 W)
 *
 * Both weight forms come from the same BF16 master W [N, K]: w_codes /
 * w_scales / w_t from nvfp4_quantize(W), w_packed_* from int4_quantize +
 * int4_pack_weights.  Only the form the chosen path reads must be non-NULL.
 * crossover_m < 0 selects nvq_default_crossover_m(): the largest M at which
 * the W4A16 path was measured faster than quantize + W4A4 on B200 for the
 * Qwen3-8B gate_up shape (K = 4096, N = 24576), weights read from HBM
 * (python profile_case.py --op crossover).
 * workspace: nvq_linear_workspace_bytes(M, N, K, crossover_m) bytes, 16-byte
 * aligned (activation codes, scales, t and the quantizer's scratch), NULL when
 * that is 0.  Output y_bf16 [M, N] BF16, row stride N.
 * Shape rules: those of the chosen path (W4A16: N % 32 == 0, K % 128 == 0;
 * W4A4: N % 8 == 0, K % 64 == 0).  Errors as the underlying calls.
 * ------------------------------------------------------------------------ */
int64_t nvq_default_crossover_m(void);
size_t nvq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t crossover_m);
nvq_status nvq_linear(const void* x_bf16, int64_t M, int64_t N, int64_t K,
                      const uint8_t* w_codes, const uint8_t* w_scales, const float* w_t,
                      const uint8_t* w_packed_codes, const void* w_packed_scales,
                      int64_t crossover_m, void* y_bf16, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ------------------------------------------------------------------------ *
 * Prefill over layers whose NVFP4 weights live in pinned host memory
 * (Disaggregated Quantization page, singularity-lens.com, its ODP scheme:
 * prefill weights read layer block by layer block into two device buffers,
 * the next read overlapping the current compute; here the weights come from
 * pinned host memory, not from an SSD): layer l's
 * weights are copied into device slot l % 2 on copy_stream while layer l - 1
 * runs on compute_stream (activation quantize + W4A4 GEMM), so transfers and
 * GEMMs overlap; a slot is refilled only after the GEMM that read it ended.
 *
 * Per layer: w_codes_host / w_scales_host / w_t_host as written by
 * nvfp4_quantize for W [N, K] (N*K/2 bytes, nvfp4_scales_bytes(N, K) bytes,
 * one float), in pinned host memory (cudaHostAlloc or registered); x_bf16 a
 * device [M, K] BF16 input; y_bf16 a device [M, N] BF16 output.  Layers are
 * independent (the caller chains them through x / y if it wants to).
 * workspace: nvq_prefill_streamed_workspace_bytes(layers, n, M) device bytes,
 * 16-byte aligned: two weight slots sized for the largest layer plus the
 * activation quantizer's outputs and scratch.
 * Both streams must belong to the current device; the call only enqueues work
 * (it returns before the copies and kernels ran); the caller synchronises
 * compute_stream before reading any y.  Shape rules: those of
 * nvfp4_gemm_w4a4 per layer.  NULL pointers, bad shapes or a small
 * workspace are reported before anything is enqueued.
 * ------------------------------------------------------------------------ */
typedef struct {
  const uint8_t* w_codes_host;
  const uint8_t* w_scales_host;
  const float* w_t_host;
  const void* x_bf16;
  void* y_bf16;
  int64_t N, K;
} nvq_stream_layer;

size_t nvq_prefill_streamed_workspace_bytes(const nvq_stream_layer* layers, int n, int64_t M);
nvq_status nvq_prefill_streamed(const nvq_stream_layer* layers, int n, int64_t M, void* workspace,
                                size_t workspace_bytes, void* compute_stream, void* copy_stream);

#ifdef __cplusplus
}
#endif
#endif /* NVQ_H_ */
