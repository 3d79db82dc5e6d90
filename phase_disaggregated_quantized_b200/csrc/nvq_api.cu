// Host side of the libnvq C ABI (include/nvq.h): argument validation, TMA
// descriptor encoding and kernel launches.  All kernels live in this single
// translation unit so the device error word needs no relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/nvq.h"
#include "int4.cuh"
#include "nvfp4_gemm.cuh"
#include "nvfp4_quantize.cuh"
#include "ptx.cuh"
#include "w4a16_gemm.cuh"

namespace nvq {
// Diagnostic kernel: lane 0 initialises an mbarrier for one arrival that never
// comes and waits for its first phase with the given limit.
__global__ void bounded_wait_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  mbar_wait_for(b, 0, limit_ns);
}
}  // namespace nvq

namespace {

thread_local char g_detail[256] = "";

nvq_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_detail, sizeof(g_detail), "%s: %s", where, cudaGetErrorString(e));
  return NVQ_ERR_CUDA;
}

nvq_status fail(nvq_status s, const char* what) {
  snprintf(g_detail, sizeof(g_detail), "%s", what);
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nvq_status launch_status(const char* where) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NVQ_OK : cuda_fail(e, where);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor map: inner dimension `inner` elements, `outer` rows,
// row pitch `pitch_bytes`, box {box_inner, box_outer}.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int64_t kMaxDim = (int64_t)1 << 31;
// 16-element blocks of one quantize call, and output tiles of one GEMM: the
// kernels step through them with 32-bit grid-stride counters, which stay below
// 2^31 + one grid and so never wrap.
constexpr int64_t kMaxBlocks = (int64_t)1 << 31;
bool gemm_tiles_fit(int64_t M, int64_t N) { return ((M + 127) / 128) * ((N + 127) / 128) < kMaxBlocks; }

// Decode launch: a persistent grid of clusters of nvq::w4a16::CS CTAs, as many
// as can be resident at once (one CTA per SM), never more clusters than output
// tiles (32 weight rows dense, 16 for 2:4 sparse).  Batch rows are handled 8 * NT8 at a time.
constexpr int kMaxDevices = 64;

template <int NT8, bool SPARSE = false>
nvq_status launch_w4a16(const void* x, const uint8_t* pc, const void* ps, void* y, int64_t M, int64_t N, int64_t K,
                        cudaStream_t stream) {
  using C = nvq::w4a16::Cfg<NT8, SPARSE>;
  auto fn = nvq::w4a16::w4a16_kernel<NT8, SPARSE>;
  static std::atomic<int> max_clusters[kMaxDevices];   // 0: not queried yet on that device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "w4a16_gemm: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(NVQ_ERR_CUDA, "w4a16_gemm: device index out of range");
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nvq::w4a16::CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may launch during the previous kernel's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int maxc = max_clusters[dev].load(std::memory_order_acquire);
  if (maxc == 0) {                              // two threads may both get here: same result
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "w4a16_gemm: shared memory attribute");
    cfg.gridDim = dim3(nvq::w4a16::CS, 1, 1);
    e = cudaOccupancyMaxActiveClusters(&maxc, fn, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "w4a16_gemm: cudaOccupancyMaxActiveClusters");
    if (maxc < 1) return fail(NVQ_ERR_CUDA, "w4a16_gemm: no cluster of the decode kernel fits on this GPU");
    max_clusters[dev].store(maxc, std::memory_order_release);
  }
  const int64_t tiles = N / nvq::w4a16::Unit<SPARSE>::ROWS;
  const int64_t nclu = std::min<int64_t>(maxc, tiles);
  cfg.gridDim = dim3((unsigned)(nclu * nvq::w4a16::CS), 1, 1);
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, fn, static_cast<const __nv_bfloat16*>(x), pc, static_cast<const uint8_t*>(ps),
                         static_cast<__nv_bfloat16*>(y), (uint32_t)M, (uint32_t)N, (uint32_t)K);
  if (e != cudaSuccess) return cuda_fail(e, "w4a16_kernel launch");
  return launch_status("w4a16_kernel");
}

// Workspace of nvq_linear's W4A4 path: activation codes, tiled scales, t and
// the quantizer's scratch, each section 256-byte aligned.
struct LinearWs {
  size_t codes, scales, t, scratch, total;
};
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
LinearWs linear_ws_layout(int64_t M, int64_t K) {
  LinearWs L;
  L.codes = 0;
  L.scales = align256((size_t)M * (size_t)(K / 2));
  L.t = L.scales + align256(nvfp4_scales_bytes(M, K));
  L.scratch = L.t + 256;
  L.total = L.scratch + align256(std::max<size_t>(16, nvfp4_quantize_workspace_bytes(M, K)));
  return L;
}

// Workspace of nvq_prefill_streamed: two weight slots sized for the largest
// layer (codes, tiled scales, t) and one set of activation quantizer outputs
// sized for the largest K, sections 256-byte aligned.
struct StreamWs {
  bool ok = false;
  size_t slot[2] = {0, 0};
  size_t scales_off = 0, t_off = 0;                 // inside a slot
  size_t act = 0;                                   // activation codes, then the rest
  size_t act_scales_off = 0, act_t_off = 0, act_scratch_off = 0, act_scratch_bytes = 0;
  size_t total = 0;
};
StreamWs stream_ws_layout(const nvq_stream_layer* layers, int n, int64_t M) {
  StreamWs W;
  size_t codes = 0, scales = 0, acodes = 0, ascales = 0, ascratch = 16;
  for (int l = 0; l < n; ++l) {
    const int64_t N = layers[l].N, K = layers[l].K;
    if (N <= 0 || K <= 0 || N >= kMaxDim || K >= kMaxDim || M >= kMaxDim) return W;
    codes = std::max(codes, (size_t)N * (size_t)(K / 2));
    scales = std::max(scales, nvfp4_scales_bytes(N, K));
    acodes = std::max(acodes, (size_t)M * (size_t)(K / 2));
    ascales = std::max(ascales, nvfp4_scales_bytes(M, K));
    ascratch = std::max(ascratch, nvfp4_quantize_workspace_bytes(M, K));
  }
  W.scales_off = align256(codes);
  W.t_off = W.scales_off + align256(scales);
  const size_t slot_bytes = W.t_off + 256;
  W.slot[0] = 0;
  W.slot[1] = slot_bytes;
  W.act = 2 * slot_bytes;
  W.act_scales_off = align256(acodes);
  W.act_t_off = W.act_scales_off + align256(ascales);
  W.act_scratch_off = W.act_t_off + 256;
  W.act_scratch_bytes = align256(ascratch);
  W.total = W.act + W.act_scratch_off + W.act_scratch_bytes;
  W.ok = true;
  return W;
}

}  // namespace

extern "C" {

int nvq_abi_version(void) { return 1; }

const char* nvq_status_string(nvq_status s) {
  switch (s) {
    case NVQ_OK: return "NVQ_OK";
    case NVQ_ERR_INVALID_ARG: return "NVQ_ERR_INVALID_ARG";
    case NVQ_ERR_UNSUPPORTED_SHAPE: return "NVQ_ERR_UNSUPPORTED_SHAPE";
    case NVQ_ERR_MISALIGNED: return "NVQ_ERR_MISALIGNED";
    case NVQ_ERR_WORKSPACE: return "NVQ_ERR_WORKSPACE";
    case NVQ_ERR_CUDA: return "NVQ_ERR_CUDA";
    case NVQ_ERR_DEVICE_TIMEOUT: return "NVQ_ERR_DEVICE_TIMEOUT";
  }
  return "NVQ_ERR_UNKNOWN";
}

const char* nvq_last_error_detail(void) { return g_detail; }

nvq_status nvq_check_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "nvq_check_device_error: synchronize");
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, nvq::g_device_error, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "nvq_check_device_error: read");
  if (word != 0u) {
    const unsigned int zero = 0u;
    e = cudaMemcpyToSymbol(nvq::g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "nvq_check_device_error: clear");
    return fail(NVQ_ERR_DEVICE_TIMEOUT, "a kernel gave up on a bounded wait");
  }
  return NVQ_OK;
}

// One thread waits on an mbarrier that nothing completes, with the same bounded
// wait the pipelines use, so the wait runs out and raises the error word.
nvq_status nvq_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 100000000ull)
    return fail(NVQ_ERR_INVALID_ARG, "nvq_selftest_wait_timeout: limit_ns outside [1 us, 100 ms]");
  nvq::bounded_wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return launch_status("bounded_wait_probe_kernel");
}

// ------------------------------------------------------------------ NVFP4 quantize
size_t nvfp4_scales_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 64) return 0;
  return (size_t)((rows + 127) / 128 * 128) * (size_t)(K / 16);
}

// 512-byte atoms of 128 rows x 4 blocks, row-tile major: the atom of (row, kb)
// is (row / 128) * (K / 64) + kb / 4; inside it the byte is 16 (row % 32) +
// 4 ((row % 128) / 32) + kb % 4 -- the 32 x 16-byte matrix whose column c holds
// rows 32 c + lane, as the block-scaled MMA reads scales from TMEM.
int64_t nvfp4_scale_offset(int64_t row, int64_t kblock, int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0 || K % 64 != 0 || row < 0 || row >= rows || kblock < 0 || kblock >= K / 16) return -1;
  const int64_t atom = (row / 128) * (K / 64) + kblock / 4;
  return atom * 512 + 16 * (row % 32) + 4 * ((row % 128) / 32) + kblock % 4;
}

size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 0;
  return (size_t)nvq::kAmaxMaxBlocks * sizeof(float);
}

}  // extern "C"

namespace {

nvq_status quantize_validate(const char* name, const void* x_bf16, int64_t rows, int64_t K, uint8_t* codes,
                             uint8_t* scales, float* tensor_scale_out) {
  char msg[160];
  if (rows < 0 || K <= 0) {
    snprintf(msg, sizeof(msg), "%s: rows < 0 or K <= 0", name);
    return fail(NVQ_ERR_INVALID_ARG, msg);
  }
  if (K % 64 != 0) {
    snprintf(msg, sizeof(msg), "%s: K %% 64 != 0", name);
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, msg);
  }
  if (rows >= kMaxDim || K >= kMaxDim || (rows * (K / 16)) >= kMaxBlocks) {
    snprintf(msg, sizeof(msg), "%s: tensor too large", name);
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, msg);
  }
  if (tensor_scale_out == nullptr) {
    snprintf(msg, sizeof(msg), "%s: tensor_scale_out is NULL", name);
    return fail(NVQ_ERR_INVALID_ARG, msg);
  }
  if (rows > 0 && (x_bf16 == nullptr || codes == nullptr || scales == nullptr)) {
    snprintf(msg, sizeof(msg), "%s: NULL tensor pointer", name);
    return fail(NVQ_ERR_INVALID_ARG, msg);
  }
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales)) {
    snprintf(msg, sizeof(msg), "%s: pointer not 16-byte aligned", name);
    return fail(NVQ_ERR_MISALIGNED, msg);
  }
  return NVQ_OK;
}

// CTAs of the amax pre-pass over rows x K elements (rows > 0): four 16-byte
// loads per thread per sweep, at most kAmaxMaxBlocks partials.
int amax_grid(int64_t rows, int64_t K) {
  const size_t nvec = (size_t)rows * (size_t)K / 8;
  const size_t want = (nvec + 4 * nvq::kAmaxThreads - 1) / (4 * nvq::kAmaxThreads);
  return (int)std::max<size_t>(1, std::min<size_t>(nvq::kAmaxMaxBlocks, want));
}

// The quantize pass over rows x K.  Right after the amax pass of the same call
// (after_amax) it is launched as a programmatic dependent of that pass: its CTAs
// start and request their first blocks of x during the pass's tail and wait for
// it before reading the partials.  Otherwise a plain launch (its x may come from
// the kernel just before it).
nvq_status launch_quantize_kernel(const void* x_bf16, int64_t rows, int64_t K, const float* tensor_scale_in,
                                  const float* partial, int amax_blocks, uint8_t* codes, uint8_t* scales,
                                  float* tensor_scale_out, bool after_amax, cudaStream_t stream) {
  const uint64_t nblocks = (uint64_t)rows * (uint64_t)(K / 16);
  const uint64_t want = (nblocks + nvq::kQuantThreads - 1) / nvq::kQuantThreads;
  const int grid = (int)std::max<uint64_t>(1, std::min<uint64_t>(want, (uint64_t)sm_count()));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(nvq::kQuantThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = after_amax ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, nvq::nvfp4_quantize_kernel, static_cast<const uint4*>(x_bf16),
                                           (uint32_t)rows, (uint32_t)K, tensor_scale_in, partial, amax_blocks,
                                           reinterpret_cast<uint2*>(codes), scales, tensor_scale_out);
  if (e != cudaSuccess) return cuda_fail(e, "nvfp4_quantize_kernel launch");
  return launch_status("nvfp4_quantize_kernel");
}

// amax pre-pass (when t is not given) into `partial[0 .. amax_blocks)`, then the quantize pass.
nvq_status quantize_launch(const void* x_bf16, int64_t rows, int64_t K, const float* tensor_scale_in, uint8_t* codes,
                           uint8_t* scales, float* tensor_scale_out, float* partial, int amax_blocks,
                           cudaStream_t stream) {
  if (amax_blocks > 0) {
    const size_t nvec = (size_t)rows * (size_t)K / 8;
    nvq::nvfp4_amax_kernel<<<amax_blocks, nvq::kAmaxThreads, 0, stream>>>(static_cast<const uint4*>(x_bf16), nvec,
                                                                           partial);
    nvq_status st = launch_status("nvfp4_amax_kernel");
    if (st != NVQ_OK) return st;
  }
  return launch_quantize_kernel(x_bf16, rows, K, tensor_scale_in, partial, amax_blocks, codes, scales,
                                tensor_scale_out, amax_blocks > 0, stream);
}

}  // namespace

extern "C" {

nvq_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t K, const float* tensor_scale_in,
                          uint8_t* codes, uint8_t* scales, float* tensor_scale_out, void* workspace,
                          size_t workspace_bytes, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (rows < 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_quantize: rows < 0 or K <= 0");
  if (K % 64 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_quantize: K % 64 != 0");
  if (rows >= kMaxDim || K >= kMaxDim || (rows * (K / 16)) >= kMaxBlocks)
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_quantize: tensor too large");
  if (tensor_scale_out == nullptr) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_quantize: tensor_scale_out is NULL");
  if (rows > 0 && (x_bf16 == nullptr || codes == nullptr || scales == nullptr))
    return fail(NVQ_ERR_INVALID_ARG, "nvfp4_quantize: NULL tensor pointer");
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales))
    return fail(NVQ_ERR_MISALIGNED, "nvfp4_quantize: pointer not 16-byte aligned");
  const bool need_amax = tensor_scale_in == nullptr && rows > 0;
  int amax_blocks = 0;
  if (need_amax) {
    const size_t nvec = (size_t)rows * (size_t)K / 8;
    amax_blocks = amax_grid(rows, K);
    if (workspace == nullptr || workspace_bytes < (size_t)amax_blocks * sizeof(float))
      return fail(NVQ_ERR_WORKSPACE, "nvfp4_quantize: workspace missing or too small");
    if ((reinterpret_cast<uintptr_t>(workspace) & 3u) != 0)
      return fail(NVQ_ERR_MISALIGNED, "nvfp4_quantize: workspace not 4-byte aligned");
    nvq::nvfp4_amax_kernel<<<amax_blocks, nvq::kAmaxThreads, 0, stream>>>(
        static_cast<const uint4*>(x_bf16), nvec, static_cast<float*>(workspace));
    nvq_status st = launch_status("nvfp4_amax_kernel");
    if (st != NVQ_OK) return st;
  }
  return launch_quantize_kernel(x_bf16, rows, K, tensor_scale_in, static_cast<const float*>(workspace),
                                amax_blocks, codes, scales, tensor_scale_out, need_amax, stream);
}

nvq_status nvfp4_amax(const void* x_bf16, int64_t rows, int64_t K, float* amax_out, void* workspace,
                      size_t workspace_bytes, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (rows < 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_amax: rows < 0 or K <= 0");
  if (K % 64 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_amax: K % 64 != 0");
  if (rows >= kMaxDim || K >= kMaxDim || (rows * (K / 16)) >= kMaxBlocks)
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_amax: tensor too large");
  if (amax_out == nullptr || (rows > 0 && x_bf16 == nullptr)) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_amax: NULL pointer");
  if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(amax_out) & 3u) != 0)
    return fail(NVQ_ERR_MISALIGNED, "nvfp4_amax: x not 16-byte or amax_out not 4-byte aligned");
  int amax_blocks = 0;
  if (rows > 0) {
    amax_blocks = amax_grid(rows, K);
    if (workspace == nullptr || workspace_bytes < (size_t)amax_blocks * sizeof(float))
      return fail(NVQ_ERR_WORKSPACE, "nvfp4_amax: workspace missing or too small");
    if ((reinterpret_cast<uintptr_t>(workspace) & 3u) != 0)
      return fail(NVQ_ERR_MISALIGNED, "nvfp4_amax: workspace not 4-byte aligned");
    const size_t nvec = (size_t)rows * (size_t)K / 8;
    nvq::nvfp4_amax_kernel<<<amax_blocks, nvq::kAmaxThreads, 0, stream>>>(static_cast<const uint4*>(x_bf16), nvec,
                                                                           static_cast<float*>(workspace));
    nvq_status st = launch_status("nvfp4_amax_kernel");
    if (st != NVQ_OK) return st;
  }
  nvq::nvfp4_amax_finish_kernel<<<1, 32, 0, stream>>>(static_cast<const float*>(workspace), amax_blocks, amax_out);
  return launch_status("nvfp4_amax_finish_kernel");
}

nvq_status nvfp4_scale_from_amax(const float* amax, float* tensor_scale_out, void* stream_) {
  if (amax == nullptr || tensor_scale_out == nullptr) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_scale_from_amax: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(amax) & 3u) != 0 || (reinterpret_cast<uintptr_t>(tensor_scale_out) & 3u) != 0)
    return fail(NVQ_ERR_MISALIGNED, "nvfp4_scale_from_amax: pointer not 4-byte aligned");
  nvq::nvfp4_scale_from_amax_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream_)>>>(amax, tensor_scale_out);
  return launch_status("nvfp4_scale_from_amax_kernel");
}

// ------------------------------------------------------------------ NVFP4 GEMM
}  // extern "C"

namespace {

// EPI 0: y_bf16 receives Y.  EPI 1: h_* receive NVFP4(silu(gate) * up) with the
// static scale t_h (B rows interleaved in blocks of 128: gate, up, ...).
template <int EPI>
nvq_status launch_w4a4(const uint8_t* x_codes, const uint8_t* x_scales, const float* t_x, const uint8_t* w_codes,
                       const uint8_t* w_scales, const float* t_w, void* y_bf16, int64_t M, int64_t N, int64_t K,
                       uint8_t* h_codes, uint8_t* h_scales, const float* t_h, cudaStream_t stream) {
  using namespace nvq::w4a4;
  CUtensorMap ma, mb, my;
  memset(&my, 0, sizeof(my));                               // EPI 1 never touches Y
  if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, x_codes, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2,
                   BKB, BM) ||
      !make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                   BKB, BN) ||
      (EPI == 0 && !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y_bf16, (uint64_t)N, (uint64_t)M,
                                (uint64_t)N * 2, C_COLS, 32)))   // one epilogue warp: 32 rows x 64 columns
    return fail(NVQ_ERR_CUDA, "nvfp4_gemm_w4a4: tensor map encoding failed");
  Params p;
  p.x_scales = x_scales;
  p.w_scales = w_scales;
  p.t_x = t_x;
  p.t_w = t_w;
  p.M = (uint32_t)M;
  p.N = (uint32_t)N;
  p.K = (uint32_t)K;
  p.num_m_tiles = (uint32_t)((M + BM - 1) / BM);
  p.num_n_tiles = (uint32_t)((N + BN - 1) / BN);
  p.num_k_stages = (uint32_t)((K / 2 + BKB - 1) / BKB);
  p.k_atoms = (uint32_t)(K / 64);
  p.n_row_atoms = (uint32_t)((N + 127) / 128);
  // Sweep the smaller operand every wave (it stays in L2), stream the larger once.
  p.m_fastest = (uint64_t)M <= (uint64_t)N ? 1u : 0u;   // both operands have K/2 + K/16 bytes per row
  p.h_codes = h_codes;
  p.h_scales = h_scales;
  p.t_h = t_h;
  p.h_katoms = (uint32_t)(N / 2 / 64);
  // The shared-memory opt-in is a per-device setting of the kernel: once per device.
  int dev = 0;
  const cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) return cuda_fail(de, "nvfp4_gemm_w4a4: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(NVQ_ERR_CUDA, "nvfp4_gemm_w4a4: device index out of range");
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];   // zero = cudaSuccess
  std::call_once(once[dev], [dev] {
    attr_err[dev] = cudaFuncSetAttribute(nvfp4_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BYTES);
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "nvfp4_gemm_w4a4: smem attribute");
  const uint64_t tiles = (uint64_t)p.num_m_tiles * p.num_n_tiles;
  const int grid = (int)std::min<uint64_t>(tiles, (uint64_t)sm_count());
  nvfp4_gemm_kernel<EPI><<<grid, THREADS, SMEM_BYTES, stream>>>(ma, mb, my, p);
  return launch_status("nvfp4_gemm_kernel");
}

}  // namespace

extern "C" {

nvq_status nvfp4_gemm_w4a4(const uint8_t* x_codes, const uint8_t* x_scales, const float* t_x,
                           const uint8_t* w_codes, const uint8_t* w_scales, const float* t_w, void* y_bf16,
                           int64_t M, int64_t N, int64_t K, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (M < 0 || N <= 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_gemm_w4a4: bad sizes");
  if (N % 8 != 0 || K % 64 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_gemm_w4a4: need N % 8 == 0, K % 64 == 0");
  if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || !gemm_tiles_fit(M, N))
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_gemm_w4a4: too large");
  if (!x_codes || !x_scales || !t_x || !w_codes || !w_scales || !t_w || !y_bf16)
    return fail(NVQ_ERR_INVALID_ARG, "nvfp4_gemm_w4a4: NULL pointer");
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(y_bf16) || (reinterpret_cast<uintptr_t>(t_x) & 3u) || (reinterpret_cast<uintptr_t>(t_w) & 3u))
    return fail(NVQ_ERR_MISALIGNED, "nvfp4_gemm_w4a4: pointer not aligned");
  if (M == 0) return NVQ_OK;
  return launch_w4a4<0>(x_codes, x_scales, t_x, w_codes, w_scales, t_w, y_bf16, M, N, K, nullptr, nullptr, nullptr,
                        stream);
}

nvq_status nvfp4_gemm_w4a4_swiglu(const uint8_t* x_codes, const uint8_t* x_scales, const float* t_x,
                                  const uint8_t* w_codes, const uint8_t* w_scales, const float* t_w,
                                  const float* t_h, uint8_t* h_codes, uint8_t* h_scales, int64_t M, int64_t N,
                                  int64_t K, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (M < 0 || N <= 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_gemm_w4a4_swiglu: bad sizes");
  if (N % 256 != 0 || K % 64 != 0)
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_gemm_w4a4_swiglu: need N % 256 == 0, K % 64 == 0");
  if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || !gemm_tiles_fit(M, N))
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_gemm_w4a4_swiglu: too large");
  if (!x_codes || !x_scales || !t_x || !w_codes || !w_scales || !t_w || !t_h || !h_codes || !h_scales)
    return fail(NVQ_ERR_INVALID_ARG, "nvfp4_gemm_w4a4_swiglu: NULL pointer");
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(h_codes) || !aligned16(h_scales) || (reinterpret_cast<uintptr_t>(t_x) & 3u) ||
      (reinterpret_cast<uintptr_t>(t_w) & 3u) || (reinterpret_cast<uintptr_t>(t_h) & 3u))
    return fail(NVQ_ERR_MISALIGNED, "nvfp4_gemm_w4a4_swiglu: pointer not aligned");
  if (M == 0) return NVQ_OK;
  return launch_w4a4<1>(x_codes, x_scales, t_x, w_codes, w_scales, t_w, nullptr, M, N, K, h_codes, h_scales, t_h,
                        stream);
}

// ------------------------------------------------------------------ INT4
nvq_status int4_quantize(const void* w_bf16, int64_t N, int64_t K, uint8_t* codes, void* scales_bf16,
                         void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (N < 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "int4_quantize: bad sizes");
  if (K % 128 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "int4_quantize: K % 128 != 0");
  if (N >= kMaxDim || K >= kMaxDim) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "int4_quantize: too large");
  if (N == 0) return NVQ_OK;
  if (!w_bf16 || !codes || !scales_bf16) return fail(NVQ_ERR_INVALID_ARG, "int4_quantize: NULL pointer");
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(scales_bf16))
    return fail(NVQ_ERR_MISALIGNED, "int4_quantize: pointer not 16-byte aligned");
  const uint64_t groups = (uint64_t)N * (uint64_t)(K / 128);
  const uint64_t want = (groups + 7) / 8;
  const int grid = (int)std::max<uint64_t>(1, std::min<uint64_t>(want, (uint64_t)sm_count() * 16));
  nvq::int4_quantize_kernel<<<grid, nvq::kInt4QuantThreads, 0, stream>>>(
      static_cast<const uint2*>(w_bf16), (uint32_t)N, (uint32_t)K, reinterpret_cast<uint16_t*>(codes),
      static_cast<uint16_t*>(scales_bf16));
  return launch_status("int4_quantize_kernel");
}

nvq_status int4_pack_weights(const uint8_t* codes, const void* scales_bf16, int64_t N, int64_t K,
                             uint8_t* packed_codes, void* packed_scales, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (N < 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "int4_pack_weights: bad sizes");
  if (N % 32 != 0 || K % 128 != 0)
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "int4_pack_weights: need N % 32 == 0, K % 128 == 0");
  if (N >= kMaxDim || K >= kMaxDim) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "int4_pack_weights: too large");
  if (N == 0) return NVQ_OK;
  if (!codes || !scales_bf16 || !packed_codes || !packed_scales)
    return fail(NVQ_ERR_INVALID_ARG, "int4_pack_weights: NULL pointer");
  if (!aligned16(codes) || !aligned16(scales_bf16) || !aligned16(packed_codes) || !aligned16(packed_scales))
    return fail(NVQ_ERR_MISALIGNED, "int4_pack_weights: pointer not 16-byte aligned");
  const uint64_t nwords = (uint64_t)N * (uint64_t)K / 8;
  const int grid = (int)std::max<uint64_t>(1, std::min<uint64_t>((nwords + 255) / 256, (uint64_t)sm_count() * 16));
  nvq::int4_pack_kernel<<<grid, 256, 0, stream>>>(codes, static_cast<const uint16_t*>(scales_bf16), (uint32_t)N,
                                                  (uint32_t)K, reinterpret_cast<uint32_t*>(packed_codes),
                                                  static_cast<uint32_t*>(packed_scales));
  return launch_status("int4_pack_kernel");
}

// ------------------------------------------------------------------ W4A16 decode GEMM
size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)M;
  (void)N;
  (void)K;
  return 0;                                      // partial sums stay on chip
}

nvq_status w4a16_gemm(const void* x_bf16, const uint8_t* packed_codes, const void* packed_scales, void* y_bf16,
                      int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes, void* stream_) {
  (void)workspace;
  (void)workspace_bytes;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (M < 0 || N <= 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "w4a16_gemm: bad sizes");
  if (N % 32 != 0 || K % 128 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "w4a16_gemm: need N % 32 == 0, K % 128 == 0");
  if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || (N / 32) * (K / 128) >= ((int64_t)1 << 32))
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "w4a16_gemm: too large");
  if (M == 0) return NVQ_OK;
  if (!x_bf16 || !packed_codes || !packed_scales || !y_bf16) return fail(NVQ_ERR_INVALID_ARG, "w4a16_gemm: NULL pointer");
  if (!aligned16(x_bf16) || !aligned16(packed_codes) || !aligned16(packed_scales) || !aligned16(y_bf16))
    return fail(NVQ_ERR_MISALIGNED, "w4a16_gemm: pointer not 16-byte aligned");
  if (M <= 8) return launch_w4a16<1>(x_bf16, packed_codes, packed_scales, y_bf16, M, N, K, stream);
  if (M <= 16) return launch_w4a16<2>(x_bf16, packed_codes, packed_scales, y_bf16, M, N, K, stream);
  return launch_w4a16<4>(x_bf16, packed_codes, packed_scales, y_bf16, M, N, K, stream);
}

// ------------------------------------------------------------------ 2:4 sparse INT4 decode
nvq_status int4_pack_sparse24(const void* w_bf16, const uint8_t* codes, const void* scales_bf16, int64_t N,
                              int64_t K, uint8_t* packed, void* packed_scales, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (N < 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "int4_pack_sparse24: bad sizes");
  if (N % 32 != 0 || K % 128 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "int4_pack_sparse24: need N % 32 == 0, K % 128 == 0");
  if (N >= kMaxDim || K >= kMaxDim) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "int4_pack_sparse24: too large");
  if (N == 0) return NVQ_OK;
  if (!w_bf16 || !codes || !scales_bf16 || !packed || !packed_scales)
    return fail(NVQ_ERR_INVALID_ARG, "int4_pack_sparse24: NULL pointer");
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(scales_bf16) || !aligned16(packed) || !aligned16(packed_scales))
    return fail(NVQ_ERR_MISALIGNED, "int4_pack_sparse24: pointer not 16-byte aligned");
  const uint64_t threads = (uint64_t)(N / 32) * (uint64_t)(K / 128) * 256;
  const int grid = (int)std::max<uint64_t>(1, std::min<uint64_t>((threads + 255) / 256, (uint64_t)sm_count() * 16));
  nvq::int4_pack_sparse24_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint2*>(w_bf16), codes,
                                                           static_cast<const uint16_t*>(scales_bf16), (uint32_t)N,
                                                           (uint32_t)K, reinterpret_cast<uint32_t*>(packed),
                                                           static_cast<uint32_t*>(packed_scales));
  return launch_status("int4_pack_sparse24_kernel");
}

nvq_status w4a16_sparse24_gemm(const void* x_bf16, const uint8_t* packed, const void* packed_scales, void* y_bf16,
                               int64_t M, int64_t N, int64_t K, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (M < 0 || N <= 0 || K <= 0) return fail(NVQ_ERR_INVALID_ARG, "w4a16_sparse24_gemm: bad sizes");
  if (N % 32 != 0 || K % 128 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "w4a16_sparse24_gemm: need N % 32 == 0, K % 128 == 0");
  if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || (N / 32) * (K / 128) >= ((int64_t)1 << 32))
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "w4a16_sparse24_gemm: too large");
  if (M == 0) return NVQ_OK;
  if (!x_bf16 || !packed || !packed_scales || !y_bf16) return fail(NVQ_ERR_INVALID_ARG, "w4a16_sparse24_gemm: NULL pointer");
  if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(packed_scales) || !aligned16(y_bf16))
    return fail(NVQ_ERR_MISALIGNED, "w4a16_sparse24_gemm: pointer not 16-byte aligned");
  if (M <= 8) return launch_w4a16<1, true>(x_bf16, packed, packed_scales, y_bf16, M, N, K, stream);
  if (M <= 16) return launch_w4a16<2, true>(x_bf16, packed, packed_scales, y_bf16, M, N, K, stream);
  return launch_w4a16<4, true>(x_bf16, packed, packed_scales, y_bf16, M, N, K, stream);
}

// ------------------------------------------------------------------ phase dispatch
// Largest M at which W4A16 beat quantize + W4A4 on B200 for K = 4096, N = 24576
// with weights read from HBM (profile_case --op crossover: 25.1 vs 28.9 us at
// M = 16, 39.9 vs 30.0 us at M = 32).
constexpr int64_t kDefaultCrossoverM = 16;

int64_t nvq_default_crossover_m(void) { return kDefaultCrossoverM; }

size_t nvq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t crossover_m) {
  (void)N;
  if (crossover_m < 0) crossover_m = kDefaultCrossoverM;
  if (M <= crossover_m || M <= 0 || K <= 0 || K % 64 != 0) return 0;
  return linear_ws_layout(M, K).total;
}

size_t nvq_workspace_bytes(int op, int64_t M, int64_t N, int64_t K) {
  switch (op) {
    case NVQ_OP_NVFP4_QUANTIZE: return nvfp4_quantize_workspace_bytes(M, K);
    case NVQ_OP_NVFP4_GEMM: return 0;
    case NVQ_OP_W4A16_GEMM: return w4a16_workspace_bytes(M, N, K);
    case NVQ_OP_LINEAR: return nvq_linear_workspace_bytes(M, N, K, -1);
  }
  return SIZE_MAX;
}

nvq_status nvq_linear(const void* x_bf16, int64_t M, int64_t N, int64_t K, const uint8_t* w_codes,
                      const uint8_t* w_scales, const float* w_t, const uint8_t* w_packed_codes,
                      const void* w_packed_scales, int64_t crossover_m, void* y_bf16, void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (crossover_m < 0) crossover_m = kDefaultCrossoverM;
  if (M <= crossover_m) {
    if (!w_packed_codes || !w_packed_scales) return fail(NVQ_ERR_INVALID_ARG, "nvq_linear: W4A16 path needs the packed INT4 weights");
    return w4a16_gemm(x_bf16, w_packed_codes, w_packed_scales, y_bf16, M, N, K, nullptr, 0, stream);
  }
  if (!w_codes || !w_scales || !w_t) return fail(NVQ_ERR_INVALID_ARG, "nvq_linear: W4A4 path needs the NVFP4 weights");
  if (K <= 0 || K % 64 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvq_linear: W4A4 path needs K % 64 == 0");
  if (N <= 0 || N % 8 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvq_linear: W4A4 path needs N % 8 == 0");
  const LinearWs L = linear_ws_layout(M, K);
  if (workspace == nullptr || workspace_bytes < L.total) return fail(NVQ_ERR_WORKSPACE, "nvq_linear: workspace too small");
  if (!aligned16(workspace)) return fail(NVQ_ERR_MISALIGNED, "nvq_linear: workspace not 16-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* xc = ws + L.codes;
  uint8_t* xs = ws + L.scales;
  float* tx = reinterpret_cast<float*>(ws + L.t);
  nvq_status st = nvfp4_quantize(x_bf16, M, K, nullptr, xc, xs, tx, ws + L.scratch, L.total - L.scratch, stream);
  if (st != NVQ_OK) return st;
  return nvfp4_gemm_w4a4(xc, xs, tx, w_codes, w_scales, w_t, y_bf16, M, N, K, stream);
}

// ------------------------------------------------------------------ prefill with host-resident weights
size_t nvq_prefill_streamed_workspace_bytes(const nvq_stream_layer* layers, int n, int64_t M) {
  if (layers == nullptr || n <= 0 || M < 0) return 0;
  StreamWs W = stream_ws_layout(layers, n, M);
  return W.ok ? W.total : 0;
}

nvq_status nvq_prefill_streamed(const nvq_stream_layer* layers, int n, int64_t M, void* workspace,
                                size_t workspace_bytes, void* compute_stream_, void* copy_stream_) {
  if (layers == nullptr || n <= 0 || M < 0) return fail(NVQ_ERR_INVALID_ARG, "nvq_prefill_streamed: bad layer list or M");
  for (int l = 0; l < n; ++l) {
    const nvq_stream_layer& L = layers[l];
    if (!L.w_codes_host || !L.w_scales_host || !L.w_t_host || !L.x_bf16 || !L.y_bf16)
      return fail(NVQ_ERR_INVALID_ARG, "nvq_prefill_streamed: NULL pointer in a layer");
    if (L.N <= 0 || L.K <= 0) return fail(NVQ_ERR_INVALID_ARG, "nvq_prefill_streamed: bad layer sizes");
    if (L.N % 8 != 0 || L.K % 64 != 0) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvq_prefill_streamed: need N % 8 == 0, K % 64 == 0");
    if (M >= kMaxDim || L.N >= kMaxDim || L.K >= kMaxDim) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvq_prefill_streamed: too large");
    if (!aligned16(L.x_bf16) || !aligned16(L.y_bf16)) return fail(NVQ_ERR_MISALIGNED, "nvq_prefill_streamed: x / y not 16-byte aligned");
  }
  const StreamWs W = stream_ws_layout(layers, n, M);
  if (!W.ok) return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvq_prefill_streamed: sizes overflow");
  if (workspace == nullptr || workspace_bytes < W.total) return fail(NVQ_ERR_WORKSPACE, "nvq_prefill_streamed: workspace too small");
  if (!aligned16(workspace)) return fail(NVQ_ERR_MISALIGNED, "nvq_prefill_streamed: workspace not 16-byte aligned");
  if (M == 0) return NVQ_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(compute_stream_), xs = static_cast<cudaStream_t>(copy_stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // ready[s]: slot s holds the next layer's weights; freed[s]: the GEMM that read slot s ended.
  cudaEvent_t ready[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
  nvq_status st = NVQ_OK;
  for (int s = 0; s < 2 && st == NVQ_OK; ++s) {
    cudaError_t e = cudaEventCreateWithFlags(&ready[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&freed[s], cudaEventDisableTiming);
    if (e != cudaSuccess) st = cuda_fail(e, "nvq_prefill_streamed: event");
  }
  if (st == NVQ_OK) {                            // work already queued on compute_stream may still read the slots
    cudaError_t e = cudaEventRecord(freed[0], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(xs, freed[0], 0);
    if (e != cudaSuccess) st = cuda_fail(e, "nvq_prefill_streamed: stream order");
  }
  for (int l = 0; l < n && st == NVQ_OK; ++l) {
    const nvq_stream_layer& L = layers[l];
    const int s = l & 1;
    uint8_t* slot = ws + W.slot[s];
    const size_t cb = (size_t)L.N * (size_t)(L.K / 2), sb = nvfp4_scales_bytes(L.N, L.K);
    cudaError_t e = cudaSuccess;
    if (l >= 2) e = cudaStreamWaitEvent(xs, freed[s], 0);       // the GEMM of layer l - 2 read this slot
    if (e == cudaSuccess) e = cudaMemcpyAsync(slot, L.w_codes_host, cb, cudaMemcpyHostToDevice, xs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(slot + W.scales_off, L.w_scales_host, sb, cudaMemcpyHostToDevice, xs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(slot + W.t_off, L.w_t_host, sizeof(float), cudaMemcpyHostToDevice, xs);
    if (e == cudaSuccess) e = cudaEventRecord(ready[s], xs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ready[s], 0);
    if (e != cudaSuccess) { st = cuda_fail(e, "nvq_prefill_streamed: copy"); break; }
    uint8_t* xc = ws + W.act;
    uint8_t* xsc = xc + W.act_scales_off;
    float* tx = reinterpret_cast<float*>(xc + W.act_t_off);
    st = nvfp4_quantize(L.x_bf16, M, L.K, nullptr, xc, xsc, tx, xc + W.act_scratch_off, W.act_scratch_bytes, cs);
    if (st == NVQ_OK)
      st = nvfp4_gemm_w4a4(xc, xsc, tx, slot, slot + W.scales_off, reinterpret_cast<const float*>(slot + W.t_off),
                           L.y_bf16, M, L.N, L.K, cs);
    if (st == NVQ_OK) {
      e = cudaEventRecord(freed[s], cs);
      if (e != cudaSuccess) st = cuda_fail(e, "nvq_prefill_streamed: event record");
    }
  }
  for (int s = 0; s < 2; ++s) {                  // released once the work recorded on them completes
    if (ready[s]) cudaEventDestroy(ready[s]);
    if (freed[s]) cudaEventDestroy(freed[s]);
  }
  return st;
}

}  // extern "C"

// ------------------------------------------------------------------ NVFP4 quantize without allocation
// For callers that cannot allocate device memory or lend a workspace: the amax
// partials live in this fixed file-scope array instead.  Every GPU that loads
// the library holds it (4 KiB) until the process exits.  All calls on a device
// share it, so calls that overlap on the GPU race; each call overwrites every
// slot it reads, so nothing has to be cleared between calls.
namespace {

constexpr int kNoallocPartials = 1024;                   // scratch capacity (floats)
constexpr int64_t kNoallocMaxElems = (int64_t)1 << 30;   // largest rows * K this entry point takes
constexpr int kNoallocMaxDevices = 64;
// The amax pre-pass uses the same grid as nvfp4_quantize, never more CTAs
// (partials) than the array holds.
static_assert(nvq::kAmaxMaxBlocks <= kNoallocPartials, "amax partials must fit the fixed scratch");

static __device__ __align__(256) float g_noalloc_amax_partials[kNoallocPartials];

std::mutex g_noalloc_mutex;
float* g_noalloc_scratch[kNoallocMaxDevices] = {};

// Device address of the scratch array on the current device, resolved once per
// device (with that device current) and cached for the life of the process.
nvq_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "nvfp4_quantize_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kNoallocMaxDevices) return fail(NVQ_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: device ordinal >= 64");
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_scratch[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_amax_partials);
    if (e != cudaSuccess) return cuda_fail(e, "nvfp4_quantize_noalloc: cudaGetSymbolAddress");
    g_noalloc_scratch[dev] = static_cast<float*>(ptr);
  }
  *out = g_noalloc_scratch[dev];
  return NVQ_OK;
}

}  // namespace

extern "C" {

nvq_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t K, const float* tensor_scale_in,
                                  uint8_t* codes, uint8_t* scales, float* tensor_scale_out, void* stream_) {
  // The size limit comes first: an oversized call is rejected before any
  // pointer is looked at.
  if (rows > 0 && K > 0 && rows > kNoallocMaxElems / K)
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE,
                "nvfp4_quantize_noalloc: rows*K exceeds 2^30 elements, the largest tensor this entry point "
                "takes; use nvfp4_quantize with a workspace");
  nvq_status st = quantize_validate("nvfp4_quantize_noalloc", x_bf16, rows, K, codes, scales, tensor_scale_out);
  if (st != NVQ_OK) return st;
  int amax_blocks = 0;
  if (tensor_scale_in == nullptr && rows > 0) amax_blocks = amax_grid(rows, K);
  if (amax_blocks > kNoallocPartials)
    return fail(NVQ_ERR_UNSUPPORTED_SHAPE, "nvfp4_quantize_noalloc: amax partials exceed the fixed scratch");
  float* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != NVQ_OK) return st;
  return quantize_launch(x_bf16, rows, K, tensor_scale_in, codes, scales, tensor_scale_out, scratch, amax_blocks,
                         static_cast<cudaStream_t>(stream_));
}

}  // extern "C"
