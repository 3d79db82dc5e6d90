"""Phase-specialised quantized linear layers for B200 (sm_100a).

Thin Python binding of the C-ABI library ``libnvq.so`` (declared in
``include/nvq.h``).  Every function here only marshals arguments: it allocates
outputs with torch when the caller does not pass them, takes device pointers,
and calls the library entry point of the same name on the current CUDA stream.
All arithmetic runs in the library's CUDA kernels.  There is no CPU fallback:
if the library or a GPU is missing, the calls raise.

Prefill (Mix-Quant page, gist.science, section 2): ``nvfp4_quantize`` then
``nvfp4_gemm_w4a4``.  Decode (MARLIN page, abeam.tech): ``int4_quantize`` and
``int4_pack_weights`` offline, then ``w4a16_gemm``.  ``nvq_linear`` picks one
of the two by the batch size M (Disaggregated Quantization page,
singularity-lens.com: one master weight kept in both formats).
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "nvq.h")

_lib = None

STATUS = {0: "NVQ_OK", 1: "NVQ_ERR_INVALID_ARG", 2: "NVQ_ERR_UNSUPPORTED_SHAPE", 3: "NVQ_ERR_MISALIGNED",
          4: "NVQ_ERR_WORKSPACE", 5: "NVQ_ERR_CUDA", 6: "NVQ_ERR_DEVICE_TIMEOUT"}


class StreamLayer(ctypes.Structure):
    """nvq_stream_layer of include/nvq.h."""
    _fields_ = [("w_codes_host", ctypes.c_void_p), ("w_scales_host", ctypes.c_void_p),
                ("w_t_host", ctypes.c_void_p), ("x_bf16", ctypes.c_void_p), ("y_bf16", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class NvqError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} {detail}".rstrip())


def header_functions() -> list[str]:
    """Names of the functions declared in include/nvq.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+([a-z][a-z0-9_]*)\s*\(", text, flags=re.M)


def lib() -> ctypes.CDLL:
    """Load libnvq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libnvq.so not built at {LIB_PATH}; run "
                               "`python -m phase_disaggregated_quantized_b200.build_lib`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        sig = {
            "nvq_abi_version": ([], i32),
            "nvq_status_string": ([i32], ctypes.c_char_p),
            "nvq_last_error_detail": ([], ctypes.c_char_p),
            "nvq_check_device_error": ([vp], i32),
            "nvq_selftest_wait_timeout": ([ctypes.c_uint64, vp], i32),
            "nvfp4_scales_bytes": ([i64, i64], sz),
            "nvfp4_scale_offset": ([i64, i64, i64, i64], i64),
            "nvq_workspace_bytes": ([i32, i64, i64, i64], sz),
            "nvfp4_quantize_workspace_bytes": ([i64, i64], sz),
            "nvfp4_quantize": ([vp, i64, i64, vp, vp, vp, vp, vp, sz, vp], i32),
            "nvfp4_quantize_noalloc": ([vp, i64, i64, vp, vp, vp, vp, vp], i32),
            "nvfp4_amax": ([vp, i64, i64, vp, vp, sz, vp], i32),
            "nvfp4_scale_from_amax": ([vp, vp, vp], i32),
            "nvfp4_gemm_w4a4": ([vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, vp], i32),
            "nvfp4_gemm_w4a4_swiglu": ([vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, vp], i32),
            "int4_quantize": ([vp, i64, i64, vp, vp, vp], i32),
            "int4_pack_weights": ([vp, vp, i64, i64, vp, vp, vp], i32),
            "w4a16_workspace_bytes": ([i64, i64, i64], sz),
            "w4a16_gemm": ([vp, vp, vp, vp, i64, i64, i64, vp, sz, vp], i32),
            "int4_pack_sparse24": ([vp, vp, vp, i64, i64, vp, vp, vp], i32),
            "w4a16_sparse24_gemm": ([vp, vp, vp, vp, i64, i64, i64, vp], i32),
            "nvq_default_crossover_m": ([], i64),
            "nvq_linear_workspace_bytes": ([i64, i64, i64, i64], sz),
            "nvq_linear": ([vp, i64, i64, i64, vp, vp, vp, vp, vp, i64, vp, vp, sz, vp], i32),
            "nvq_prefill_streamed_workspace_bytes": ([ctypes.POINTER(StreamLayer), i32, i64], sz),
            "nvq_prefill_streamed": ([ctypes.POINTER(StreamLayer), i32, i64, vp, sz, vp, vp], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes, fn.restype = args, res
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise NvqError(status, where, lib().nvq_last_error_detail().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libnvq calls take CUDA tensors")


def nvfp4_scales_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_scales_bytes(rows, K))


NVQ_OP_NVFP4_QUANTIZE, NVQ_OP_NVFP4_GEMM, NVQ_OP_W4A16_GEMM, NVQ_OP_LINEAR = 0, 1, 2, 3


def nvfp4_scale_offset(row: int, kblock: int, rows: int, K: int) -> int:
    """Byte offset of the scale of (row, 16-element block) in the tiled scales of a [rows, K] tensor (-1: out of range)."""
    return int(lib().nvfp4_scale_offset(row, kblock, rows, K))


def nvq_workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return int(lib().nvq_workspace_bytes(op, M, N, K))


def nvfp4_quantize_workspace_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_quantize_workspace_bytes(rows, K))


def w4a16_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().w4a16_workspace_bytes(M, N, K))


def check_device_error(stream=None):
    _check(lib().nvq_check_device_error(_stream(stream)), "nvq_check_device_error")


def selftest_wait_timeout(limit_ns: int, stream=None):
    """Launch the library's timeout diagnostic (one bounded wait that runs out)."""
    _check(lib().nvq_selftest_wait_timeout(limit_ns, _stream(stream)), "nvq_selftest_wait_timeout")


def nvfp4_quantize(x, tensor_scale_in=None, *, codes=None, scales=None, tensor_scale_out=None, workspace=None,
                   stream=None):
    """BF16 [rows, K] -> (codes uint8 [rows, K/2], tiled scales uint8, t float32 [1])."""
    _need_cuda(x, tensor_scale_in)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    rows, K = x.shape
    dev = x.device
    if codes is None:
        codes = torch.empty(rows, K // 2, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(max(1, nvfp4_scales_bytes(rows, K)), dtype=torch.uint8, device=dev)
    if tensor_scale_out is None:
        tensor_scale_out = torch.empty(1, dtype=torch.float32, device=dev)
    need = nvfp4_quantize_workspace_bytes(rows, K) if tensor_scale_in is None else 0
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().nvfp4_quantize(_ptr(x), rows, K, _ptr(tensor_scale_in), _ptr(codes), _ptr(scales),
                                _ptr(tensor_scale_out), _ptr(workspace), ws_bytes, _stream(stream)),
           "nvfp4_quantize")
    return codes, scales, tensor_scale_out


def nvfp4_amax(x, *, amax_out=None, workspace=None, stream=None):
    """max |x| of a BF16 [rows, K] tensor -> float32 [1] on the device (0 for rows == 0)."""
    _need_cuda(x, amax_out, workspace)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    rows, K = x.shape
    if amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=x.device)
    need = nvfp4_quantize_workspace_bytes(rows, K)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().nvfp4_amax(_ptr(x), rows, K, _ptr(amax_out), _ptr(workspace), ws_bytes, _stream(stream)),
           "nvfp4_amax")
    return amax_out


def nvfp4_scale_from_amax(amax, *, tensor_scale_out=None, stream=None):
    """t of a tensor whose max |x| is amax (float32 [1] on the device) -> float32 [1]."""
    _need_cuda(amax, tensor_scale_out)
    if tensor_scale_out is None:
        tensor_scale_out = torch.empty(1, dtype=torch.float32, device=amax.device)
    _check(lib().nvfp4_scale_from_amax(_ptr(amax), _ptr(tensor_scale_out), _stream(stream)),
           "nvfp4_scale_from_amax")
    return tensor_scale_out


def nvfp4_quantize_row_shard(x, group=None, *, codes=None, scales=None, stream=None):
    """NVFP4-quantize this rank's rows of one tensor whose rows are split over
    the ranks of a torch.distributed group, with the tensor scale of the whole
    tensor: local max |x| (nvfp4_amax), a 4-byte all-reduce(MAX) over the group,
    t from the result (nvfp4_scale_from_amax), then nvfp4_quantize with that t.
    Returns (codes, scales, t) as nvfp4_quantize does."""
    import torch.distributed as dist
    amax = nvfp4_amax(x, stream=stream)
    if stream is None:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    else:
        with torch.cuda.stream(stream):
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    t = nvfp4_scale_from_amax(amax, stream=stream)
    return nvfp4_quantize(x, t, codes=codes, scales=scales, stream=stream)


def nvfp4_quantize_noalloc(x, tensor_scale_in=None, *, codes, scales, tensor_scale_out, stream=None):
    """nvfp4_quantize for callers that cannot allocate: the library uses its own
    fixed device scratch (rows * K <= 2^30), so all outputs must be passed in."""
    _need_cuda(x, tensor_scale_in, codes, scales, tensor_scale_out)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    rows, K = x.shape
    _check(lib().nvfp4_quantize_noalloc(_ptr(x), rows, K, _ptr(tensor_scale_in), _ptr(codes), _ptr(scales),
                                        _ptr(tensor_scale_out), _stream(stream)), "nvfp4_quantize_noalloc")
    return codes, scales, tensor_scale_out


def nvfp4_gemm_w4a4(xq, wq, M: int, N: int, K: int, *, y=None, stream=None):
    """Y [M, N] bf16 = dequant(xq) @ dequant(wq)^T; xq / wq are (codes, scales, t)."""
    xc, xs, tx = xq
    wc, ws, tw = wq
    _need_cuda(xc, xs, tx, wc, ws, tw)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=xc.device)
    _check(lib().nvfp4_gemm_w4a4(_ptr(xc), _ptr(xs), _ptr(tx), _ptr(wc), _ptr(ws), _ptr(tw), _ptr(y), M, N, K,
                                 _stream(stream)), "nvfp4_gemm_w4a4")
    return y


def interleave_gate_up(w_gate, w_up):
    """[I, K] gate and up weights -> [2I, K] with rows interleaved in blocks of
    128 (gate block b, then up block b), the order nvfp4_gemm_w4a4_swiglu reads."""
    I, K = w_gate.shape
    assert w_up.shape == (I, K) and I % 128 == 0
    return torch.stack([w_gate.view(I // 128, 128, K), w_up.view(I // 128, 128, K)], dim=1).reshape(2 * I, K)


def nvfp4_gemm_w4a4_swiglu(xq, wq, M: int, N: int, K: int, t_h, *, h_codes=None, h_scales=None, stream=None):
    """NVFP4 H = silu(gate) * up of the gate_up GEMM (weight rows interleaved by
    interleave_gate_up), quantized with the static tensor scale t_h (device
    float tensor [1]).  Returns (h_codes [M, N/4] uint8, h_scales, t_h)."""
    xc, xs, tx = xq
    wc, ws, tw = wq
    _need_cuda(xc, xs, tx, wc, ws, tw, t_h)
    I = N // 2
    if h_codes is None:
        h_codes = torch.empty(M, I // 2, dtype=torch.uint8, device=xc.device)
    if h_scales is None:
        h_scales = torch.empty(max(1, nvfp4_scales_bytes(M, I)), dtype=torch.uint8, device=xc.device)
    _check(lib().nvfp4_gemm_w4a4_swiglu(_ptr(xc), _ptr(xs), _ptr(tx), _ptr(wc), _ptr(ws), _ptr(tw), _ptr(t_h),
                                        _ptr(h_codes), _ptr(h_scales), M, N, K, _stream(stream)),
           "nvfp4_gemm_w4a4_swiglu")
    return h_codes, h_scales, t_h


def int4_quantize(w, *, codes=None, scales=None, stream=None):
    """BF16 [N, K] -> (codes uint8 [N, K/2], scales bf16 [N, K/128])."""
    _need_cuda(w)
    assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.is_contiguous()
    N, K = w.shape
    if codes is None:
        codes = torch.empty(N, K // 2, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(N, K // 128, dtype=torch.bfloat16, device=w.device)
    _check(lib().int4_quantize(_ptr(w), N, K, _ptr(codes), _ptr(scales), _stream(stream)), "int4_quantize")
    return codes, scales


def int4_pack_weights(codes, scales, N: int, K: int, *, packed_codes=None, packed_scales=None, stream=None):
    """Offline reorder into the decode kernel's fragment order."""
    _need_cuda(codes, scales)
    if packed_codes is None:
        packed_codes = torch.empty(N * K // 2, dtype=torch.uint8, device=codes.device)
    if packed_scales is None:
        packed_scales = torch.empty(N * (K // 128) * 2, dtype=torch.uint8, device=codes.device)
    _check(lib().int4_pack_weights(_ptr(codes), _ptr(scales), N, K, _ptr(packed_codes), _ptr(packed_scales),
                                   _stream(stream)), "int4_pack_weights")
    return packed_codes, packed_scales


def w4a16_gemm(x, packed_codes, packed_scales, N: int, *, y=None, workspace=None, stream=None):
    """BF16 X [M, K] times packed INT4 W [N, K] -> Y [M, N] bf16."""
    _need_cuda(x, packed_codes, packed_scales)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    M, K = x.shape
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    need = w4a16_workspace_bytes(M, N, K)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().w4a16_gemm(_ptr(x), _ptr(packed_codes), _ptr(packed_scales), _ptr(y), M, N, K, _ptr(workspace),
                            ws_bytes, _stream(stream)), "w4a16_gemm")
    return y


def int4_pack_sparse24(w, codes, scales, *, packed=None, packed_scales=None, stream=None):
    """2:4-prune the BF16 master w [N, K] and pack its kept INT4 codes (from
    int4_quantize(w)) for w4a16_sparse24_gemm."""
    _need_cuda(w, codes, scales)
    N, K = w.shape
    if packed is None:
        packed = torch.empty(N * K * 3 // 8, dtype=torch.uint8, device=w.device)
    if packed_scales is None:
        packed_scales = torch.empty(N * (K // 128) * 2, dtype=torch.uint8, device=w.device)
    _check(lib().int4_pack_sparse24(_ptr(w), _ptr(codes), _ptr(scales), N, K, _ptr(packed), _ptr(packed_scales),
                                    _stream(stream)), "int4_pack_sparse24")
    return packed, packed_scales


def w4a16_sparse24_gemm(x, packed, packed_scales, N: int, *, y=None, stream=None):
    """BF16 X [M, K] times the 2:4-sparse packed INT4 W [N, K] -> Y [M, N] bf16."""
    _need_cuda(x, packed, packed_scales)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    M, K = x.shape
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _check(lib().w4a16_sparse24_gemm(_ptr(x), _ptr(packed), _ptr(packed_scales), _ptr(y), M, N, K, _stream(stream)),
           "w4a16_sparse24_gemm")
    return y


def default_crossover_m() -> int:
    """Largest M served by the W4A16 path when nvq_linear is given crossover < 0."""
    return int(lib().nvq_default_crossover_m())


def nvq_linear_workspace_bytes(M: int, N: int, K: int, crossover_m: int = -1) -> int:
    return int(lib().nvq_linear_workspace_bytes(M, N, K, crossover_m))


def nvq_linear(x, w4a4=None, w4a16=None, N: int | None = None, *, crossover_m: int = -1, y=None, workspace=None,
               stream=None):
    """Y [M, N] bf16 = X W^T through the path nvq_linear picks for this M.

    w4a4: (codes, scales, t) of the NVFP4 master; w4a16: (packed_codes,
    packed_scales) of the INT4 master; pass the form(s) the chosen path reads."""
    _need_cuda(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_contiguous()
    M, K = x.shape
    if N is None:
        raise ValueError("N is required")
    wc, wsc, wt = (None, None, None) if w4a4 is None else w4a4
    pc, ps = (None, None) if w4a16 is None else w4a16
    _need_cuda(wc, wsc, wt, pc, ps)
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    need = nvq_linear_workspace_bytes(M, N, K, crossover_m)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().nvq_linear(_ptr(x), M, N, K, _ptr(wc), _ptr(wsc), _ptr(wt), _ptr(pc), _ptr(ps), crossover_m,
                            _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)), "nvq_linear")
    return y


def _stream_layers(layers):
    arr = (StreamLayer * len(layers))()
    for i, L in enumerate(layers):
        wc, ws, wt = L["w_host"]
        for t in (wc, ws, wt):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("streamed weights must be pinned host tensors")
        _need_cuda(L["x"], L["y"])
        arr[i] = StreamLayer(wc.data_ptr(), ws.data_ptr(), wt.data_ptr(), L["x"].data_ptr(), L["y"].data_ptr(),
                             L["N"], L["K"])
    return arr


def prefill_streamed_workspace_bytes(layers, M: int) -> int:
    return int(lib().nvq_prefill_streamed_workspace_bytes(_stream_layers(layers), len(layers), M))


def prefill_streamed(layers, M: int, *, workspace=None, compute_stream=None, copy_stream=None):
    """Run quantize + W4A4 GEMM for each layer with its NVFP4 weights copied from
    pinned host memory into two device slots, copies overlapping the GEMMs.

    layers: list of dicts with "w_host" (codes, scales, t as pinned CPU tensors
    from nvfp4_quantize), "x" (device [M, K] bf16), "y" (device [M, N] bf16),
    "N", "K".  Enqueues only; synchronise compute_stream before reading y."""
    arr = _stream_layers(layers)
    need = int(lib().nvq_prefill_streamed_workspace_bytes(arr, len(layers), M))
    if workspace is None:
        workspace = torch.empty(max(16, need), dtype=torch.uint8, device=layers[0]["x"].device)
    if compute_stream is None:
        compute_stream = torch.cuda.current_stream()
    if copy_stream is None:
        copy_stream = compute_stream
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().nvq_prefill_streamed(arr, len(layers), M, _ptr(workspace), ws_bytes,
                                      ctypes.c_void_p(compute_stream.cuda_stream),
                                      ctypes.c_void_p(copy_stream.cuda_stream)), "nvq_prefill_streamed")
    return workspace
