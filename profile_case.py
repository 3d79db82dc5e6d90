"""Run one library call on one shape a few times, for profilers (ncu) and quick timing.

  python profile_case.py --op gemm --M 8192 --K 4096 --N 24576
  python profile_case.py --op w4a16 --M 1 --K 4096 --N 24576
  python profile_case.py --op quantize --M 8192 --K 12288 [--noalloc]
  python profile_case.py --op crossover --K 4096 --N 24576
  python profile_case.py --op streamed --M 8192 --layers 8
  python profile_case.py --op swiglu --M 8192 --K 4096 --N 24576
  python profile_case.py --op library_nvfp4 --M 8192 --K 4096 --N 24576

Inputs are drawn on the GPU from the seeded generators; the offline steps
(weight quantization and reorder) run once before the measured calls.  The
measured calls are captured in a CUDA graph and replayed once; prints the
mean CUDA-event time per call.  Inputs stay the same between calls, so small
weights can be served from L2 unless ``--copies`` cycles through more weight
bytes than L2 holds (126 MB).
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import phase_disaggregated_quantized_b200 as nvq  # noqa: E402
from phase_disaggregated_quantized_b200 import synth  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=("gemm", "w4a16", "quantize", "crossover", "streamed", "swiglu", "library_nvfp4"), required=True)
    ap.add_argument("--layers", type=int, default=8, help="streamed: transformer layers of 4 Qwen3-8B linears")
    ap.add_argument("--M", type=int, default=0)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=0)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--sparse", action="store_true", help="w4a16: the 2:4-sparse packed weights")
    ap.add_argument("--noalloc", action="store_true", help="quantize: through nvfp4_quantize_noalloc")
    ap.add_argument("--copies", type=int, default=1,
                    help="w4a16: cycle through this many weight copies (a total above L2 gives cold-cache reads)")
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if a.op == "crossover":
        return crossover(a, dev)
    if a.op == "streamed":
        return streamed(a, dev)
    if a.op == "swiglu":
        return swiglu(a, dev)
    if a.op == "library_nvfp4":
        return library_nvfp4(a, dev)
    x = synth.activations_cuda(a.M, a.K, seed=11, device=dev)
    if a.op == "gemm":
        w = synth.weights_cuda(a.N, a.K, seed=11, device=dev)
        wq = nvq.nvfp4_quantize(w)
        xq = nvq.nvfp4_quantize(x)
        y = torch.empty(a.M, a.N, dtype=torch.bfloat16, device=dev)
        run = lambda: nvq.nvfp4_gemm_w4a4(xq, wq, a.M, a.N, a.K, y=y)  # noqa: E731
        work = 2.0 * a.M * a.N * a.K
        unit = "TFLOP/s"
    elif a.op == "w4a16":
        w = synth.weights_cuda(a.N, a.K, seed=11, device=dev)
        codes, scales = nvq.int4_quantize(w)
        if a.sparse:
            packed = [nvq.int4_pack_sparse24(w, codes, scales) for _ in range(a.copies)]
        else:
            packed = [nvq.int4_pack_weights(codes, scales, a.N, a.K) for _ in range(a.copies)]
        y = torch.empty(a.M, a.N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, nvq.w4a16_workspace_bytes(a.M, a.N, a.K)), dtype=torch.uint8, device=dev)
        calls = [0]

        def run():
            pc, ps = packed[calls[0] % len(packed)]
            calls[0] += 1
            if a.sparse:
                nvq.w4a16_sparse24_gemm(x, pc, ps, a.N, y=y)
            else:
                nvq.w4a16_gemm(x, pc, ps, a.N, y=y, workspace=ws)
        wbytes = a.N * a.K * 3 / 8 if a.sparse else a.N * a.K / 2
        work = wbytes + 2 * a.N * a.K / 128 + 2 * a.M * a.K + 2 * a.M * a.N
        unit = "GB/s"
    else:
        codes = torch.empty(a.M, a.K // 2, dtype=torch.uint8, device=dev)
        sc = torch.empty(nvq.nvfp4_scales_bytes(a.M, a.K), dtype=torch.uint8, device=dev)
        t = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(nvq.nvfp4_quantize_workspace_bytes(a.M, a.K), dtype=torch.uint8, device=dev)
        if a.noalloc:                       # the entry point that keeps its scratch in the library
            run = lambda: nvq.nvfp4_quantize_noalloc(x, None, codes=codes, scales=sc, tensor_scale_out=t)  # noqa
        else:
            run = lambda: nvq.nvfp4_quantize(x, None, codes=codes, scales=sc, tensor_scale_out=t, workspace=ws)  # noqa
        work = 2.0 * a.M * a.K * 2 + a.M * a.K * (0.5 + 1 / 16)
        unit = "GB/s"
    run()                                   # first call sets kernel attributes
    torch.cuda.synchronize()
    # Time a captured graph of `iters` calls: no host launch overhead between them.
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(a.iters):
                run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        graph.replay()                      # warm
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    nvq.check_device_error()
    s = e0.elapsed_time(e1) / 1e3 / a.iters
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    print(f"{a.op} M={a.M} K={a.K} N={a.N}: {1e6 * s:.2f} us/call, {work / s / scale:.1f} {unit}")


def _graph_time(run, iters):
    """Mean seconds per call of `iters` calls captured in one CUDA graph (after a warm replay)."""
    run()
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(iters):
                run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        graph.replay()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    nvq.check_device_error()
    return e0.elapsed_time(e1) / 1e3 / iters


def library_nvfp4(a, dev):
    """Reference point, not part of the library: the same NVFP4 block-scaled GEMM
    (16-element blocks, E4M3 scales, bf16 output) through the vendor library
    (torch.nn.functional.scaled_mm, cuBLASLt), random codes, unit scales."""
    import torch.nn.functional as F
    M, K, N = a.M, a.K, a.N

    def rup(v, m):
        return (v + m - 1) // m * m
    g = torch.Generator(device=dev).manual_seed(11)
    xa = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
    wb = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
    one = 0x38                                                # E4M3 1.0
    sa = torch.full((rup(M, 128) * rup(K // 16, 4),), one, dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
    sb = torch.full((rup(N, 128) * rup(K // 16, 4),), one, dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)

    def run():
        return F.scaled_mm(xa, wb.t(), sa, F.ScalingType.BlockWise1x16, sb, F.ScalingType.BlockWise1x16,
                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                           output_dtype=torch.bfloat16)
    s = _graph_time(run, a.iters)
    print(f"library_nvfp4 M={M} K={K} N={N}: {1e6 * s:.2f} us/call, {2.0 * M * N * K / s / 1e12:.1f} TFLOP/s")


def crossover(a, dev):
    """Time both phase paths of one linear layer over a sweep of M (one BF16
    master weight quantized both ways): W4A16 (weights INT4 g128, activations
    BF16) against W4A4 (activations quantized to NVFP4 on the fly, then the
    block-scaled GEMM).  Weights are cycled through enough copies to come from
    HBM.  Prints one line per M and the largest M where W4A16 is faster."""
    K, N = a.K, a.N or 24576
    w = synth.weights_cuda(N, K, seed=5000, device=dev)
    wq = nvq.nvfp4_quantize(w)
    codes, scales = nvq.int4_quantize(w)
    copies = max(1, -(-400_000_000 // (N * K // 2)))
    packed = [nvq.int4_pack_weights(codes, scales, N, K) for _ in range(copies)]
    fp4 = [wq] + [tuple(t.clone() for t in wq) for _ in range(copies - 1)]
    del w
    last_w4a16 = 0
    rows = []
    for M in (1, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 8192, 32768):
        x = synth.activations_cuda(M, K, seed=5001, device=dev)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        xc = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        xs = torch.empty(max(1, nvq.nvfp4_scales_bytes(M, K)), dtype=torch.uint8, device=dev)
        tx = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(max(16, nvq.nvfp4_quantize_workspace_bytes(M, K)), dtype=torch.uint8, device=dev)
        k = [0]

        def w4a16():
            pc, ps = packed[k[0] % copies]
            k[0] += 1
            nvq.w4a16_gemm(x, pc, ps, N, y=y)

        def w4a4():
            wk = fp4[k[0] % copies]
            k[0] += 1
            nvq.nvfp4_quantize(x, None, codes=xc, scales=xs, tensor_scale_out=tx, workspace=ws)
            nvq.nvfp4_gemm_w4a4((xc, xs, tx), wk, M, N, K, y=y)

        iters = 8 if M <= 2048 else 3
        t16 = _graph_time(w4a16, iters) if M <= 8192 else float("inf")
        t4 = _graph_time(w4a4, iters)
        if t16 < t4:
            last_w4a16 = M
        rows.append((M, t16, t4))
        print(f"M={M:6d}  w4a16 {1e6 * t16:10.2f} us   w4a4+quantize {1e6 * t4:10.2f} us   "
              f"faster: {'w4a16' if t16 < t4 else 'w4a4'}", flush=True)
    print(f"crossover: W4A16 faster up to M = {last_w4a16} (K={K}, N={N})")
    return rows


def streamed(a, dev):
    """Prefill over `layers` transformer layers (the four Qwen3-8B linears each)
    with NVFP4 weights in pinned host memory: time the resident-weight pass,
    the host->device copies alone, and nvq_prefill_streamed with the copies on
    their own stream and on the compute stream."""
    M = a.M or 8192
    shapes = [(K, N) for _, K, N in synth.QWEN3_8B_LINEARS]
    xs = {K: synth.activations_cuda(M, K, seed=6000 + K, device=dev) for K, _ in shapes}
    ys = {(K, N): torch.empty(M, N, dtype=torch.bfloat16, device=dev) for K, N in shapes}
    layers, resident, wbytes = [], [], 0
    for li in range(a.layers):
        for i, (K, N) in enumerate(shapes):
            w = synth.weights_cuda(N, K, seed=7000 + 10 * li + i, device=dev)
            wq = nvq.nvfp4_quantize(w)
            del w
            host = tuple(t.cpu().pin_memory() for t in wq)
            wbytes += sum(t.numel() * t.element_size() for t in host)
            layers.append(dict(w_host=host, x=xs[K], y=ys[(K, N)], N=N, K=K))
            resident.append(wq)
    torch.cuda.synchronize()
    compute, copy = torch.cuda.current_stream(), torch.cuda.Stream()
    ws = torch.empty(max(16, nvq.prefill_streamed_workspace_bytes(layers, M)), dtype=torch.uint8, device=dev)
    dev_w = torch.empty(max(t.numel() * t.element_size() for L in layers for t in L["w_host"]), dtype=torch.uint8,
                        device=dev)

    def timed(fn, reps=3):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(compute)
        for _ in range(reps):
            fn()
        copy_done = torch.cuda.Event()
        copy_done.record(copy)
        compute.wait_event(copy_done)
        e1.record(compute)
        torch.cuda.synchronize()
        nvq.check_device_error()
        return e0.elapsed_time(e1) / 1e3 / reps

    def run_resident():
        for L, wq in zip(layers, resident):
            nvq.nvfp4_gemm_w4a4(nvq.nvfp4_quantize(L["x"]), wq, M, L["N"], L["K"], y=L["y"])

    def run_copies():
        copy.wait_stream(compute)
        with torch.cuda.stream(copy):
            for L in layers:
                for t in L["w_host"]:
                    dev_w[: t.numel() * t.element_size()].copy_(t.view(torch.uint8).view(-1), non_blocking=True)

    def run_streamed():
        nvq.prefill_streamed(layers, M, workspace=ws, compute_stream=compute, copy_stream=copy)

    def run_serial():
        nvq.prefill_streamed(layers, M, workspace=ws, compute_stream=compute, copy_stream=compute)

    t_res = timed(run_resident)
    t_copy = timed(run_copies)
    t_str = timed(run_streamed)
    t_ser = timed(run_serial)
    flops = sum(2.0 * M * L["N"] * L["K"] for L in layers)
    hidden = (t_res + t_copy - t_str) / min(t_res, t_copy)
    print(f"M={M} layers={a.layers} linears={len(layers)} weights={wbytes / 1e6:.0f} MB (pinned host)")
    print(f"resident weights : {1e3 * t_res:8.3f} ms  ({flops / t_res / 1e12:.0f} TFLOP/s)")
    print(f"copies alone     : {1e3 * t_copy:8.3f} ms  ({wbytes / t_copy / 1e9:.1f} GB/s host->device)")
    print(f"streamed, 2 strm : {1e3 * t_str:8.3f} ms  (bound max(resident, copies) = {1e3 * max(t_res, t_copy):.3f} ms)")
    print(f"streamed, 1 strm : {1e3 * t_ser:8.3f} ms  (no overlap)")
    print(f"overlap: {100 * hidden:.0f}% of the shorter of compute / copy hidden")


def swiglu(a, dev):
    """gate_up GEMM with the SiLU * mul -> NVFP4 epilogue against the same GEMM
    writing BF16 and against the unfused chain (BF16 GEMM, then silu * mul by
    torch, then nvfp4_quantize of H with the same static scale)."""
    M, K, N = a.M or 8192, a.K, a.N or 24576
    I = N // 2
    x = synth.activations_cuda(M, K, seed=8000, device=dev)
    wg = synth.weights_cuda(I, K, seed=8001, device=dev)
    wu = synth.weights_cuda(I, K, seed=8002, device=dev)
    wi = nvq.interleave_gate_up(wg, wu).contiguous()
    wc = torch.cat([wg, wu])                                   # gate rows, then up rows (plain layout)
    del wg, wu
    xq, wqi, wqc = nvq.nvfp4_quantize(x), nvq.nvfp4_quantize(wi), nvq.nvfp4_quantize(wc)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    t_h = torch.tensor([0.02], dtype=torch.float32, device=dev)
    hc = torch.empty(M, I // 2, dtype=torch.uint8, device=dev)
    hs = torch.empty(nvq.nvfp4_scales_bytes(M, I), dtype=torch.uint8, device=dev)
    ht = torch.empty(1, dtype=torch.float32, device=dev)

    def fused():
        nvq.nvfp4_gemm_w4a4_swiglu(xq, wqi, M, N, K, t_h, h_codes=hc, h_scales=hs)

    def plain():
        nvq.nvfp4_gemm_w4a4(xq, wqc, M, N, K, y=y)

    def unfused():
        nvq.nvfp4_gemm_w4a4(xq, wqc, M, N, K, y=y)
        h = torch.nn.functional.silu(y[:, :I]) * y[:, I:]
        nvq.nvfp4_quantize(h, t_h, codes=hc, scales=hs, tensor_scale_out=ht)

    flops = 2.0 * M * N * K
    tf, tp, tu = _graph_time(fused, 5), _graph_time(plain, 5), _graph_time(unfused, 5)
    print(f"M={M} K={K} N={N} (I={I})")
    print(f"fused SiLU*mul -> NVFP4 epilogue : {1e6 * tf:9.1f} us  {flops / tf / 1e12:7.0f} TFLOP/s")
    print(f"same GEMM, BF16 output           : {1e6 * tp:9.1f} us  {flops / tp / 1e12:7.0f} TFLOP/s")
    print(f"unfused: BF16 GEMM + silu*mul + quantize : {1e6 * tu:9.1f} us")
    print(f"H bytes written: fused {M * I // 2 + M * I // 16} vs BF16 Y {2 * M * N}")


if __name__ == "__main__":
    main()
