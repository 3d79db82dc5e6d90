"""Benchmark of the phase-specialised quantized linear layers on B200.

One step = one pass of the hot path over one batch of synthetic input:
  prefill  Qwen3-8B-shaped linears at M = 8192 tokens, each layer
           amax + NVFP4 RTN quantize of the BF16 activations, then the W4A4
           block-scaled GEMM against NVFP4 weights quantized offline;
  decode   the same four (K, N) shapes as INT4 g128 weight-only GEMMs at batch
           M in {1, 4, 8, 16, 32} (weights quantized and reordered offline).
The headline `value` is prefill GEMM TFLOP/s over the whole prefill pass
(quantization included); the `decode` object holds the INT4 decode GB/s.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs the same per-rank workload (independent prefill
requests and decode batches; weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 prefill GEMM TFLOPS; INT4 W-only decode GB/s; both as % of B200 roofline"
LINEARS = (("qkv_proj", 4096, 6144), ("o_proj", 4096, 4096), ("gate_up_proj", 4096, 24576),
           ("down_proj", 12288, 4096))
PREFILL_M = 8192
DECODE_BATCHES = (1, 4, 8, 16, 32)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0     # nominal dense ratio: 9 PF NVFP4 / 2.25 PF BF16


def rank_seed(base: int, layer: int, rank: int) -> int:
    """Seed of one layer's synthetic input on one rank: every rank draws its own
    batch, so N ranks process N independent workloads (weak scaling)."""
    return base + 10 * layer + 100000 * rank


def max_over_ranks(torch, dist, values, device):
    """Element-wise maximum of per-rank timings over the process group (the job
    takes as long as its slowest rank); a no-op without a multi-rank group."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Units processed by all ranks together per second of the slowest rank."""
    return world * units_per_rank / seconds


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(name: str) -> str:
    p = os.path.join(ROOT, "phase_disaggregated_quantized_b200", "csrc", name)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def profiled_traffic(summary: str, source: str):
    """DRAM bytes per launch from a committed ncu summary, if it still matches the source."""
    p = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(p):
        return None
    want = kernel_source_hash(source)
    vals = {}
    for line in open(p):
        if line.startswith("traffic_"):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("traffic_source_hash") != want:
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id is not None:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_smi_id(torch, dev: int):
    try:
        bus = torch.cuda.get_device_properties(dev).pci_bus_id
        out = subprocess.run(["nvidia-smi", "--query-gpu=index,pci.bus_id", "--format=csv,noheader"],
                             capture_output=True, text=True, timeout=20).stdout
        for line in out.strip().splitlines():
            idx, pci = [p.strip() for p in line.split(",")]
            if pci.lower().endswith(bus.lower()[-12:]) or bus.lower().endswith(pci.lower()[-12:]):
                return idx
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[dev]
    return str(dev)


# ------------------------------------------------------------------ CPU oracle baseline
def oracle_sample_step(x_rows: int = 64, w_rows: int = 256, seed_base: int = 2000):
    """One bounded step of the CPU oracle on the prefill workload: per layer, a
    sample of `x_rows` activation rows and `w_rows` weight rows (each sample
    quantized as its own tensor), NVFP4 RTN quantization, exact dequantization
    and the float64 GEMM.  Returns (GEMM flops of the sample, seconds)."""
    from oracle import nvfp4 as onv
    from phase_disaggregated_quantized_b200 import synth
    import torch
    flops = 0.0
    t0 = time.perf_counter()
    for i, (name, K, N) in enumerate(LINEARS):
        seed = seed_base + 10 * i
        x = synth.activations(x_rows, K, seed=seed)          # a row sample of the layer input
        w = synth.weights(w_rows, K, seed=seed)
        xf = onv.bf16_bits_to_f64(x.view(torch.int16).numpy().view(np.uint16))
        wf = onv.bf16_bits_to_f64(w.view(torch.int16).numpy().view(np.uint16))
        xc, xs, tx = onv.quantize(xf)
        wc, ws, tw = onv.quantize(wf)
        onv.gemm_ref(onv.dequantize(xc, xs, tx), onv.dequantize(wc, ws, tw))
        flops += 2.0 * x_rows * w_rows * K
    return flops, time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline(budget_s: float = 15.0):
    flops, secs = 0.0, 0.0
    n = 0
    while secs < budget_s and n < 50:
        f, s = oracle_sample_step()
        flops += f
        secs += s
        n += 1
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} oracle steps; each: 4 Qwen3-8B linears, 64 activation rows x 256 weight rows, "
                      f"NVFP4 RTN quantize + exact dequant + float64 GEMM ({secs:.1f} s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample_step()
    flops, secs = 0.0, 0.0
    for _ in range(args.steps):
        f, s = oracle_sample_step()
        flops += f
        secs += s
    value = flops / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "Qwen3-8B prefill linears (row sample), CPU oracle",
                       "seq_len": PREFILL_M, "linears": [list(l) for l in LINEARS]},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": "each step: 4 Qwen3-8B linears, 64 activation rows x 256 weight rows"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def run_gpu(args):
    import torch
    import torch.distributed as dist
    import phase_disaggregated_quantized_b200 as nvq
    from phase_disaggregated_quantized_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    nvq.lib()
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    # ---------------- prefill buffers (weights quantized offline, untimed)
    pre = []
    for i, (name, K, N) in enumerate(LINEARS):
        seed = rank_seed(2000, i, rank)
        x = synth.activations_cuda(PREFILL_M, K, seed, device=dev)
        w = synth.weights_cuda(N, K, seed, device=dev)
        wq = nvq.nvfp4_quantize(w)
        M = PREFILL_M
        pre.append(dict(name=name, K=K, N=N, x=x, wq=wq,
                        xc=torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
                        xs=torch.empty(nvq.nvfp4_scales_bytes(M, K), dtype=torch.uint8, device=dev),
                        tx=torch.empty(1, dtype=torch.float32, device=dev),
                        ws=torch.empty(nvq.nvfp4_quantize_workspace_bytes(M, K), dtype=torch.uint8, device=dev),
                        y=torch.empty(M, N, dtype=torch.bfloat16, device=dev)))
        del w
    # ---------------- decode buffers: one weight copy per batch size (no L2 reuse across uses)
    dec_w = []
    for c in range(len(DECODE_BATCHES)):
        layer = []
        for i, (name, K, N) in enumerate(LINEARS):
            w = synth.weights_cuda(N, K, 3000 + 10 * i + c, device=dev)
            codes, scales = nvq.int4_quantize(w)
            pc, ps = nvq.int4_pack_weights(codes, scales, N, K)
            layer.append((pc, ps))
            del w, codes, scales
        dec_w.append(layer)
    dec = []
    for mi, M in enumerate(DECODE_BATCHES):
        for i, (name, K, N) in enumerate(LINEARS):
            x = synth.activations_cuda(M, K, rank_seed(4000 + M, i, rank), device=dev)
            wsb = nvq.w4a16_workspace_bytes(M, N, K)
            dec.append(dict(M=M, K=K, N=N, layer=i, x=x, pc=dec_w[mi][i][0], ps=dec_w[mi][i][1],
                            y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                            ws=torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)))
    torch.cuda.synchronize()

    # external=True: the records become timestamp nodes of the captured graph
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    q_ev = [(ev(), ev()) for _ in pre]
    g_ev = [(ev(), ev()) for _ in pre]
    # Decode is timed as two contiguous blocks (M <= 16, then M = 32): an event
    # node between kernels ends programmatic dependent launch there, so timing
    # each batch size separately would serialise calls a decode loop runs back
    # to back.  Per-batch figures come from separate graphs (per_batch_decode).
    d_ev = [(ev(), ev()), (ev(), ev())]
    pre_ev = (ev(), ev())

    def step():
        pre_ev[0].record(stream)
        for L, (qa, qb), (ga, gb) in zip(pre, q_ev, g_ev):
            qa.record(stream)
            nvq.nvfp4_quantize(L["x"], None, codes=L["xc"], scales=L["xs"], tensor_scale_out=L["tx"],
                               workspace=L["ws"], stream=stream)
            qb.record(stream)
            ga.record(stream)
            nvq.nvfp4_gemm_w4a4((L["xc"], L["xs"], L["tx"]), L["wq"], PREFILL_M, L["N"], L["K"], y=L["y"],
                                stream=stream)
            gb.record(stream)
        pre_ev[1].record(stream)
        for blk, (da, db) in enumerate(d_ev):
            da.record(stream)
            for D in dec:
                if (D["M"] <= 16) == (blk == 0):
                    nvq.w4a16_gemm(D["x"], D["pc"], D["ps"], D["N"], y=D["y"], workspace=D["ws"], stream=stream)
            db.record(stream)

    launches_per_step = 3 * len(pre) + len(dec)
    step()                                  # first calls set kernel attributes outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    smi_id = gpu_smi_id(torch, local)
    t_start, t_end = ev(), ev()
    q_ms = [0.0] * len(pre)
    g_ms = [0.0] * len(pre)
    d_ms = [0.0] * len(d_ev)
    pre_ms = 0.0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(smi_id) as clocks:
        t_start.record(stream)
        for _ in range(args.steps):
            graph.replay()
            stream.synchronize()                # read this replay's kernel events
            pre_ms += pre_ev[0].elapsed_time(pre_ev[1])
            for j in range(len(pre)):
                q_ms[j] += q_ev[j][0].elapsed_time(q_ev[j][1])
                g_ms[j] += g_ev[j][0].elapsed_time(g_ev[j][1])
            for j in range(len(d_ev)):
                d_ms[j] += d_ev[j][0].elapsed_time(d_ev[j][1])
        t_end.record(stream)
        torch.cuda.synchronize()
    total_ms = t_start.elapsed_time(t_end)
    if world > 1:
        dist.barrier()
    nvq.check_device_error(stream)

    K_steps = args.steps
    gemm_flops = sum(2.0 * PREFILL_M * L["N"] * L["K"] for L in pre)
    pre_s = pre_ms / 1e3 / K_steps
    gemm_s = sum(g_ms) / 1e3 / K_steps
    quant_s = sum(q_ms) / 1e3 / K_steps

    def dec_bytes(D):
        M, K, N = D["M"], D["K"], D["N"]
        return N * K / 2 + 2 * N * K / 128 + 2 * M * K + 2 * M * N

    dec_b = sum(dec_bytes(D) for D in dec if D["M"] <= 16)
    dec_s = d_ms[0] / 1e3 / K_steps
    per_batch = per_batch_decode(torch, nvq, dec, dec_w, stream, dec_bytes)

    peaks, peaks_kind = load_peaks()
    fp4_peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * FP4_OVER_BF16
    fp4_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP4_OVER_BF16
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    # max over ranks of the step time and of the per-kernel sums
    total_ms, pre_s, gemm_s, dec_s = max_over_ranks(torch, dist if world > 1 else None,
                                                    [total_ms, pre_s, gemm_s, dec_s], dev)
    gemm_tflops = gemm_flops / gemm_s / 1e12          # per GPU (slowest rank): the kernel's roofline
    value = whole_job_rate(gemm_flops, world, pre_s) / 1e12

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if rank == 0 or world > 1:
        e2e = measure_e2e(torch, nvq, pre, stream, steps=max(2, min(args.steps, 5)))
    if world > 1:
        e2e["seconds"] = max_over_ranks(torch, dist, [e2e["seconds"]], dev)[0]

    if rank == 0:
        clk = clocks.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K_steps,
            "warmup": args.warmup, "ms_per_step": total_ms / K_steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": "Qwen3-8B prefill linears, M=8192 tokens, NVFP4 W4A4 "
                                   "(+ the same shapes as INT4 g128 W4A16 decode at M in {1,4,8,16,32})",
                       "seq_len": PREFILL_M, "linears": [list(l) for l in LINEARS],
                       "l2": "inputs larger than L2 (prefill pass touches ~1.3 GB; five decode weight copies)",
                       "parallelism": f"independent per-rank workloads x{world}"},
            "prefill": {"gemm_only_tflops": gemm_tflops, "quantize_ms": 1e3 * quant_s, "gemm_ms": 1e3 * gemm_s,
                        "pass_ms": 1e3 * pre_s,
                        "per_layer_gemm_tflops": {L["name"]: 2.0 * PREFILL_M * L["N"] * L["K"] /
                                                  (g_ms[j] / 1e3 / K_steps) / 1e12 for j, L in enumerate(pre)}},
            "roofline": {"bound": "tensor", "kernel": "nvfp4_gemm_kernel", "achieved": gemm_tflops,
                         "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                         "peak_source": f"{peaks_kind} bf16 sustained x 4 (nominal FP4/BF16 dense ratio)",
                         "frac_of_burst_peak": gemm_tflops / fp4_burst,
                         "traffic": profiled_traffic("nvfp4_gemm_qwen3_8b_prefill.md", "nvfp4_gemm.cuh")},
            "decode": {"metric": "INT4 W-only decode GB/s (M <= 16)", "value": dec_b / dec_s / 1e9,
                       "unit": "GB/s", "per_batch": per_batch,
                       "roofline": {"bound": "hbm", "kernel": "w4a16_kernel", "achieved": dec_b / dec_s / 1e9,
                                    "peak": hbm, "unit": "GB/s", "frac": dec_b / dec_s / 1e9 / hbm,
                                    "peak_source": f"{peaks_kind} copy bandwidth",
                                    "traffic": profiled_traffic("w4a16_decode_qwen3_8b.md", "w4a16_gemm.cuh")}},
            "clocks": clk,
            "gpu_launches": launches_per_step * K_steps,
        }
        line["e2e"] = {"value": world * gemm_flops / e2e["seconds"] / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]}
        if world == 1:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def per_batch_decode(torch, nvq, dec, dec_w, stream, dec_bytes, reps: int = 20):
    """Per batch size: the four decode layers run back to back, cycling through
    all weight copies (about 0.5 GB, so every weight byte comes from HBM), one
    captured graph per batch size."""
    out = {}
    for M in DECODE_BATCHES:
        calls = []
        for copy in dec_w:
            for D in dec:
                if D["M"] == M:
                    pc, ps = copy[D["layer"]]
                    calls.append((D, pc, ps))
        def run():
            for D, pc, ps in calls:
                nvq.w4a16_gemm(D["x"], pc, ps, D["N"], y=D["y"], workspace=D["ws"], stream=stream)
        run()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run()
        g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        s = a.elapsed_time(b) / 1e3 / reps
        by = sum(dec_bytes(D) for D, _, _ in calls)
        out[str(M)] = {"GB/s": by / s / 1e9, "us_per_call": 1e6 * s / len(calls)}
        del g
    return out


def measure_e2e(torch, nvq, pre, stream, steps: int):
    """Prefill pass through the public binding with pinned host inputs/outputs:
    H2D of each layer's activations, quantize + GEMM, D2H of each layer's output.
    The copies run on two copy streams, so the next layers' inputs go up and the
    finished layers' outputs come down while a layer is quantized and multiplied
    (both PCIe directions at once); events order every buffer's reuse, within a
    step and across steps."""
    hx = [torch.empty(L["x"].shape, dtype=torch.bfloat16, pin_memory=True) for L in pre]
    hy = [torch.empty(L["y"].shape, dtype=torch.bfloat16, pin_memory=True) for L in pre]
    for h, L in zip(hx, pre):
        h.copy_(L["x"].cpu())
    dx = [torch.empty_like(L["x"]) for L in pre]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    x_in = [torch.cuda.Event() for _ in pre]        # layer i's input is on the device
    x_used = [torch.cuda.Event() for _ in pre]      # layer i's quantize has read it
    y_done = [torch.cuda.Event() for _ in pre]      # layer i's GEMM has written y
    y_out = [torch.cuda.Event() for _ in pre]       # layer i's y is on the host
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def one(first: bool):
        for i, (L, h, d, hyy) in enumerate(zip(pre, hx, dx, hy)):
            with torch.cuda.stream(up):
                if not first:
                    up.wait_event(x_used[i])                 # the last step's quantize is done with d
                d.copy_(h, non_blocking=True)
                x_in[i].record(up)
            stream.wait_event(x_in[i])
            nvq.nvfp4_quantize(d, None, codes=L["xc"], scales=L["xs"], tensor_scale_out=L["tx"],
                               workspace=L["ws"], stream=stream)
            x_used[i].record(stream)
            if not first:
                stream.wait_event(y_out[i])                  # the last step's y has left the device
            nvq.nvfp4_gemm_w4a4((L["xc"], L["xs"], L["tx"]), L["wq"], PREFILL_M, L["N"], L["K"], y=L["y"],
                                stream=stream)
            y_done[i].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(y_done[i])
                hyy.copy_(L["y"], non_blocking=True)
                y_out[i].record(down)

    one(True)
    torch.cuda.synchronize()
    a.record(stream)
    up.wait_event(a)
    down.wait_event(a)
    for _ in range(steps):
        one(False)
    stream.wait_event(y_out[-1])                             # the step's last copy, after all others
    b.record(stream)
    torch.cuda.synchronize()
    secs = a.elapsed_time(b) / 1e3 / steps
    h2d = sum(h.numel() * 2 for h in hx)
    d2h = sum(h.numel() * 2 for h in hy)
    return {"seconds": secs, "h2d": h2d, "d2h": d2h}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 400 on the GPU, about one second; 20 for the CPU oracle arm)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="nvq", choices=("nvq", "reference"))
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else 400
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
