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
QUANTIZE_LAUNCHES = 2   # kernels per nvfp4_quantize call with a computed tensor scale (amax pass, quantize)


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
def fp4_peaks(peaks):
    """Dense NVFP4 peaks (burst, sustained) in TFLOP/s: the measured BF16 cuBLAS
    figures times the nominal dense FP4 / BF16 ratio."""
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP4_OVER_BF16
    sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * FP4_OVER_BF16
    return burst, sust


def pick_fp4_peak(burst: float, sustained: float, clock_reasons):
    """The burst peak applies unless the run's own clock record shows the power
    cap (the sustained figure was measured under it)."""
    if "sw_power_cap" in (clock_reasons or []):
        return sustained, "sustained (sw_power_cap seen during the timed region)"
    return burst, "burst (no sw_power_cap during the timed region)"


def mean_sd(vals):
    vals = [float(v) for v in vals]
    m = statistics.fmean(vals)
    sd = statistics.stdev(vals) if len(vals) > 1 else 0.0
    return m, sd


def split_steps(steps: int, repeats: int):
    """K timed steps as `repeats` contiguous blocks (sizes differ by at most one)."""
    repeats = max(1, min(repeats, steps))
    return [steps // repeats + (1 if r < steps % repeats else 0) for r in range(repeats)]


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
                            ws=torch.zeros(max(wsb, 16), dtype=torch.uint8, device=dev)))
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

    launches_per_step = QUANTIZE_LAUNCHES * len(pre) + len(pre) + len(dec)
    step()                                  # first calls set kernel attributes outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    torch.cuda.synchronize()

    def replay_and_read():
        """One step; its per-kernel device times (ms) from the graph's event nodes."""
        graph.replay()
        stream.synchronize()
        return (pre_ev[0].elapsed_time(pre_ev[1]),
                sum(a.elapsed_time(b) for a, b in g_ev),
                sum(a.elapsed_time(b) for a, b in q_ev),
                d_ev[0][0].elapsed_time(d_ev[0][1]),
                d_ev[1][0].elapsed_time(d_ev[1][1]),
                [a.elapsed_time(b) for a, b in g_ev])

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    # ---------------- noise sizing: two identical conditions, interleaved
    noise = None
    if rank == 0 or world > 1:
        blocks = {"A": [], "B": []}
        for b in range(6):
            vals = [replay_and_read()[0] for _ in range(10)]
            blocks["A" if b % 2 == 0 else "B"].append(statistics.fmean(vals))
        (ma, sa), (mb, sb) = mean_sd(blocks["A"]), mean_sd(blocks["B"])
        noise = {"what": "the same prefill pass timed as two conditions A and B, 3 interleaved blocks of "
                         "10 steps each", "A_ms": ma, "A_sd_ms": sa, "B_ms": mb, "B_sd_ms": sb,
                 "diff_pct": 100.0 * abs(ma - mb) / ma}

    smi_id = gpu_smi_id(torch, local)
    t_start, t_end = ev(), ev()
    reps = {"pass": [], "gemm": [], "quant": [], "dec16": [], "dec32": []}
    g_layer = [0.0] * len(pre)
    sizes = split_steps(args.steps, args.repeats)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(smi_id) as clocks:
        t_start.record(stream)
        for n in sizes:
            acc = [0.0] * 5
            for _ in range(n):
                r = replay_and_read()
                for j in range(5):
                    acc[j] += r[j]
                for j in range(len(pre)):
                    g_layer[j] += r[5][j]
            for key, v in zip(reps, acc):
                reps[key].append(v / n)
        t_end.record(stream)
        torch.cuda.synchronize()
    total_ms = t_start.elapsed_time(t_end)
    if world > 1:
        dist.barrier()
    nvq.check_device_error(stream)

    K_steps = args.steps
    gemm_flops = sum(2.0 * PREFILL_M * L["N"] * L["K"] for L in pre)
    pass_m, pass_sd = mean_sd(reps["pass"])
    gemm_m, gemm_sd = mean_sd(reps["gemm"])
    quant_m, quant_sd = mean_sd(reps["quant"])
    d16_m, d16_sd = mean_sd(reps["dec16"])

    def dec_bytes(D):
        M, K, N = D["M"], D["K"], D["N"]
        return N * K / 2 + 2 * N * K / 128 + 2 * M * K + 2 * M * N

    dec_b = sum(dec_bytes(D) for D in dec if D["M"] <= 16)
    # max over ranks of the step time and of the per-kernel means
    total_ms, pass_m, gemm_m, d16_m = max_over_ranks(torch, dist if world > 1 else None,
                                                     [total_ms, pass_m, gemm_m, d16_m], dev)
    gemm_tflops = gemm_flops / (gemm_m / 1e3) / 1e12      # per GPU (slowest rank): the kernel's roofline
    value = whole_job_rate(gemm_flops, world, pass_m / 1e3) / 1e12
    dec_gbs = dec_b / (d16_m / 1e3) / 1e9
    per_batch = per_batch_decode(torch, nvq, dec, dec_w, stream, dec_bytes)

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if rank == 0 or world > 1:
        e2e = measure_e2e(torch, nvq, pre, stream, steps=max(2, min(args.steps, 5)))
    if world > 1:
        e2e["seconds"] = max_over_ranks(torch, dist, [e2e["seconds"]], dev)[0]

    peaks, peaks_kind = load_peaks()
    fp4_burst, fp4_sust = fp4_peaks(peaks)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    extra = {}
    if rank == 0 and not args.no_extra:
        del pre, dec, dec_w
        torch.cuda.empty_cache()
        extra["config4"] = measure_config4(torch, nvq, synth, stream, dev, fp4_burst, fp4_sust, args.repeats)
        extra["crossover"] = measure_crossover(torch, nvq, synth, stream, dev, args.repeats)

    if rank == 0:
        clk = clocks.summary()
        fp4_peak, peak_rule = pick_fp4_peak(fp4_burst, fp4_sust, clk["reasons"])
        layer_tflops = {LINEARS[j][0]: 2.0 * PREFILL_M * LINEARS[j][2] * LINEARS[j][1] /
                        (g_layer[j] / K_steps / 1e3) / 1e12 for j in range(len(LINEARS))}
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
            "protocol": {"repeats": len(sizes), "steps_per_repeat": sizes,
                         "interleaved": "each step runs the prefill pass then the decode blocks",
                         "noise": noise},
            "prefill": {"pass_ms": pass_m, "pass_sd_ms": pass_sd,
                        "gemm_ms": gemm_m, "gemm_sd_ms": gemm_sd,
                        "quantize_ms": quant_m, "quantize_sd_ms": quant_sd,
                        "gemm_only_tflops": gemm_tflops,
                        "per_layer_gemm_tflops": layer_tflops},
            "roofline": {"bound": "tensor", "kernel": "nvfp4_gemm_kernel", "achieved": gemm_tflops,
                         "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                         "peak_source": f"{peaks_kind} bf16 x 4 (nominal FP4/BF16 dense ratio), {peak_rule}",
                         "frac_of_burst_peak": gemm_tflops / fp4_burst,
                         "frac_of_sustained_peak": gemm_tflops / fp4_sust,
                         "traffic": profiled_traffic("nvfp4_gemm_qwen3_8b_prefill.md", "nvfp4_gemm.cuh")},
            "decode": {"metric": "INT4 W-only decode GB/s (M <= 16)", "value": dec_gbs, "unit": "GB/s",
                       "block_ms": d16_m, "block_sd_ms": d16_sd, "per_batch": per_batch,
                       "roofline": {"bound": "hbm", "kernel": "w4a16_kernel", "achieved": dec_gbs,
                                    "peak": hbm, "unit": "GB/s", "frac": dec_gbs / hbm,
                                    "peak_source": f"{peaks_kind} copy bandwidth",
                                    "traffic": profiled_traffic("w4a16_decode_qwen3_8b.md", "w4a16_gemm.cuh")}},
            "clocks": clk,
            "gpu_launches": launches_per_step * K_steps,
        }
        line.update(extra)
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


def graph_layer_times(torch, stream, calls, reps):
    """Capture `calls` (a list of no-argument launchers) in one graph with an
    event pair around each; replay it `reps` times.  Returns per-call lists of
    device milliseconds (one entry per replay)."""
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    evs = [(ev(), ev()) for _ in calls]

    def run():
        for (a, b), c in zip(evs, calls):
            a.record(stream)
            c()
            b.record(stream)

    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    g.replay()
    torch.cuda.synchronize()
    out = [[] for _ in calls]
    for _ in range(reps):
        g.replay()
        stream.synchronize()
        for i, (a, b) in enumerate(evs):
            out[i].append(a.elapsed_time(b))
    del g
    return out


def measure_config4(torch, nvq, synth, stream, dev, fp4_burst, fp4_sust, repeats):
    """Qwen3-32B prefill linears at M = 32768 tokens: the W4A4 GEMM of each
    layer, inputs quantized once beforehand (untimed), every operand larger
    than L2.  One graph of the four GEMMs replayed `repeats` times."""
    M = 32768
    layers = []
    for i, (name, K, N) in enumerate(synth.QWEN3_32B_LINEARS):
        x = synth.activations_cuda(M, K, seed=4000 + 10 * i, device=dev)
        w = synth.weights_cuda(N, K, seed=4000 + 10 * i, device=dev)
        xq, wq = nvq.nvfp4_quantize(x), nvq.nvfp4_quantize(w)
        del x, w
        layers.append(dict(name=name, K=K, N=N, xq=xq, wq=wq,
                           y=torch.empty(M, N, dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()
    calls = [(lambda L=L: nvq.nvfp4_gemm_w4a4(L["xq"], L["wq"], M, L["N"], L["K"], y=L["y"], stream=stream))
             for L in layers]
    with ClockSampler(gpu_smi_id(torch, dev.index)) as clocks:
        times = graph_layer_times(torch, stream, calls, max(repeats, 5))
    nvq.check_device_error(stream)
    clk = clocks.summary()
    peak, rule = pick_fp4_peak(fp4_burst, fp4_sust, clk["reasons"])
    out = {"workload": "Qwen3-32B prefill linears, M=32768 tokens, NVFP4 W4A4 GEMM (quantized inputs resident)",
           "repeats": len(times[0]), "peak": peak, "peak_rule": rule, "clocks": clk, "layers": {}}
    flops_all, ms_all = 0.0, 0.0
    for L, t in zip(layers, times):
        m, sd = mean_sd(t)
        fl = 2.0 * M * L["N"] * L["K"]
        tf = fl / (m / 1e3) / 1e12
        flops_all += fl
        ms_all += m
        out["layers"][L["name"]] = {"K": L["K"], "N": L["N"], "ms": m, "sd_ms": sd, "tflops": tf,
                                    "frac": tf / peak, "frac_of_burst_peak": tf / fp4_burst}
    out["tflops"] = flops_all / (ms_all / 1e3) / 1e12
    out["frac"] = out["tflops"] / peak
    out["frac_of_burst_peak"] = out["tflops"] / fp4_burst
    del layers
    torch.cuda.empty_cache()
    return out


def measure_crossover(torch, nvq, synth, stream, dev, repeats, copies=4):
    """The phase crossover on the gate_up shape (K = 4096, N = 24576): one BF16
    master weight quantized both ways (NVFP4 for W4A4, INT4 g128 for W4A16),
    both paths timed at every M.  Each graph cycles through `copies` copies of
    the weights (about 210-230 MB, above L2), so weights come from HBM; the
    W4A4 path includes the activation quantize (amax + codes)."""
    K, N = 4096, 24576
    Mmax = max(synth.CROSSOVER_BATCHES)
    w = synth.weights_cuda(N, K, seed=5000, device=dev)
    wq = nvq.nvfp4_quantize(w)
    codes, scales = nvq.int4_quantize(w)
    pc, ps = nvq.int4_pack_weights(codes, scales, N, K)
    del w, codes, scales
    wq_c = [tuple(t.clone() for t in wq) for _ in range(copies)]
    pk_c = [(pc.clone(), ps.clone()) for _ in range(copies)]
    xc = torch.empty(Mmax, K // 2, dtype=torch.uint8, device=dev)
    xs = torch.empty(nvq.nvfp4_scales_bytes(Mmax, K), dtype=torch.uint8, device=dev)
    tx = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(nvq.nvfp4_quantize_workspace_bytes(Mmax, K), dtype=torch.uint8, device=dev)
    y = torch.empty(Mmax * N, dtype=torch.bfloat16, device=dev)
    dws = torch.zeros(max(16, nvq.w4a16_workspace_bytes(Mmax, N, K)), dtype=torch.uint8, device=dev)
    out = {"workload": "gate_up K=4096 N=24576, weights cycled through 4 copies (from HBM)",
           "repeats": max(repeats, 5), "per_M": {}}
    faster16 = []
    for M in synth.CROSSOVER_BATCHES:
        x = synth.activations_cuda(M, K, seed=5000 + M, device=dev)
        yM = y[:M * N].view(M, N)
        sb = nvq.nvfp4_scales_bytes(M, K)

        def w16(i, x=x, yM=yM):
            p = pk_c[i % copies]
            nvq.w4a16_gemm(x, p[0], p[1], N, y=yM, workspace=dws, stream=stream)

        def w4(i, x=x, yM=yM, M=M, sb=sb):
            q = (xc[:M], xs[:sb], tx)
            nvq.nvfp4_quantize(x, None, codes=q[0], scales=q[1], tensor_scale_out=tx, workspace=ws, stream=stream)
            nvq.nvfp4_gemm_w4a4(q, wq_c[i % copies], M, N, K, y=yM, stream=stream)

        res = {}
        for name, fn in (("w4a16", w16), ("w4a4", w4)):
            ncall = 2 * copies
            t = graph_layer_times(torch, stream, [lambda fn=fn: [fn(i) for i in range(ncall)]],
                                  out["repeats"])[0]
            m, sd = mean_sd([v / ncall for v in t])
            res[name + "_us"] = 1e3 * m
            res[name + "_sd_us"] = 1e3 * sd
        res["faster"] = "w4a16" if res["w4a16_us"] < res["w4a4_us"] else "w4a4"
        if res["faster"] == "w4a16":
            faster16.append(M)
        out["per_M"][str(M)] = res
        del x
    nvq.check_device_error(stream)
    out["w4a16_faster_up_to_M"] = max(faster16) if faster16 else 0
    del wq_c, pk_c, xc, xs, y
    torch.cuda.empty_cache()
    return out


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
    ap.add_argument("--repeats", type=int, default=5, help="timed steps are split into this many repeats (mean, sd)")
    ap.add_argument("--no-extra", action="store_true", help="skip the Qwen3-32B and crossover measurements")
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
