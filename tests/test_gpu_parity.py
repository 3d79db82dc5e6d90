"""GPU parity: the CUDA path (through the C-ABI) against the CPU oracle.

Bar: quantized codes, block scales and tensor scales bit-exact; GEMM outputs
within |y - y_ref| <= 8e-3 |y_ref| + 1e-3 rms(y_ref).  Inputs come from the
seeded generators (phase_disaggregated_quantized_b200.synth) or are built here
on and around the rounding decision points.
"""
import numpy as np
import pytest
import torch

import phase_disaggregated_quantized_b200 as nvq
from phase_disaggregated_quantized_b200 import synth
from oracle import int4 as oint4
from oracle import nvfp4 as onv

from helpers import bf16_bits, bf16_to_f64, oracle_int4, oracle_nvfp4, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from phase_disaggregated_quantized_b200 import build_lib
    build_lib.build()
    nvq.lib()
    yield
    nvq.check_device_error()


def gpu_quant(x_cpu, t_in=None):
    x = x_cpu.cuda()
    tin = None if t_in is None else torch.tensor([t_in], dtype=torch.float32, device="cuda")
    c, s, t = nvq.nvfp4_quantize(x, tin)
    nvq.check_device_error()
    return c, s, t


def assert_quant_parity(x_cpu, t_in=None):
    rows, K = x_cpu.shape
    pc, s, t = oracle_nvfp4(x_cpu, t_in)
    gc, gs, gt = gpu_quant(x_cpu, t_in)
    assert float(gt.item()) == t
    np.testing.assert_array_equal(u8(gc), pc)
    np.testing.assert_array_equal(u8(gs), onv.scales_to_tiled(s, rows, K))   # padding rows zero too
    return gc, gs, gt


def assert_quant_whole(x_cpu, gq, chunk=1024):
    """Codes, tiled scales (padding rows zero) and t of a GPU quantize of a
    large tensor against the oracle, bit for bit over the whole tensor.  The
    oracle runs on row chunks with the tensor's t (rows are independent once t
    is fixed); t itself comes from max|x| of the whole tensor."""
    rows, K = x_cpu.shape
    t = onv.tensor_scale_from_amax(float(x_cpu.abs().max()))
    assert float(gq[2].item()) == t
    gc, gs = u8(gq[0]), u8(gq[1]).reshape(-1)
    assert gs.size == onv.scales_bytes(rows, K)
    seen = np.zeros(gs.size, dtype=bool)
    offs_all = onv.scale_offsets(rows, K)
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        c, s, _ = onv.quantize(bf16_to_f64(x_cpu[r0:r1]), t_in=t)
        np.testing.assert_array_equal(gc[r0:r1], onv.pack_codes(c))
        offs = offs_all[r0:r1]
        np.testing.assert_array_equal(gs[offs], s)
        seen[offs.reshape(-1)] = True
    assert not gs[~seen].any()                               # padding rows of the tiled layout


def _bf16_tensor(values) -> torch.Tensor:
    return torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)


# ------------------------------------------------------------------ NVFP4 quantize

def test_quantize_tiny_case_bit_exact():
    x, w = synth.tiny_case()
    assert_quant_parity(x)
    assert_quant_parity(w)


@pytest.mark.parametrize("rows,K", [(1, 64), (77, 192), (130, 1024), (300, 512), (129, 4096)])
def test_quantize_ragged_shapes(rows, K):
    assert_quant_parity(synth.activations(rows, K, seed=rows * 7 + K))


def test_quantize_caller_scale_and_saturation():
    x = synth.activations(64, 256, seed=3)
    assert_quant_parity(x, t_in=0.01)
    assert_quant_parity(x, t_in=1e-6)        # every block scale clamps at 448
    assert_quant_parity(x, t_in=3.0)         # many blocks underflow to a zero scale


def test_quantize_zero_and_signed_zero():
    x = torch.zeros(130, 128, dtype=torch.bfloat16)
    x[5, 7] = -0.0
    x[129, 127] = -0.0
    gc, gs, gt = assert_quant_parity(x)
    assert float(gt.item()) == 1.0


def _decision_point_tensor(seed, t, rows=64, K=512):
    """Elements on and one bf16 ulp around mu_i * S * t for random E4M3 scales S."""
    g = np.random.default_rng(seed)
    out = np.zeros((rows, K), dtype=np.float32)
    mids = onv.E2M1_MIDPOINTS
    for r in range(rows):
        for b in range(K // 16):
            S = onv.e4m3_value(int(g.integers(1, 127)))
            d = S * t
            vals = [6 * d] + [float(g.choice(mids)) * d for _ in range(15)]
            out[r, 16 * b:16 * b + 16] = vals
    xb = torch.tensor(out).to(torch.bfloat16)
    bits = xb.view(torch.int16)
    bits += torch.tensor(g.integers(-1, 2, size=(rows, K)), dtype=torch.int16)
    xb = bits.view(torch.bfloat16)
    sign = torch.tensor(g.integers(0, 2, size=(rows, K)).astype(bool))
    xb[sign] = -xb[sign]
    return xb


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_quantize_decision_points_bit_exact(seed):
    t = float(np.float32(1.3 ** (seed - 2) / 2688 * 17.0))
    x = _decision_point_tensor(seed, t)
    assert_quant_parity(x, t_in=t)           # ties and near-ties under a caller scale
    assert_quant_parity(x)                   # and under the computed scale


@pytest.mark.parametrize("amax", [87.0, 64.0, 162.0, 5.5, 127.5, 21.0, 1.0])
def test_quantize_computed_scale_near_ties_bit_exact(amax):
    """t = fl(amax / 2688) with amax a bf16 value: wherever mu_i S carries the
    factor 21 (2688 = 2^7 * 21), the threshold mu_i S t lies within t's rounding
    error of a bf16 value.  Elements on and one ulp around every mu_i S t, with
    the tensor's max |x| pinned to amax so that the computed t is that one (21
    gives an exact t and exact ties)."""
    t = float(np.float32(np.float32(amax) / np.float32(2688.0)))
    x = _decision_point_tensor(int(amax * 8) % 1000, t, rows=96, K=1024)
    xf = x.float().clamp(-amax, amax)
    xf[0, 0] = amax
    x = xf.to(torch.bfloat16)
    _, _, gt = assert_quant_parity(x)
    assert float(gt.item()) == t


def test_quantize_grid_round_trip():
    g = np.random.default_rng(4)
    rows, K = 8, 256
    vals = np.zeros((rows, K))
    vals[0, 0] = 2688.0
    for r in range(rows):
        for b in range(K // 16):
            if r == 0 and b == 0:
                continue
            S = onv.e4m3_value(int(g.integers(1, 100)))
            c = g.integers(0, 8, size=16)
            c[g.integers(16)] = 7
            vals[r, 16 * b:16 * b + 16] = onv.E2M1_MAGNITUDES[c] * S * np.where(g.random(16) < 0.5, -1, 1)
    x = _bf16_tensor(vals)
    gc, gs, gt = assert_quant_parity(x)
    assert float(gt.item()) == 1.0
    deq = onv.dequantize(onv.unpack_codes(u8(gc)), onv.scales_from_tiled(u8(gs), rows, K), 1.0)
    np.testing.assert_array_equal(deq, bf16_to_f64(x))


# ------------------------------------------------------------------ NVFP4 GEMM

def gemm_case(x_cpu, w_cpu, t_in_x=None, t_in_w=None):
    M, K = x_cpu.shape
    N = w_cpu.shape[0]
    xq = gpu_quant(x_cpu, t_in_x)
    wq = gpu_quant(w_cpu, t_in_w)
    y = nvq.nvfp4_gemm_w4a4(xq, wq, M, N, K)
    nvq.check_device_error()
    xc, xs, tx = onv.quantize(bf16_to_f64(x_cpu), t_in=t_in_x)
    wc, ws, tw = onv.quantize(bf16_to_f64(w_cpu), t_in=t_in_w)
    y_ref = onv.gemm_ref(onv.dequantize(xc, xs, tx), onv.dequantize(wc, ws, tw))
    return bf16_to_f64(y), y_ref


def test_gemm_tiny_case():
    x, w = synth.tiny_case()
    y, y_ref = gemm_case(x, w)
    ok, worst = onv.within_tolerance(y, y_ref)
    assert ok, worst


@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (77, 136, 192), (200, 264, 320), (129, 520, 1024),
                                   (300, 256, 4096), (256, 512, 256), (5, 1000, 128),
                                   (257, 520, 512), (513, 8, 256), (1000, 1000, 320), (300, 264, 64),
                                   (640, 2048, 1024)])
def test_gemm_ragged_shapes(M, N, K):
    x = synth.activations(M, K, seed=M + N + K)
    w = synth.weights(N, K, seed=M * N)
    y, y_ref = gemm_case(x, w)
    ok, worst = onv.within_tolerance(y, y_ref)
    assert ok, (M, N, K, worst)


def test_gemm_unit_scales_exact_integer_case():
    """All block scales 1 and t = 1: Y = RNE_bf16 of an exact quarter-integer sum."""
    g = np.random.default_rng(8)
    M, N, K = 200, 264, 512
    cx = g.integers(0, 16, size=(M, K))
    cw = g.integers(0, 16, size=(N, K))
    cx[:, ::16] = 7
    cw[:, ::16] = 7 | 8
    x = _bf16_tensor(onv.e2m1_signed(cx.astype(np.uint8)))
    w = _bf16_tensor(onv.e2m1_signed(cw.astype(np.uint8)))
    y, y_ref = gemm_case(x, w, 1.0, 1.0)
    want = torch.tensor(y_ref, dtype=torch.float64).to(torch.float32).to(torch.bfloat16)
    np.testing.assert_array_equal(y, bf16_to_f64(want))


@pytest.mark.parametrize("layer", range(4))
def test_gemm_qwen3_8b_prefill_full_size(layer):
    """M = 8192 on each Qwen3-8B linear: codes, scales and t of X and W bit-exact
    over the whole tensors; the GEMM on sampled rows and columns against the
    oracle."""
    name, K, N = synth.QWEN3_8B_LINEARS[layer]
    M = 8192
    x = synth.activations(M, K, seed=2000 + 10 * layer)
    w = synth.weights(N, K, seed=2000 + 10 * layer)
    gx = gpu_quant(x)
    gw = gpu_quant(w)
    y = nvq.nvfp4_gemm_w4a4(gx, gw, M, N, K)
    nvq.check_device_error()
    assert_quant_whole(x, gx)
    assert_quant_whole(w, gw)
    g = np.random.default_rng(layer)
    mi = np.sort(g.choice(M, 48, replace=False))
    ni = np.sort(g.choice(N, 48, replace=False))
    xf, wf = bf16_to_f64(x[torch.tensor(mi)]), bf16_to_f64(w[torch.tensor(ni)])
    tx, tw = float(gx[2].item()), float(gw[2].item())
    xc, xs, _ = onv.quantize(xf, t_in=tx)
    wc, ws, _ = onv.quantize(wf, t_in=tw)
    y_ref = onv.gemm_ref(onv.dequantize(xc, xs, tx), onv.dequantize(wc, ws, tw))
    y_s = bf16_to_f64(y[torch.tensor(mi).cuda()][:, torch.tensor(ni).cuda()])
    ok, worst = onv.within_tolerance(y_s, y_ref)
    assert ok, (name, worst)


@pytest.mark.parametrize("layer", range(4))
def test_gemm_qwen3_32b_prefill_full_size_sampled(layer):
    """M = 32768 on each Qwen3-32B linear (up to 1.7 GB of activations); sampled
    rows and columns against the oracle.  Inputs are drawn on the GPU by the
    seeded generators (a CPU draw of 0.8 G values would dominate the test); the
    oracle receives them as bytes and takes max|x| of the whole tensor itself."""
    name, K, N = synth.QWEN3_32B_LINEARS[layer]
    M = 32768
    x = synth.activations_cuda(M, K, seed=4000 + 10 * layer)
    w = synth.weights_cuda(N, K, seed=4000 + 10 * layer)
    gx = gpu_quant(x)
    gw = gpu_quant(w)
    y = nvq.nvfp4_gemm_w4a4(gx, gw, M, N, K)
    nvq.check_device_error()
    g = np.random.default_rng(100 + layer)
    mi = np.sort(g.choice(M, 32, replace=False))
    ni = np.sort(g.choice(N, 32, replace=False))
    x_cpu, w_cpu = x.cpu(), w.cpu()
    tx = onv.tensor_scale_from_amax(float(x_cpu.abs().max()))
    tw = onv.tensor_scale_from_amax(float(w_cpu.abs().max()))
    xc, xs, _ = onv.quantize(bf16_to_f64(x_cpu[torch.tensor(mi)]), t_in=tx)
    wc, ws, _ = onv.quantize(bf16_to_f64(w_cpu[torch.tensor(ni)]), t_in=tw)
    del x_cpu, w_cpu
    assert float(gx[2].item()) == tx and float(gw[2].item()) == tw
    np.testing.assert_array_equal(u8(gx[0][torch.tensor(mi).cuda()]), onv.pack_codes(xc))
    np.testing.assert_array_equal(u8(gw[0][torch.tensor(ni).cuda()]), onv.pack_codes(wc))
    offs_x, offs_w = onv.scale_offsets(M, K, row_index=mi), onv.scale_offsets(N, K, row_index=ni)
    np.testing.assert_array_equal(u8(gx[1])[offs_x], xs)
    np.testing.assert_array_equal(u8(gw[1])[offs_w], ws)
    y_ref = onv.gemm_ref(onv.dequantize(xc, xs, tx), onv.dequantize(wc, ws, tw))
    y_s = bf16_to_f64(y[torch.tensor(mi).cuda()][:, torch.tensor(ni).cuda()])
    ok, worst = onv.within_tolerance(y_s, y_ref)
    assert ok, (name, worst)


# ------------------------------------------------------------------ INT4 / W4A16

def gpu_int4(w_cpu):
    N, K = w_cpu.shape
    codes, scales = nvq.int4_quantize(w_cpu.cuda())
    pc, ps = nvq.int4_pack_weights(codes, scales, N, K)
    nvq.check_device_error()
    return codes, scales, pc, ps


@pytest.mark.parametrize("N,K", [(512, 512), (32, 128), (4096, 4096), (96, 384)])
def test_int4_quantize_and_pack_bit_exact(N, K):
    w = synth.weights(N, K, seed=N + K)
    if N == 96:
        w[3, :128] = 0                                       # an all-zero group
    codes, scales, pc, ps = gpu_int4(w)
    u, s_bits = oracle_int4(w)
    np.testing.assert_array_equal(u8(codes), oint4.pack_nibbles(u))
    np.testing.assert_array_equal(bf16_bits(scales), s_bits)
    opc, ops = oint4.pack_weights(u, s_bits)
    np.testing.assert_array_equal(u8(pc), opc)
    np.testing.assert_array_equal(u8(ps), ops)
    u2, s2 = oint4.unpack_weights(u8(pc), u8(ps), N, K)
    np.testing.assert_array_equal(u2, u)
    np.testing.assert_array_equal(s2, s_bits)


def w4a16_case(x_cpu, w_cpu, packed=None):
    N, K = w_cpu.shape
    if packed is None:
        packed = gpu_int4(w_cpu)
    _, _, pc, ps = packed
    y = nvq.w4a16_gemm(x_cpu.cuda(), pc, ps, N)
    nvq.check_device_error()
    u, s_bits = oracle_int4(w_cpu)
    y_ref = oint4.w4a16_ref(bf16_to_f64(x_cpu), oint4.dequantize(u, s_bits))
    return bf16_to_f64(y), y_ref


@pytest.mark.parametrize("M", [1, 4, 16])
def test_w4a16_tiny_case(M):
    _, w = synth.tiny_case()
    x = synth.activations(M, 512, seed=M, n_outliers=4)
    y, y_ref = w4a16_case(x, w)
    ok, worst = onv.within_tolerance(y, y_ref)
    assert ok, worst


@pytest.mark.parametrize("M,N,K", [(3, 1024, 1024), (13, 288, 384), (33, 1024, 2048), (100, 544, 640),
                                   (1, 32, 128), (8, 8192, 128), (64, 4096, 1024), (5, 96, 1152)])
def test_w4a16_ragged(M, N, K):
    x = synth.activations(M, K, seed=M + K)
    w = synth.weights(N, K, seed=N)
    y, y_ref = w4a16_case(x, w)
    ok, worst = onv.within_tolerance(y, y_ref)
    assert ok, (M, N, K, worst)


@pytest.mark.parametrize("layer", range(4))
def test_w4a16_qwen3_8b_decode_full_size(layer):
    name, K, N = synth.QWEN3_8B_LINEARS[layer]
    w = synth.weights(N, K, seed=3000 + 10 * layer)
    packed = gpu_int4(w)
    for M in synth.DECODE_BATCHES:
        x = synth.activations(M, K, seed=3000 + 10 * layer + M)
        y, y_ref = w4a16_case(x, w, packed)
        ok, worst = onv.within_tolerance(y, y_ref)
        assert ok, (name, M, worst)


@pytest.mark.parametrize("M", synth.CROSSOVER_BATCHES)
def test_crossover_sweep_both_paths_sampled(M):
    """gate_up (K=4096, N=24576): one master W quantized both ways, both paths at M."""
    K, N = 4096, 24576
    w = synth.weights(N, K, seed=5000)
    x = synth.activations(M, K, seed=5000 + M)
    g = np.random.default_rng(M)
    mi = np.sort(g.choice(M, min(M, 32), replace=False))
    ni = np.sort(g.choice(N, 64, replace=False))
    xf, wf = bf16_to_f64(x), bf16_to_f64(w)
    # W4A4
    gx, gw = gpu_quant(x), gpu_quant(w)
    y4 = nvq.nvfp4_gemm_w4a4(gx, gw, M, N, K)
    assert_quant_whole(x, gx)
    tx, tw = onv.tensor_scale(xf), onv.tensor_scale(wf)
    xc, xs, _ = onv.quantize(xf[mi], t_in=tx)
    wc, ws, _ = onv.quantize(wf[ni], t_in=tw)
    y_ref = onv.gemm_ref(onv.dequantize(xc, xs, tx), onv.dequantize(wc, ws, tw))
    y_s = bf16_to_f64(y4[torch.tensor(mi).cuda()][:, torch.tensor(ni).cuda()])
    ok, worst = onv.within_tolerance(y_s, y_ref)
    assert ok, ("w4a4", M, worst)
    # W4A16
    _, _, pc, ps = gpu_int4(w)
    y16 = nvq.w4a16_gemm(x.cuda(), pc, ps, N)
    nvq.check_device_error()
    u, s_bits = oint4.quantize(wf[ni])
    y_ref = oint4.w4a16_ref(xf[mi], oint4.dequantize(u, s_bits))
    y_s = bf16_to_f64(y16[torch.tensor(mi).cuda()][:, torch.tensor(ni).cuda()])
    ok, worst = onv.within_tolerance(y_s, y_ref)
    assert ok, ("w4a16", M, worst)


def test_crossover_master_weight_both_formats_whole_tensor():
    """The one BF16 master weight of the crossover sweep (gate_up, N = 24576,
    K = 4096) in both formats, bit-exact over the whole tensor: NVFP4 codes,
    tiled scales and t; INT4 g128 codes and BF16 scales; and the packed decode
    layout."""
    K, N = 4096, 24576
    w = synth.weights(N, K, seed=5000)
    assert_quant_whole(w, gpu_quant(w))
    codes, scales, pc, ps = gpu_int4(w)
    u_parts, s_parts = [], []
    for r0 in range(0, N, 2048):
        u, s_bits = oracle_int4(w[r0:r0 + 2048])
        np.testing.assert_array_equal(u8(codes[r0:r0 + 2048]), oint4.pack_nibbles(u))
        np.testing.assert_array_equal(bf16_bits(scales[r0:r0 + 2048]), s_bits)
        u_parts.append(u)
        s_parts.append(s_bits)
    opc, ops = oint4.pack_weights(np.concatenate(u_parts), np.concatenate(s_parts))
    np.testing.assert_array_equal(u8(pc), opc)
    np.testing.assert_array_equal(u8(ps), ops)


# ------------------------------------------------------------------ 2:4 sparse INT4 decode

def gpu_sparse24(w_cpu):
    N, K = w_cpu.shape
    wd = w_cpu.cuda()
    codes, scales = nvq.int4_quantize(wd)
    p, ps = nvq.int4_pack_sparse24(wd, codes, scales)
    nvq.check_device_error()
    return p, ps


@pytest.mark.parametrize("N,K", [(32, 128), (64, 512), (96, 384)])
def test_sparse24_pack_bit_exact(N, K):
    from oracle import sparse24 as osp
    w = synth.weights(N, K, seed=N * 7 + K)
    w[1, :8] = 0                                              # runs of zeros: ties everywhere
    w[2, 4:8] = w[2, 4]                                       # four equal magnitudes
    p, ps = gpu_sparse24(w)
    u, meta, s_bits, _ = osp.quantize(bf16_to_f64(w))
    op, ops = osp.pack(u, meta, s_bits)
    np.testing.assert_array_equal(u8(p), op)
    np.testing.assert_array_equal(u8(ps), ops)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (4, 512, 1024), (8, 1024, 256), (13, 288, 384), (16, 512, 512),
                                   (32, 1024, 2048), (40, 256, 1024), (1, 32, 128)])
def test_sparse24_decode_matches_oracle(M, N, K):
    from oracle import sparse24 as osp
    x = synth.activations(M, K, seed=M + 3 * K)
    w = synth.weights(N, K, seed=N + 5)
    p, ps = gpu_sparse24(w)
    y = nvq.w4a16_sparse24_gemm(x.cuda(), p, ps, N)
    nvq.check_device_error()
    u, meta, s_bits, _ = osp.quantize(bf16_to_f64(w))
    y_ref = osp.w4a16_ref(bf16_to_f64(x), u, meta, s_bits)
    ok, worst = onv.within_tolerance(bf16_to_f64(y), y_ref)
    assert ok, (M, N, K, worst)


@pytest.mark.parametrize("layer", range(4))
def test_sparse24_decode_qwen3_8b_full_size(layer):
    from oracle import sparse24 as osp
    name, K, N = synth.QWEN3_8B_LINEARS[layer]
    w = synth.weights(N, K, seed=3100 + 10 * layer)
    p, ps = gpu_sparse24(w)
    u, meta, s_bits, _ = osp.quantize(bf16_to_f64(w))
    for M in (1, 16):
        x = synth.activations(M, K, seed=3200 + M + layer)
        y = nvq.w4a16_sparse24_gemm(x.cuda(), p, ps, N)
        nvq.check_device_error()
        y_ref = osp.w4a16_ref(bf16_to_f64(x), u, meta, s_bits)
        ok, worst = onv.within_tolerance(bf16_to_f64(y), y_ref)
        assert ok, (name, M, worst)


# ------------------------------------------------------------------ phase dispatch

@pytest.mark.parametrize("M", [1, 8, 9, 40])
def test_nvq_linear_dispatches_by_batch_size(M):
    """One master W in both formats; nvq_linear must return exactly what the
    path it picks returns, and that path must match its oracle."""
    K, N = 512, 384
    w = synth.weights(N, K, seed=77)
    x = synth.activations(M, K, seed=78)
    wq = gpu_quant(w)
    packed = gpu_int4(w)
    xg = x.cuda()
    crossover = 8
    y = nvq.nvq_linear(xg, wq, packed[2:], N, crossover_m=crossover)
    nvq.check_device_error()
    if M <= crossover:
        direct = nvq.w4a16_gemm(xg, packed[2], packed[3], N)
        got, ref = w4a16_case(x, w, packed)
    else:
        direct = nvq.nvfp4_gemm_w4a4(nvq.nvfp4_quantize(xg), wq, M, N, K)
        got, ref = gemm_case(x, w)
    nvq.check_device_error()
    assert torch.equal(y, direct)
    np.testing.assert_array_equal(bf16_to_f64(y), got)
    ok, worst = onv.within_tolerance(got, ref)
    assert ok, (M, worst)


def test_nvq_linear_default_crossover_uses_w4a16_at_batch_one():
    K, N = 4096, 4096
    w = synth.weights(N, K, seed=79)
    x = synth.activations(1, K, seed=80).cuda()
    packed = gpu_int4(w)
    y = nvq.nvq_linear(x, None, packed[2:], N)           # no NVFP4 form needed at M = 1
    assert torch.equal(y, nvq.w4a16_gemm(x, packed[2], packed[3], N))


# ------------------------------------------------------------------ gate_up GEMM with SiLU * mul -> NVFP4

def _swiglu_case(M, I, K, seed, rows=None, t_scale=1.0, gpu_inputs=False):
    """Runs the fused kernel and returns what the oracle comparison needs."""
    from oracle import swiglu as osw
    gen = synth.activations_cuda if gpu_inputs else synth.activations
    wgen = synth.weights_cuda if gpu_inputs else synth.weights
    x = gen(M, K, seed=seed)
    wg, wu = wgen(I, K, seed=seed + 1), wgen(I, K, seed=seed + 2)
    wi = nvq.interleave_gate_up(wg.cuda(), wu.cuda()).contiguous()
    xq = gpu_quant(x)
    wq = gpu_quant(wi)
    x_cpu = x.cpu()
    wg_c, wu_c = wg.cpu(), wu.cpu()
    tx = onv.tensor_scale_from_amax(float(x_cpu.abs().max()))
    tw = onv.tensor_scale_from_amax(float(torch.maximum(wg_c.abs().max(), wu_c.abs().max())))
    assert float(xq[2].item()) == tx and float(wq[2].item()) == tw
    rows = np.arange(M) if rows is None else rows
    xc, xs, _ = onv.quantize(bf16_to_f64(x_cpu[torch.tensor(rows)]), t_in=tx)
    gc, gs, _ = onv.quantize(bf16_to_f64(wg_c), t_in=tw)
    uc, us, _ = onv.quantize(bf16_to_f64(wu_c), t_in=tw)
    xh = onv.dequantize(xc, xs, tx)
    G, U, H = osw.gate_up_ref(xh, onv.dequantize(gc, gs, tw), onv.dequantize(uc, us, tw))
    t_h = float(np.float32(t_scale * float(np.max(np.abs(H))) / 2688.0))
    th_dev = torch.tensor([t_h], dtype=torch.float32, device="cuda")
    hc, hs, _ = nvq.nvfp4_gemm_w4a4_swiglu(xq, wq, M, 2 * I, K, th_dev)
    nvq.check_device_error()
    codes = onv.unpack_codes(u8(hc))[rows]
    scales = onv.scales_from_tiled(u8(hs), M, I)[rows]
    # The kernel evaluates silu with the fast exponential and division (relative
    # error about 1e-6 for the |G| seen here); 1e-5 covers it.
    band = osw.error_band(G, U, rel_eval=1e-5)
    return osw.consistent(codes, scales, H, band, t_h), u8(hs), M, I


@pytest.mark.parametrize("M,I,K,t_scale", [(200, 256, 256, 1.0), (128, 384, 512, 1.0), (72, 128, 64, 1.0),
                                           (300, 256, 256, 1.0), (520, 384, 320, 1.0),
                                           (130, 256, 320, 0.05), (64, 256, 256, 40.0)])
def test_swiglu_gemm_emits_valid_nvfp4(M, I, K, t_scale):
    """Every block scale and code is the exact RTN result for some H' inside the
    GEMM error band of the oracle's H; nearly all agree with the oracle's own
    RTN of H.  t_scale < 1 saturates many blocks at the largest scale, > 1
    sends small blocks to zero scales."""
    (ok, s_rate, c_rate), hs, M_, I_ = _swiglu_case(M, I, K, seed=300 + M + K, t_scale=t_scale)
    assert ok
    assert s_rate >= 0.99 and c_rate >= 0.99, (s_rate, c_rate)
    full = onv.scales_from_tiled(hs, M_, I_)
    assert full.shape == (M_, I_ // 16)
    pad = onv.padded_rows(M_)
    if pad > M_:                                             # padding rows of the tiled layout are zero
        offs = onv.scale_offsets(pad, I_)[M_:]
        assert not hs[offs].any()


def test_swiglu_gemm_qwen3_8b_gate_up_full_size_sampled():
    """M = 8192, K = 4096, I = 12288 (gate_up N = 24576): 24 sampled rows, every
    H column of those rows."""
    g = np.random.default_rng(9)
    rows = np.sort(g.choice(8192, 24, replace=False))
    (ok, s_rate, c_rate), _, _, _ = _swiglu_case(8192, 12288, 4096, seed=5100, rows=rows, gpu_inputs=True)
    assert ok
    assert s_rate >= 0.99 and c_rate >= 0.99, (s_rate, c_rate)


# ------------------------------------------------------------------ weights streamed from host

def test_prefill_streamed_matches_oracle_and_resident_weights():
    """Five layers with NVFP4 weights in pinned host memory, copies on their own
    stream (Disaggregated Quantization page, ODP: two device buffers, the next
    layer's weights read while the current one computes): every output is
    within the GEMM bar of the oracle (NVFP4 RTN of X and W, float64 GEMM) and
    equals the GEMM run on device-resident weights, also when the same
    workspace is reused by a second call right away."""
    M = 200
    shapes = [(512, 256), (384, 512), (1024, 256), (256, 1024), (640, 384)]
    layers, want, refs = [], [], []
    for i, (N, K) in enumerate(shapes):
        w_cpu = synth.weights(N, K, seed=90 + i)
        x_cpu = synth.activations(M, K, seed=95 + i)
        w, x = w_cpu.cuda(), x_cpu.cuda()
        wq = nvq.nvfp4_quantize(w)
        want.append(nvq.nvfp4_gemm_w4a4(nvq.nvfp4_quantize(x), wq, M, N, K))
        xc, xs, tx = onv.quantize(bf16_to_f64(x_cpu))
        wc, ws_, tw = onv.quantize(bf16_to_f64(w_cpu))
        refs.append(onv.gemm_ref(onv.dequantize(xc, xs, tx), onv.dequantize(wc, ws_, tw)))
        host = tuple(t.cpu().pin_memory() for t in wq)
        layers.append(dict(w_host=host, x=x, y=torch.empty(M, N, dtype=torch.bfloat16, device="cuda"), N=N, K=K))
    torch.cuda.synchronize()
    copy_stream = torch.cuda.Stream()
    ws = nvq.prefill_streamed(layers, M, copy_stream=copy_stream)
    torch.cuda.synchronize()
    nvq.check_device_error()
    for i, (L, ref, y_ref) in enumerate(zip(layers, want, refs)):
        ok, worst = onv.within_tolerance(bf16_to_f64(L["y"]), y_ref)
        assert ok, (i, worst)
        assert torch.equal(L["y"], ref)
    for L in layers:
        L["y"].zero_()
    nvq.prefill_streamed(layers, M, workspace=ws, copy_stream=copy_stream)
    nvq.prefill_streamed(layers, M, workspace=ws, copy_stream=copy_stream)     # slots refilled while read?
    torch.cuda.synchronize()
    for L, ref in zip(layers, want):
        assert torch.equal(L["y"], ref)


def test_device_error_word_is_clear_after_normal_runs():
    nvq.check_device_error()


def test_bounded_wait_timeout_is_reported_and_context_stays_usable():
    """A wait that nothing completes gives up after its limit, raises the error
    word and returns; the host reads NVQ_ERR_DEVICE_TIMEOUT once, and the
    kernels that follow still match the oracle."""
    nvq.check_device_error()                                  # start clean
    nvq.selftest_wait_timeout(2_000_000)                      # 2 ms
    with pytest.raises(nvq.NvqError) as e:
        nvq.check_device_error()
    assert e.value.status == 6                                # NVQ_ERR_DEVICE_TIMEOUT
    nvq.check_device_error()                                  # the check cleared the word
    x = synth.activations(4, 512, seed=11)
    w = synth.weights(256, 512, seed=12)
    y, y_ref = w4a16_case(x, w)
    ok, worst = onv.within_tolerance(y, y_ref)
    assert ok, worst
    nvq.check_device_error()


@pytest.mark.parametrize("rows,K,cut", [(384, 512, 128), (256, 4096, 128), (300, 192, 256)])
def test_row_split_quantize_matches_one_whole_tensor_call(rows, K, cut):
    """Rows split into two shards at `cut`: per-shard nvfp4_amax, their max (the
    all-reduce(MAX) across ranks, here on one device), nvfp4_scale_from_amax,
    then nvfp4_quantize of each shard with that t give the bytes of one call
    over the whole tensor, and the oracle's t."""
    x = synth.activations(rows, K, seed=rows + K, n_outliers=3).cuda()
    whole_c, whole_s, whole_t = nvq.nvfp4_quantize(x)
    shards = [x[:cut].contiguous(), x[cut:].contiguous()]
    amaxes = [nvq.nvfp4_amax(sh) for sh in shards]
    amax = torch.maximum(amaxes[0], amaxes[1])
    t = nvq.nvfp4_scale_from_amax(amax)
    parts = [nvq.nvfp4_quantize(sh, t) for sh in shards]
    nvq.check_device_error()
    assert float(amax.item()) == float(bf16_to_f64(x.cpu()).__abs__().max())
    assert float(t.item()) == onv.tensor_scale(bf16_to_f64(x.cpu())) == float(whole_t.item())
    assert torch.equal(torch.cat([parts[0][0], parts[1][0]]), whole_c)
    logical = [onv.scales_from_tiled(u8(p[1]), sh.shape[0], K) for p, sh in zip(parts, shards)]
    np.testing.assert_array_equal(np.concatenate(logical), onv.scales_from_tiled(u8(whole_s), rows, K))


def test_amax_of_empty_and_zero_shards_and_scale_of_zero():
    z = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    assert float(nvq.nvfp4_amax(z).item()) == 0.0
    zero = torch.zeros(64, 128, dtype=torch.bfloat16, device="cuda")
    a = nvq.nvfp4_amax(zero)
    assert float(a.item()) == 0.0
    assert float(nvq.nvfp4_scale_from_amax(a).item()) == 1.0              # the all-zero reading
    for v in (1.0, 2688.0, 3.0e-30, 1.0e30, 448.0 * 6.0 * 7.0):
        t = nvq.nvfp4_scale_from_amax(torch.tensor([v], dtype=torch.float32, device="cuda"))
        assert float(t.item()) == onv.tensor_scale_from_amax(float(np.float32(v)))
    nvq.check_device_error()
