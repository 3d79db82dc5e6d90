"""Pins of the CPU oracle against facts the pages and mathematics fix.

Each test plants the oracle against something other than itself: hand-derived
values (tests/golden), grid identities, closed forms, exhaustive brute force
with exact rationals, or an independent restatement (oracle/tiny_ref.py) that
searches the whole grid with Fractions instead of comparing against midpoints.
"""
import os
import random
from fractions import Fraction

import numpy as np
import pytest

from oracle import int4, nvfp4, tiny_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                out.append(line.split())
    return out


def _bf16(v):
    """Round a float to the nearest bf16 value (ties to even) using torch's cast."""
    import torch
    return float(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).float())


def _with_unit_tensor_scale(blocks):
    """Prepend a block holding 2688 so the tensor amax is 2688 and t == 1."""
    head = [2688.0] + [0.0] * 15
    return np.array([head + [v for b in blocks for v in b]], dtype=np.float64)


# --------------------------------------------------------------------- NVFP4

def test_e2m1_ties_and_grid_from_golden():
    rows = _rows("e2m1_ties.txt")
    vals = [float(r[0]) for r in rows]
    want = [int(r[1]) for r in rows]
    # one block: the values plus 6.0 so that amax_b = 6 -> s = 1 (t = 1)
    for sign in (1.0, -1.0):
        for v, w in zip(vals, want):
            blk = [6.0, sign * v] + [0.0] * 14
            if v > 6.0:
                blk = [sign * v] + [0.0] * 15
                x = _with_unit_tensor_scale([blk])
                codes, s, t = nvfp4.quantize(x, t_in=1.0)
                # amax_b = v > 6 -> s = RNE(v/6), every code saturates at <= 7
                assert codes[0, 16] & 7 == 7
                continue
            x = _with_unit_tensor_scale([blk])
            codes, s, t = nvfp4.quantize(x)
            assert t == 1.0
            assert s[0, 1] == 0x38          # e4m3(1.0): exponent 7, mantissa 0
            assert codes[0, 17] == (w | (8 if sign < 0 else 0)), (v, sign)


def test_near_ties_round_toward_exact_side():
    """m*d +- 1 bf16 ulp must leave the tie toward the side of the exact value."""
    mids = nvfp4.E2M1_MIDPOINTS
    for i, mu in enumerate(mids):
        up = np.nextafter(np.float32(mu), np.float32(np.inf))
        # next bf16 above / below mu
        above = _bf16_next(mu, +1)
        below = _bf16_next(mu, -1)
        blk = [6.0, above, below] + [0.0] * 13
        x = _with_unit_tensor_scale([blk])
        codes, s, t = nvfp4.quantize(x)
        assert t == 1.0 and s[0, 1] == 0x38
        assert codes[0, 17] == i + 1, (mu, above)
        assert codes[0, 18] == i, (mu, below)
        del up


def _bf16_next(v, direction):
    import torch
    b = torch.tensor([v], dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
    b = b + direction
    return float(b.view(torch.bfloat16).float())


def test_grid_round_trip_is_identity():
    rng = random.Random(7)
    blocks, want_s, want_c = [], [], []
    for _ in range(24):
        s = rng.randrange(1, 127)                      # any finite positive E4M3
        S = nvfp4.e4m3_value(s)
        if 6 * S > 2688:
            continue
        codes = [rng.randrange(16) for _ in range(16)]
        codes[rng.randrange(16)] = 7 | (rng.randrange(2) << 3)   # block amax = 6 S
        vals = []
        for c in codes:
            m = nvfp4.E2M1_MAGNITUDES[c & 7] * S
            vals.append(-m if c & 8 else m)
        codes = [c if (c & 7) else 0 for c in codes]    # +0.0 carries no sign
        vals = [v if v != 0 else 0.0 for v in vals]
        blocks.append(vals)
        want_s.append(s)
        want_c.extend(codes)
    x = _with_unit_tensor_scale(blocks)
    codes, s, t = nvfp4.quantize(x)
    assert t == 1.0
    assert list(s[0, 1:]) == want_s
    assert list(codes[0, 16:]) == want_c
    assert np.array_equal(nvfp4.dequantize(codes, s, t), x)


def test_tensor_scale_golden():
    for amax, num, e in _rows("tensor_scale.txt"):
        amax, num, e = float(amax), int(num), int(e)
        x = np.zeros((1, 16))
        x[0, 3] = -amax
        assert nvfp4.tensor_scale(x) == num * 2.0 ** e
        # numpy's own fp32 division agrees on these (library special case)
        if amax:
            assert float(np.float32(amax) / np.float32(2688)) == num * 2.0 ** e


def test_all_zero_tensor():
    x = np.zeros((2, 32))
    x[1, 5] = -0.0
    codes, s, t = nvfp4.quantize(x)
    assert t == 1.0 and not s.any()
    assert codes[1, 5] == 8 and codes.sum() == 8


def test_scale_clamp_saturates():
    g = np.random.default_rng(1)
    x = np.array([[_bf16(v) for v in g.standard_normal(64)]])
    x[np.abs(x) < 0.01] = 0.5
    codes, s, t = nvfp4.quantize(x, t_in=1e-6)
    assert np.all(s == 0x7E)                   # 448
    assert np.all((codes & 7) == 7)            # +-6
    assert np.array_equal(codes >> 3, np.signbit(x).astype(np.uint8))


def test_block_scale_underflow_and_min_subnormal():
    tie = 6 * 2.0 ** -10                       # amax/6 == 2^-10: midpoint of 0 and 2^-9
    above = _bf16_next(tie, +1)
    below = _bf16_next(tie, -1)
    x = np.array([[tie] + [-1e-4] + [0.0] * 14 + [above] + [0.0] * 15 + [below] + [0.0] * 15])
    codes, s, t = nvfp4.quantize(x, t_in=1.0)
    assert list(s[0]) == [0, 1, 0]              # tie -> even code 0; above -> 2^-9
    assert codes[0, 0] == 0 and codes[0, 1] == 8   # zero scale: sign only
    assert codes[0, 16] & 7 == 5                # above / 2^-9 = 3.02 -> nearest 3 (code 5)
    assert np.all(codes[0, 32:] & 7 == 0)


def test_scale_layout_golden_and_bijective():
    offs = nvfp4.scale_offsets(256, 128)
    for r, kb, off in _rows("scale_layout.txt"):
        assert offs[int(r), int(kb)] == int(off)
    assert sorted(offs.ravel().tolist()) == list(range(256 * 8))
    # ragged rows: still injective, all offsets inside the padded buffer
    o2 = nvfp4.scale_offsets(130, 320)
    assert len(set(o2.ravel().tolist())) == o2.size
    assert o2.max() < nvfp4.scales_bytes(130, 320)


def test_pack_low_nibble_even():
    c = np.array([[1, 2, 15, 8]], dtype=np.uint8)
    assert list(nvfp4.pack_codes(c)[0]) == [0x21, 0x8F]
    assert np.array_equal(nvfp4.unpack_codes(nvfp4.pack_codes(c)), c)


def _rand_bf16_matrix(rng, rows, cols, scale=1.0, zeros=0.0):
    v = np.array([[_bf16(rng.gauss(0, scale)) for _ in range(cols)] for _ in range(rows)])
    if zeros:
        mask = np.array([[rng.random() < zeros for _ in range(cols)] for _ in range(rows)])
        v[mask] = 0.0
    return v


def _adversarial_rows(rng, t, rows, cols):
    """Rows whose elements sit on or next to an E2M1 decision point of their block."""
    out = []
    for _ in range(rows):
        row = []
        for _b in range(cols // 16):
            S = nvfp4.e4m3_value(rng.randrange(40, 100))
            d = S * t
            blk = [_bf16(6 * d)]
            for _ in range(15):
                mu = rng.choice(list(nvfp4.E2M1_MIDPOINTS))
                v = _bf16(mu * d)
                v = _bf16_next(v, rng.choice((-1, 0, 1))) if v else v
                row_v = -v if rng.random() < 0.5 else v
                blk.append(row_v)
            row.extend(blk)
        out.append(row)
    return np.array(out)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_nvfp4_quantize_matches_fraction_restatement(seed):
    rng = random.Random(seed)
    x = _rand_bf16_matrix(rng, 6, 64, scale=3.0, zeros=0.05)
    x[2, 7] = -0.0
    x[rng.randrange(6), rng.randrange(64)] *= 20
    codes, s, t = nvfp4.quantize(x)
    tc, ts, tt = tiny_ref.nvfp4_quantize(x.tolist())
    assert t == float(tt)
    assert codes.tolist() == tc
    assert s.tolist() == ts


def test_nvfp4_quantize_adversarial_matches_fraction_restatement():
    rng = random.Random(11)
    t = float(tiny_ref.f32_nearest(Fraction(_bf16(1.7)) / 2688))
    x = _adversarial_rows(rng, t, 4, 64)
    codes, s, tt = nvfp4.quantize(x, t_in=t)
    tc, ts, _ = tiny_ref.nvfp4_quantize(x.tolist(), t_in=t)
    assert codes.tolist() == tc and s.tolist() == ts


@pytest.mark.parametrize("M,N", [(1, 1), (2, 3), (4, 4), (3, 2)])
def test_gemm_brute_force_exact(M, N):
    rng = random.Random(M * 10 + N)
    x = _rand_bf16_matrix(rng, M, 64, 2.0)
    w = _rand_bf16_matrix(rng, N, 64, 0.05)
    xc, xs, tx = nvfp4.quantize(x)
    wc, ws, tw = nvfp4.quantize(w)
    y = nvfp4.gemm_ref(nvfp4.dequantize(xc, xs, tx), nvfp4.dequantize(wc, ws, tw))
    exact = tiny_ref.nvfp4_gemm(xc.tolist(), xs.tolist(), Fraction(tx),
                                wc.tolist(), ws.tolist(), Fraction(tw))
    for m in range(M):
        for n in range(N):
            # float64 dot of 64 exact 60-bit products: error <= 64 * 2^-52 * sum|terms|
            terms = np.abs(nvfp4.dequantize(xc, xs, tx)[m] * nvfp4.dequantize(wc, ws, tw)[n]).sum()
            assert abs(Fraction(y[m, n]) - exact[m][n]) <= Fraction(64 * terms) * Fraction(2) ** -52


def test_gemm_unit_scales_is_integer_matmul():
    """All s = 1 and t = 1: Y = (1/4) * (2 e2m1(X)) @ (2 e2m1(W))^T exactly."""
    g = np.random.default_rng(5)
    cx = g.integers(0, 16, size=(8, 128)).astype(np.uint8)
    cw = g.integers(0, 16, size=(6, 128)).astype(np.uint8)
    for c in (cx, cw):                          # one +-6 per block -> s = 1 under t = 1
        c[:, ::16] = 7
    x = nvfp4.e2m1_signed(cx)
    w = nvfp4.e2m1_signed(cw)
    xc, xs, tx = nvfp4.quantize(x, t_in=1.0)
    wc, ws, tw = nvfp4.quantize(w, t_in=1.0)
    assert np.all(xs == 0x38) and np.all(ws == 0x38)
    y = nvfp4.gemm_ref(nvfp4.dequantize(xc, xs, tx), nvfp4.dequantize(wc, ws, tw))
    xi = (2 * x).astype(np.int64)
    wi = (2 * w).astype(np.int64)
    assert np.array_equal(y * 4, (xi @ wi.T).astype(np.float64))


def test_tolerance_bar():
    y_ref = np.array([1.0, -2.0, 0.0, 4.0])
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    ok, _ = nvfp4.within_tolerance(y_ref + 8e-3 * np.abs(y_ref) + 0.99e-3 * rms, y_ref)
    assert ok
    ok, _ = nvfp4.within_tolerance(y_ref + np.array([0, 0, 1.01e-3 * rms, 0]), y_ref)
    assert not ok


# ---------------------------------------------------------------------- INT4

def test_int4_scale_hand_values():
    # amax 7 -> 1; amax 3.5 -> 0.5; amax 1 -> 1/7 = 1.142857..*2^-3, 0.142857*128 =
    # 18.29 -> significand 18 -> bf16 bits 0x3E12; amax 0 -> scale 0, codes 8.
    cases = [(7.0, 0x3F80), (3.5, 0x3F00), (1.0, 0x3E12), (0.0, 0x0000)]
    for amax, bits in cases:
        w = np.zeros((1, 128))
        w[0, 5] = amax
        u, s = int4.quantize(w)
        assert int(s[0, 0]) == bits
        if amax:
            assert u[0, 5] == 15            # q = 7
        assert np.all(u[0, np.arange(128) != 5] == 8)


def test_int4_codes_range_and_ties():
    w = np.zeros((1, 128))
    w[0, 0] = 7.0                           # s = 1
    w[0, 1:8] = [0.5, 1.5, 2.5, -0.5, -1.5, -7.0, 3.5]
    u, s = int4.quantize(w)
    q = u.astype(int) - 8
    assert list(q[0, :8]) == [7, 0, 2, 2, 0, -2, -7, 4]


@pytest.mark.parametrize("seed", [0, 1])
def test_int4_matches_fraction_restatement(seed):
    rng = random.Random(seed)
    w = _rand_bf16_matrix(rng, 3, 256, 0.02)
    w[1, :128] = 0.0
    u, s = int4.quantize(w)
    tu, ts = tiny_ref.int4_quantize(w.tolist())
    assert u.tolist() == tu and s.tolist() == ts
    assert np.all((u >= 1) | (u == 8))      # |q| <= 7 after scale rounding here
    x = _rand_bf16_matrix(rng, 2, 256, 1.0)
    y = int4.w4a16_ref(x, int4.dequantize(u, s))
    exact = tiny_ref.w4a16(x.tolist(), tu, ts)
    for m in range(2):
        for n in range(3):
            assert abs(Fraction(y[m, n]) - exact[m][n]) <= abs(exact[m][n]) * Fraction(2) ** -44 + Fraction(2) ** -60


def test_int4_reorder_is_bijection_and_hand_slots():
    g = np.random.default_rng(3)
    N, K = 32, 256
    u = g.integers(0, 16, size=(N, K)).astype(np.uint8)
    s = g.integers(0, 1 << 16, size=(N, K // 128)).astype(np.uint16)
    pc, ps = int4.pack_weights(u, s)
    assert pc.size == N * K // 2 and ps.size == N * (K // 128) * 2
    u2, s2 = int4.unpack_weights(pc, ps, N, K)
    assert np.array_equal(u, u2) and np.array_equal(s, s2)
    words = pc.view("<u4")
    # unit 0, word 0 (lane 0, j 0, tile 0): nibbles (0,0) (8,0) (0,2) (8,2) (0,1) (8,1) (0,3) (8,3)
    want = [u[0, 0], u[8, 0], u[0, 2], u[8, 2], u[0, 1], u[8, 1], u[0, 3], u[8, 3]]
    assert [(int(words[0]) >> (4 * p)) & 15 for p in range(8)] == [int(v) for v in want]
    # word 1 = lane 0, j 0, tile 1 (rows 16..31): nibble 0 = (16, 0), nibble 7 = (24, 3)
    assert (int(words[1]) & 15) == u[16, 0] and (int(words[1]) >> 28) == u[24, 3]
    # lane 5 (g=1, c=1), j = 6, tile 0 -> word 128*3 + 4*5 + 0: nibble 0 = (1, 32*1 + 4*6), nibble 7 = (9, 59)
    assert (int(words[404]) & 15) == u[1, 56]
    assert (int(words[404]) >> 28) == u[9, 59]
    # lane 5, j = 7, tile 1 -> word 384 + 20 + 3: nibble 0 = (17, 60), nibble 7 = (25, 63)
    assert (int(words[407]) & 15) == u[17, 60] and (int(words[407]) >> 28) == u[25, 63]
    # unit 1 = rows 0..31, group 1: its word 0 nibble 0 is (0, 128)
    assert (int(words[512]) & 15) == u[0, 128]
    sw = ps.view("<u2")
    assert sw[0] == s[0, 0] and sw[1] == s[8, 0] and sw[2] == s[16, 0] and sw[3] == s[24, 0]
    assert sw[4] == s[1, 0] and sw[32] == s[0, 1]


def test_int4_power_of_two_scale_is_exact_integer_dot():
    g = np.random.default_rng(9)
    q = g.integers(-7, 8, size=(4, 256))
    q[:, 0] = 7
    w = q * 0.25                                # amax 1.75 -> s = 0.25 exactly
    u, s = int4.quantize(w)
    assert np.all(s == 0x3E80)
    x = g.integers(-50, 50, size=(1, 256)).astype(np.float64)
    y = int4.w4a16_ref(x, int4.dequantize(u, s))
    assert np.array_equal(y * 4, (x.astype(np.int64) @ q.T).astype(np.float64))


def test_marlin_scale_aware_bound_closed_form():
    # MARLIN page ("weight layout"): the scale overhead caps the 4-bit speedup near 3.87x
    r = int4.bytes_ratio_bf16_over_int4_g128()
    assert abs(r - 2.0 / (0.5 + 2.0 / 128)) < 1e-12
    assert 3.87 <= r < 3.88


# ------------------------------------------------------------------ SiLU * mul epilogue (oracle/swiglu.py)

def test_silu_closed_forms():
    from oracle import swiglu
    assert swiglu.silu(np.array([0.0]))[0] == 0.0
    # silu(1) = 1 / (1 + e^-1), silu(-1) = -1 / (1 + e)
    np.testing.assert_allclose(swiglu.silu(np.array([1.0, -1.0])),
                               [1.0 / (1.0 + np.exp(-1.0)), -1.0 / (1.0 + np.e)], rtol=1e-15)
    g = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(swiglu.silu(g) - swiglu.silu(-g), g, atol=1e-12)   # silu(g) - silu(-g) = g
    assert swiglu.silu(np.array([800.0]))[0] == 800.0                              # sigmoid saturates at 1
    assert swiglu.silu(np.array([-800.0]))[0] == 0.0


def test_gate_up_reference_against_explicit_loops():
    from oracle import swiglu
    g = np.random.default_rng(5)
    x = g.standard_normal((3, 32)); wg = g.standard_normal((4, 32)); wu = g.standard_normal((4, 32))
    G, U, H = swiglu.gate_up_ref(x, wg, wu)
    for m in range(3):
        for n in range(4):
            gv = sum(x[m, k] * wg[n, k] for k in range(32))
            uv = sum(x[m, k] * wu[n, k] for k in range(32))
            assert abs(G[m, n] - gv) < 1e-12 and abs(U[m, n] - uv) < 1e-12
            assert abs(H[m, n] - gv / (1 + np.exp(-gv)) * uv) < 1e-12


def test_consistency_check_accepts_exact_and_rejects_planted_errors():
    from oracle import swiglu
    rng = np.random.default_rng(6)
    H = rng.standard_normal((4, 64)) * 3.0
    t = float(np.float32(0.01))
    codes, scales, _ = nvfp4.quantize(H, t_in=t)
    zero = np.zeros_like(H)
    ok, sr, cr = swiglu.consistent(codes, scales, H, zero, t)
    assert ok and sr == 1.0 and cr == 1.0
    bad = codes.copy()
    i = np.argmax((bad & 7) <= 5)                              # a magnitude two steps away
    bad.flat[i] = (bad.flat[i] & 8) | ((bad.flat[i] & 7) + 2)
    assert not swiglu.consistent(bad, scales, H, np.full_like(H, 1e-9), t)[0]
    flip = codes.copy()
    j = np.argmax(np.abs(H) > 1.0)
    flip.flat[j] ^= 8                                          # wrong sign on a clearly nonzero value
    assert not swiglu.consistent(flip, scales, H, zero, t)[0]
    s_bad = scales.copy()
    s_bad[0, 0] += 3
    assert not swiglu.consistent(codes, s_bad, H, zero, t)[0]


def test_consistency_check_accepts_both_sides_of_a_threshold_inside_the_band():
    from oracle import swiglu
    t = 1.0
    S = 8                                                      # E4M3 code 8 = 2^-6 ... pick the block scale
    d = nvfp4.e4m3_value(S) * t
    H = np.zeros((1, 16))
    H[0, :] = 0.25 * d                                         # every element on midpoint 0 (tie -> code 0)
    H[0, 0] = 6.0 * d                                          # block amax so the scale is exactly code S
    codes, scales, _ = nvfp4.quantize(H, t_in=t)
    assert scales[0, 0] == S and codes[0, 1] == 0
    up = codes.copy()
    up[0, 1] = 1                                               # the other side of the tie
    band = np.full_like(H, 1e-3 * d)
    assert swiglu.consistent(up, scales, H, band, t)[0]
    assert not swiglu.consistent(up, scales, H, np.zeros_like(H), t)[0]


def _band_cases(seed):
    """G, U covering the regimes of silu: around 0, around the zero of silu'
    (g = -1.2785), around the extrema of silu' (g = +-2.3994), far negative,
    far positive, and U near zero; plus typical N(0, 3) pairs."""
    rng = np.random.default_rng(seed)
    centres = [0.0, -1.278464542761074, -2.3993572805154675, 2.3993572805154675, -12.0, 15.0, 0.3]
    G = np.concatenate([c + rng.normal(0, 0.05, 60) for c in centres] + [rng.normal(0, 3, 400)])
    U = np.concatenate([rng.normal(0, 2, 60 * len(centres) - 100), rng.normal(0, 1e-3, 100),
                        rng.normal(0, 3, 400)])
    U[:20] = 0.0
    G[-20:] = 0.0
    return G[None, :], U[None, :]


def _brute_band(G, U, n=801):
    """max over g' on a grid of [G - dG, G + dG] (ends and silu's critical
    point included) and u' in {U - dU, U + dU} of |silu(g') u' - silu(G) U|."""
    from oracle import swiglu
    dG = 8e-3 * np.abs(G) + 1e-3 * np.sqrt(np.mean(G ** 2))
    dU = 8e-3 * np.abs(U) + 1e-3 * np.sqrt(np.mean(U ** 2))
    f = np.linspace(-1.0, 1.0, n)[:, None, None]
    gp = G[None] + f * dG[None]
    crit = np.full_like(G, -1.278464542761074)
    inside = (G - dG <= crit) & (crit <= G + dG)
    gp = np.concatenate([gp, np.where(inside, crit, G)[None]], axis=0)
    h0 = swiglu.silu(G) * U
    best = np.zeros_like(G)
    for up in (U - dU, U + dU):
        best = np.maximum(best, np.max(np.abs(swiglu.silu(gp) * up[None] - h0[None]), axis=0))
    return best


@pytest.mark.parametrize("seed", [0, 1])
def test_silu_mul_error_band_covers_brute_force_and_is_tight(seed):
    """The acceptance band of the SiLU * mul epilogue, pinned by brute force
    over the GEMM bar of G and U: it must contain every |H' - H| reachable
    there, and be at most about twice the largest of them."""
    from oracle import swiglu
    G, U = _band_cases(seed)
    band = swiglu.error_band(G, U)
    brute = _brute_band(G, U)
    assert np.all(band >= brute * (1 - 1e-9)), float(np.max(brute / np.maximum(band, 1e-300)))
    ratio = band / np.maximum(brute, 1e-300)
    assert np.all((ratio <= 2.05) | (band == 0)), float(np.max(ratio))
    # the evaluation term only widens the band, by the stated relative amount at most
    wide = swiglu.error_band(G, U, rel_eval=1e-5)
    assert np.all(wide >= band)
    assert np.all(wide - band <= 1e-5 * (np.abs(swiglu.silu(G)) + 1.1 * 0.5 * np.abs(G) + 1.0) * (np.abs(U) + 1.0))


def test_silu_prime_bound_matches_dense_search():
    """max |silu'| over an interval, from its ends and the two extrema of silu',
    against a dense search."""
    from oracle import swiglu
    rng = np.random.default_rng(3)
    lo = rng.uniform(-8, 8, 300)
    hi = lo + rng.uniform(0, 4, 300)
    dense = np.max(np.abs(swiglu.silu_prime(lo[None] + np.linspace(0, 1, 20001)[:, None] * (hi - lo)[None])), axis=0)
    got = swiglu.max_abs_silu_prime(lo, hi)
    assert np.all(got >= dense * (1 - 1e-12))
    assert np.all(got <= dense * (1 + 1e-7))
    # the extrema are where silu'' vanishes: about -0.0998 and +1.0998
    vals = [float(swiglu.silu_prime(c)) for c in swiglu.SILU_PRIME_EXTREMA]
    assert abs(vals[0] + 0.09984) < 1e-4 and abs(vals[1] - 1.09984) < 1e-4


# ------------------------------------------------------------------ 2:4 sparse INT4 (oracle/sparse24.py)

def test_prune24_keeps_two_largest_per_run_with_lower_index_on_ties():
    from oracle import sparse24
    w = np.array([[1.0, -3.0, 2.0, 0.5, 0.0, 0.0, 0.0, 0.0, 2.0, -2.0, 2.0, 1.0, -1.0, 1.0, 1.0, -1.0]])
    pruned, keep = sparse24.prune24(w)
    np.testing.assert_array_equal(keep[0], [0, 1, 1, 0, 1, 1, 0, 0, 1, 1, 0, 0, 1, 1, 0, 0])
    np.testing.assert_array_equal(pruned[0], [0, -3, 2, 0, 0, 0, 0, 0, 2, -2, 0, 0, -1, 1, 0, 0])
    g = np.random.default_rng(7)
    w = np.round(g.standard_normal((6, 64)) * 4) / 4                # many exact ties
    pruned, keep = sparse24.prune24(w)
    kr, ar = keep.reshape(6, 16, 4), np.abs(w).reshape(6, 16, 4)
    assert np.all(kr.sum(axis=2) == 2)
    for n in range(6):                                            # brute force over the 6 choices
        for r in range(16):
            best = max(((ar[n, r, a] + ar[n, r, b], -a, -b), (a, b)) for a in range(4) for b in range(a + 1, 4))
            a, b = best[1]
            assert kr[n, r, a] and kr[n, r, b]


def test_sparse_quantize_matches_dense_int4_of_the_pruned_weight():
    from oracle import sparse24
    w = synth_like(32, 256, seed=8)
    u_kept, meta, s_bits, keep = sparse24.quantize(w)
    pruned, _ = sparse24.prune24(w)
    u_dense, s_dense = int4.quantize(pruned)
    np.testing.assert_array_equal(sparse24.dense_codes(u_kept, meta), u_dense)
    np.testing.assert_array_equal(s_bits, s_dense)
    _, s_unpruned = int4.quantize(w)                              # a run's max is kept: same scales
    np.testing.assert_array_equal(s_bits, s_unpruned)
    i0, i1 = meta & 3, meta >> 2
    assert np.all(i0 < i1)


def test_sparse_pack_is_a_bijection_and_matches_hand_slots():
    from oracle import sparse24
    g = np.random.default_rng(9)
    N, K = 32, 256
    u = g.integers(0, 16, size=(N, K // 2)).astype(np.uint8)
    pairs = np.array([a | (b << 2) for a in range(4) for b in range(a + 1, 4)], dtype=np.uint8)
    meta = pairs[g.integers(0, 6, size=(N, K // 4))]
    s = g.integers(0, 1 << 16, size=(N, K // 128)).astype(np.uint16)
    p, ps = sparse24.pack(u, meta, s)
    assert p.size == (N // 32) * (K // 128) * 1536 and ps.size == (N // 32) * (K // 128) * 64
    u2, m2, s2 = sparse24.unpack(p, ps, N, K)
    np.testing.assert_array_equal(u2, u)
    np.testing.assert_array_equal(m2, meta)
    np.testing.assert_array_equal(s2, s)
    words = p[:512].copy().view(np.uint32)
    kr = u.reshape(N, K // 4, 2)
    w0 = int(words[0])                                            # lane 0, step 0
    assert (w0 & 0xF) == kr[0, 0, 0] and ((w0 >> 16) & 0xF) == kr[0, 0, 1]     # row 0, run 0
    assert ((w0 >> 4) & 0xF) == kr[8, 0, 0]                                     # row 8, run 0
    assert ((w0 >> 8) & 0xF) == kr[0, 2, 0] and ((w0 >> 24) & 0xF) == kr[0, 2, 1]   # compressed k 8, 9: run 2
    w = int(words[4 * 5 + 3])                                     # lane 5 (g 1, c 1), step 3
    assert (w & 0xF) == kr[1, 8 * 3 + 4, 0]                       # compressed k 2: MMA run 1 -> run 8*3+4
    m = p[512:].copy().view(np.uint32)
    m0 = int(m[0])                                                # lane (0, 0), step 0
    assert (m0 & 0xF) == meta[0, 0] and ((m0 >> 4) & 0xF) == meta[0, 4] and ((m0 >> 16) & 0xF) == meta[8, 0]
    m1 = int(m[4 * 1 + 2])                                        # lane (0, 1), step 2: MMA runs 4..7
    assert (m1 & 0xF) == meta[0, 16 + 2] and ((m1 >> 4) & 0xF) == meta[0, 16 + 6]
    t1 = p[768:768 + 512].copy().view(np.uint32)                  # unit 0, tile 1 = rows 16..31
    assert (int(t1[0]) & 0xF) == kr[16, 0, 0] and ((int(t1[0]) >> 4) & 0xF) == kr[24, 0, 0]
    assert (int(p[1536:1536 + 512].copy().view(np.uint32)[0]) & 0xF) == kr[0, 32, 0]   # unit 1: group 1
    sw = ps.view("<u2")                                           # word 2g + tt: rows 16tt + g, + 8
    assert sw[0] == s[0, 0] and sw[1] == s[8, 0] and sw[2] == s[16, 0] and sw[3] == s[24, 0] and sw[32] == s[0, 1]


def test_sparse_w4a16_reference_against_explicit_loops():
    from oracle import sparse24
    w = synth_like(16, 128, seed=10)
    x = np.random.default_rng(11).standard_normal((2, 128))
    u_kept, meta, s_bits, keep = sparse24.quantize(w)
    y = sparse24.w4a16_ref(x, u_kept, meta, s_bits)
    s = int4.bf16_bits_to_f64(s_bits)
    u = sparse24.dense_codes(u_kept, meta).astype(np.int64)
    for m in range(2):
        for n in range(16):
            ref = sum(x[m, k] * s[n, 0] * (u[n, k] - 8) for k in range(128) if keep[n, k])
            assert abs(y[m, n] - ref) < 1e-9


def synth_like(N, K, seed):
    """bf16-valued float64 weights 0.02 N(0,1) (the pins need only values on the bf16 grid)."""
    v = np.random.default_rng(seed).standard_normal((N, K)) * 0.02
    return int4.bf16_bits_to_f64(int4.f64_to_bf16_bits_rne(v))
