"""Pure-Python cross-check of the oracle, on tiny inputs only.

TEST INFRASTRUCTURE ONLY.  It re-derives every rounding by a different route
from the numpy oracle: nearest-value search over the whole target grid with
exact ``fractions.Fraction`` arithmetic (no precomputed midpoints, no float64
comparisons), exact rational dot products, and bisection over fp32 / bf16 bit
patterns.  Agreement of the two on random and adversarial inputs pins the
numpy oracle to the definitions on the Mix-Quant page (gist.science, section
2 "hybrid precision strategy") and the MARLIN page (abeam.tech, group-128
INT4 weights).
"""
from __future__ import annotations

import struct
from fractions import Fraction

E2M1 = [Fraction(v) for v in ("0", "1/2", "1", "3/2", "2", "3", "4", "6")]


def _e4m3(code: int) -> Fraction:
    e, m = code >> 3, code & 7
    return Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)


E4M3 = [_e4m3(c) for c in range(127)]        # codes 0..126; 126 = 448


def _nearest(grid, r: Fraction) -> int:
    """Index of the grid value nearest to r (grid ascending, index = code);
    ties to the even index; beyond the top saturates."""
    best, best_d = 0, None
    for i, g in enumerate(grid):
        d = abs(g - r)
        if best_d is None or d < best_d or (d == best_d and i % 2 == 0):
            best, best_d = i, d
    return best


def _f32_from_bits(b: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", b))[0])


def f32_nearest(q: Fraction) -> Fraction:
    """Nearest fp32 to q > 0 by bisection over positive bit patterns; ties to even bits."""
    lo, hi = 0, 0x7F7FFFFF
    while lo < hi:                                  # largest pattern with value <= q
        mid = (lo + hi + 1) // 2
        if _f32_from_bits(mid) <= q:
            lo = mid
        else:
            hi = mid - 1
    a, b = _f32_from_bits(lo), _f32_from_bits(lo + 1)
    if q - a < b - q or (q - a == b - q and lo % 2 == 0):
        return a
    return b


def _bf16_from_bits(b: int) -> Fraction:
    return _f32_from_bits(b << 16)


def bf16_nearest(q: Fraction) -> int:
    """bf16 bit pattern nearest to q >= 0; ties to even."""
    if q == 0:
        return 0
    lo, hi = 0, 0x7F7F
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if _bf16_from_bits(mid) <= q:
            lo = mid
        else:
            hi = mid - 1
    a, b = _bf16_from_bits(lo), _bf16_from_bits(lo + 1)
    if q - a < b - q or (q - a == b - q and lo % 2 == 0):
        return lo
    return lo + 1


def nvfp4_quantize(x, t_in=None):
    """x: list of rows of Python floats (bf16 values).  Returns (codes, scales, t)."""
    flat = [abs(Fraction(v)) for row in x for v in row]
    amax = max(flat) if flat else Fraction(0)
    if t_in is not None:
        t = Fraction(t_in)
    elif amax == 0:
        t = Fraction(1)
    else:
        t = f32_nearest(amax / 2688)
    codes, scales = [], []
    for row in x:
        crow, srow = [], []
        for b0 in range(0, len(row), 16):
            blk = row[b0:b0 + 16]
            amax_b = max(abs(Fraction(v)) for v in blk)
            s = _nearest(E4M3, amax_b / (6 * t))
            srow.append(s)
            d = E4M3[s] * t
            for v in blk:
                neg = struct.unpack("<I", struct.pack("<f", v))[0] >> 31
                mag = 0 if d == 0 else _nearest(E2M1, abs(Fraction(v)) / d)
                crow.append(mag | (neg << 3))
        codes.append(crow)
        scales.append(srow)
    return codes, scales, t


def nvfp4_value(code: int, s: int, t: Fraction) -> Fraction:
    v = E2M1[code & 7] * E4M3[s] * t
    return -v if code & 8 else v


def nvfp4_gemm(xc, xs, tx, wc, ws, tw):
    """Exact rational Y[m][n] = sum_k xhat[m][k] * what[n][k]."""
    def deq(c, s, t):
        return [[nvfp4_value(c[i][k], s[i][k // 16], t) for k in range(len(c[i]))]
                for i in range(len(c))]
    xh, wh = deq(xc, xs, tx), deq(wc, ws, tw)
    return [[sum(a * b for a, b in zip(xr, wr)) for wr in wh] for xr in xh]


def int4_quantize(w):
    """w: rows of Python floats (bf16 values).  Returns (u codes, scale bf16 bits)."""
    us, ss = [], []
    for row in w:
        urow, srow = [], []
        for g0 in range(0, len(row), 128):
            grp = [Fraction(v) for v in row[g0:g0 + 128]]
            sb = bf16_nearest(max(abs(v) for v in grp) / 7)
            s = _bf16_from_bits(sb)
            srow.append(sb)
            for v in grp:
                if s == 0:
                    q = 0
                else:
                    r = v / s
                    fl = r.numerator // r.denominator
                    rem = r - fl
                    q = fl + 1 if (rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2)) else fl
                    q = max(-8, min(7, q))
                urow.append(q + 8)
        us.append(urow)
        ss.append(srow)
    return us, ss


def w4a16(x, u, s_bits):
    """Exact rational Y[m][n] = sum_k x[m][k] * s[n][k//128] * (u[n][k] - 8)."""
    out = []
    for xr in x:
        orow = []
        for ur, sr in zip(u, s_bits):
            acc = Fraction(0)
            for k, (xv, uv) in enumerate(zip(xr, ur)):
                acc += Fraction(xv) * _bf16_from_bits(sr[k // 128]) * (uv - 8)
            orow.append(acc)
        out.append(orow)
    return out
