"""CPU oracle for the gate_up GEMM whose epilogue applies SiLU * mul and emits
NVFP4 for the next (down) projection.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  It shares
no code with the CUDA path.

What it computes (Mix-Quant page, gist.science, section 2: the prefill linears
run NVFP4 W4A4, the activations quantized by round-to-nearest with 16-element
E4M3 block scales and a tensor-level FP32 scale; the gated MLP of the Qwen3
family feeds down_proj with silu(x W_gate^T) * (x W_up^T)):

  1. G = Xhat Wg_hat^T, U = Xhat Wu_hat^T exactly in float64 (Xhat, W*_hat the
     dequantized NVFP4 operands, as in the W4A4 oracle).
  2. H = silu(G) * U with silu(g) = g / (1 + exp(-g)), float64.
  3. H quantized to NVFP4 with a caller-fixed tensor scale t_h (reading R15:
     the epilogue cannot see the whole tensor's amax before it writes, so the
     tensor scale is static), by the same exact RTN rules as the activations.

The GPU forms G and U by FP32 tensor-core accumulation, whose order the oracle
cannot reproduce, so H on the GPU differs from H here in its last bits and a
code may land on the other side of a rounding threshold.  ``consistent`` is
therefore the comparison: a GPU block scale or code is accepted when it is the
exact RTN result for some H' within the GEMM error band of H.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4 as onv


def silu(g: np.ndarray) -> np.ndarray:
    """g * sigmoid(g) = g / (1 + exp(-g)), float64."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def gate_up_ref(xhat: np.ndarray, wg_hat: np.ndarray, wu_hat: np.ndarray):
    """Steps 1-2: (G, U, H) in float64."""
    G = onv.gemm_ref(xhat, wg_hat)
    U = onv.gemm_ref(xhat, wu_hat)
    return G, U, silu(G) * U


def silu_prime(g: np.ndarray) -> np.ndarray:
    """d/dg silu(g) = sigmoid(g) (1 + g (1 - sigmoid(g))), float64."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-g))
    return sg * (1.0 + g * (1.0 - sg))


def _silu_second(g: float) -> float:
    sg = 1.0 / (1.0 + np.exp(-g))
    return sg * (1.0 - sg) * (2.0 + g * (1.0 - 2.0 * sg))


def _bisect(f, a: float, b: float) -> float:
    fa = f(a)
    for _ in range(200):
        m = 0.5 * (a + b)
        fm = f(m)
        if (fm > 0) == (fa > 0):
            a, fa = m, fm
        else:
            b = m
    return 0.5 * (a + b)


# silu' has exactly two local extrema (the zeros of silu''): a minimum near
# g = -2.3994 and a maximum near g = +2.3994; it tends to 0 and to 1 at -inf
# and +inf.  So over an interval max |silu'| is attained at an end or at one of
# these two points.
SILU_PRIME_EXTREMA = (_bisect(_silu_second, -4.0, -1.0), _bisect(_silu_second, 1.0, 4.0))


def max_abs_silu_prime(lo: np.ndarray, hi: np.ndarray) -> np.ndarray:
    """max |silu'(g)| over g in [lo, hi] (elementwise, lo <= hi)."""
    m = np.maximum(np.abs(silu_prime(lo)), np.abs(silu_prime(hi)))
    for c in SILU_PRIME_EXTREMA:
        inside = (lo <= c) & (c <= hi)
        m = np.where(inside, np.maximum(m, abs(float(silu_prime(c)))), m)
    return m


def error_band(G: np.ndarray, U: np.ndarray, rel_eval: float = 0.0) -> np.ndarray:
    """Largest |H' - H| for H' = silu(G') U' with G', U' inside the GEMM bar
    (|G' - G| <= dG = 8e-3 |G| + 1e-3 rms(G), the same for U), H = silu(G) U.

    silu(G') U' - silu(G) U = (silu(G') - silu(G)) U' + silu(G) (U' - U), and by
    the mean value theorem |silu(G') - silu(G)| <= L dG with L the largest
    |silu'| over [G - dG, G + dG]; |U'| <= |U| + dU.  Hence
        band = L dG (|U| + dU) + |silu(G)| dU.
    The bound is reached up to the variation of silu' over the interval (the
    signs of G' - G and U' - U can be chosen to align both terms), so it is at
    most about twice the true largest deviation.

    rel_eval adds rel_eval * (|silu(G)| + L dG) (|U| + dU): a relative error of
    the silu evaluation itself, for a comparison with an implementation that
    evaluates silu approximately."""
    G = np.asarray(G, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    dG = 8e-3 * np.abs(G) + 1e-3 * float(np.sqrt(np.mean(G ** 2)))
    dU = 8e-3 * np.abs(U) + 1e-3 * float(np.sqrt(np.mean(U ** 2)))
    L = max_abs_silu_prime(G - dG, G + dG)
    band = L * dG * (np.abs(U) + dU) + np.abs(silu(G)) * dU
    if rel_eval:
        band = band + rel_eval * (np.abs(silu(G)) + L * dG) * (np.abs(U) + dU)
    return band


def _scale_code(amax: np.ndarray, t: float) -> np.ndarray:
    return onv.block_scale_codes(np.asarray(amax, dtype=np.float64), t)


def _mag_code(ax: np.ndarray, s: np.ndarray, t: float) -> np.ndarray:
    """E2M1 magnitude code (0..7) of |x| >= 0 under block scale codes s."""
    return onv.element_codes(np.abs(ax), s, t) & 7


def consistent(codes: np.ndarray, scales: np.ndarray, H: np.ndarray, band: np.ndarray, t: float):
    """GPU output (codes [rows, K] one code per element, scales [rows, K/16]
    logical order) against reference H with per-element error band.

    A block scale passes when it lies between the scale codes of the smallest
    and the largest block amax any H' in the band can have; a code passes when
    its magnitude lies between the magnitude codes of |H| - band and |H| + band
    under the GPU's block scale, and its sign is that of H unless |H| <= band.
    Returns (ok, scale_match_rate, code_match_rate) where the rates count exact
    agreement with the RTN quantization of H itself."""
    H = np.asarray(H, dtype=np.float64)
    band = np.asarray(band, dtype=np.float64)
    rows, K = H.shape
    nb = K // onv.BLOCK
    Hb = np.abs(H).reshape(rows, nb, onv.BLOCK)
    Bb = band.reshape(rows, nb, onv.BLOCK)
    lo = _scale_code(np.max(np.maximum(Hb - Bb, 0.0), axis=-1), t)
    hi = _scale_code(np.max(Hb + Bb, axis=-1), t)
    s = np.asarray(scales, dtype=np.int64)
    ok_s = (lo <= s) & (s <= hi)
    s_u8 = s.astype(np.uint8)
    cb = np.asarray(codes, dtype=np.uint8).reshape(rows, nb, onv.BLOCK)
    mlo = _mag_code(np.maximum(Hb - Bb, 0.0), s_u8, t)
    mhi = _mag_code(Hb + Bb, s_u8, t)
    mag = cb & 7
    ok_m = (mlo <= mag) & (mag <= mhi)
    Hs = H.reshape(rows, nb, onv.BLOCK)
    neg = (cb >> 3) & 1
    sign_free = np.abs(Hs) <= Bb
    ok_sign = sign_free | (neg == np.signbit(Hs).astype(np.uint8))
    ref_codes, ref_s, _ = onv.quantize(H, t_in=t)
    ok = bool(np.all(ok_s) and np.all(ok_m & ok_sign))
    s_rate = float(np.mean(ref_s == s)) if s.size else 1.0
    c_rate = float(np.mean(ref_codes.reshape(rows, nb, onv.BLOCK) == cb)) if cb.size else 1.0
    return ok, s_rate, c_rate
