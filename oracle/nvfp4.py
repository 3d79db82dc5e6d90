"""CPU oracle for NVFP4 round-to-nearest quantization and the W4A4 GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  It shares
no code with the CUDA path.

What it computes (Mix-Quant page, gist.science, section 2 "hybrid precision
strategy": NVFP4 = 4-bit floats with a local scale per 16-element group plus a
tensor-level scale, quantized by plain round-to-nearest, used for both the
weights and the activations of prefill; section 2.3: the prefill worker runs the
W4A4 NVFP4 path):

  1. amax_T = max |x| over the tensor (exact on bf16 inputs).
  2. t = 1 if amax_T == 0, else fp32_RNE(amax_T / 2688); 2688 = 6 * 448 maps
     the largest block onto the largest E4M3 scale times the largest E2M1 code.
     A caller-fixed t replaces this step.
  3. Per row and 16-element block b along K:
        s_b = E4M3_RNE_satfinite(amax_b / (6 t))  on the exact quotient;
        code = sign(x) | E2M1_RNE_satfinite(|x| / (e4m3(s_b) t)), ties to the
        even code; s_b == 0 gives magnitude 0.
  4. Dequantized value = e2m1(code) * e4m3(s_b) * t, exact in float64.
  5. Y = Xhat @ What^T in float64.

Readings where the pages are silent: t = 1 for an
all-zero tensor; t = amax/2688 in fp32; RNE for both roundings, saturating at
448 and 6; zero codes under a zero scale; the sign of x kept on a zero code;
the low nibble of a byte holds the even-k element.

Exactness: every rounding decision is a comparison of a bf16 value (8
significant bits) with a midpoint times 6t or times e4m3(s) t.  Midpoints have
at most 5 significant bits, the factor 6 two, an E4M3 value four and t 24, so
each product has at most 31 significant bits and is exact in float64; the
comparisons are therefore decided on the exact real values.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

# E2M1 magnitudes of codes 0..7 (sign is bit 3).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
# Midpoints between consecutive E2M1 magnitudes; a tie at midpoint i goes to
# code i+1 when that code is even.
E2M1_MIDPOINTS = (E2M1_MAGNITUDES[:-1] + E2M1_MAGNITUDES[1:]) / 2.0
E4M3_MAX_CODE = 0x7E      # 448; 0x7F is NaN in the FN variant
TENSOR_SCALE_DIVISOR = 2688  # 6 * 448
BLOCK = 16


def e4m3_value(code: int) -> float:
    """Value of a non-negative E4M3 (FN) code: bias 7, 3 mantissa bits, no inf."""
    e, m = (code >> 3) & 0xF, code & 7
    if e == 0:
        return m * 2.0 ** -9
    return (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_VALUES = np.array([e4m3_value(c) for c in range(E4M3_MAX_CODE + 1)])
E4M3_MIDPOINTS = (E4M3_VALUES[:-1] + E4M3_VALUES[1:]) / 2.0


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64, sign of zero kept."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f32_rne(q: Fraction) -> float:
    """Round a positive exact rational to the nearest fp32 value, ties to even."""
    assert q > 0
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    e = max(e, -126)                      # subnormal step below 2^-126
    step = Fraction(2) ** (e - 23)
    n = q / step
    k = n.numerator // n.denominator
    rem = n - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    return float(k * step)


def tensor_scale(x: np.ndarray) -> float:
    """Steps 1-2: t from the tensor's amax (readings R1, R2)."""
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    return tensor_scale_from_amax(amax)


def tensor_scale_from_amax(amax: float) -> float:
    """Step 2 alone, for callers that take max|x| of a tensor too large to hold
    in float64: t = fp32_RN(amax / 2688), or 1 when amax = 0 (R1, R2)."""
    if amax == 0.0:
        return 1.0
    return f32_rne(Fraction(amax) / TENSOR_SCALE_DIVISOR)


def block_scale_codes(amax_b: np.ndarray, t: float) -> np.ndarray:
    """Step 3a: s_b = E4M3_RNE_satfinite(amax_b / (6 t)), decided exactly.

    r > mu_j  <=>  amax_b > mu_j * 6 * t  (exact products).  The code is the
    number of midpoints passed; an exact tie goes to the even code.
    """
    thr = E4M3_MIDPOINTS * 6.0 * t                       # exact, ascending
    a = np.asarray(amax_b, dtype=np.float64)
    below = np.searchsorted(thr, a, side="left")         # midpoints strictly below a
    inb = below < thr.size
    tie = np.zeros(a.shape, dtype=bool)
    tie[inb] = thr[below[inb]] == a[inb]
    up = tie & ((below + 1) % 2 == 0)
    return (below + up).astype(np.uint8)


def element_codes(x: np.ndarray, s: np.ndarray, t: float) -> np.ndarray:
    """Step 3b: 4-bit codes for x [..., nb, 16] with block scale codes s [..., nb]."""
    ax = np.abs(x)
    d = (E4M3_VALUES[s] * t)[..., None]                  # exact, 28 bits at most
    mag = np.zeros(x.shape, dtype=np.uint8)
    for i, mu in enumerate(E2M1_MIDPOINTS):
        thr = mu * d                                     # exact
        passed = (ax > thr) | ((ax == thr) & ((i + 1) % 2 == 0))
        mag += passed.astype(np.uint8)
    mag[(s == 0)[..., None].repeat(x.shape[-1], axis=-1)] = 0
    sign = np.signbit(x).astype(np.uint8) << 3
    return mag | sign


def quantize(x: np.ndarray, t_in: float | None = None):
    """NVFP4 RTN quantization of a [rows, K] float64 array of bf16 values.

    Returns (codes uint8 [rows, K] one 4-bit code per element,
             scales uint8 [rows, K/16] E4M3 codes in logical order,
             t float).
    """
    x = np.asarray(x, dtype=np.float64)
    rows, K = x.shape
    assert K % BLOCK == 0
    t = tensor_scale(x) if t_in is None else float(np.float32(t_in))
    xb = x.reshape(rows, K // BLOCK, BLOCK)
    amax_b = np.max(np.abs(xb), axis=-1)
    s = block_scale_codes(amax_b, t)
    codes = element_codes(xb, s, t).reshape(rows, K)
    return codes, s, t


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte, even k in the low nibble (reading R7)."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def e2m1_signed(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    v = E2M1_MAGNITUDES[c & 7]
    return np.where(c & 8, -v, v)


def dequantize(codes: np.ndarray, scales: np.ndarray, t: float) -> np.ndarray:
    """Step 4: e2m1(code) * e4m3(s) * t, exact in float64 (at most 30 bits)."""
    rows, K = codes.shape
    v = e2m1_signed(codes).reshape(rows, K // BLOCK, BLOCK)
    return (v * (E4M3_VALUES[scales] * t)[..., None]).reshape(rows, K)


def gemm_ref(xhat: np.ndarray, what: np.ndarray) -> np.ndarray:
    """Step 5: Y = Xhat @ What^T in float64 (BLAS dgemm as the library primitive)."""
    return np.asarray(xhat, dtype=np.float64) @ np.asarray(what, dtype=np.float64).T


def gemm_ref_at(xhat_rows: np.ndarray, what_rows: np.ndarray) -> np.ndarray:
    """Y at sampled positions: row i of xhat_rows against row i of what_rows."""
    return np.einsum("ik,ik->i", xhat_rows, what_rows)


# ---------------------------------------------------------------------------
# Scale-factor layout expected by the block-scaled tensor-core MMA.
#
# The block-scaled MMA reads E4M3 scales in 512-byte atoms covering 128 rows x
# 4 consecutive 16-element blocks: inside an atom, row r and block c sit at byte
# 16 * (r % 32) + 4 * (r // 32) + c.  Atoms are stored with the K direction
# fastest.  Rows are padded to a multiple of 128 (padding scales are zero).
# This is the published "128x4" block-scale-factor layout of the Blackwell
# microscaling MMA; it is written here from that description.
# ---------------------------------------------------------------------------

def padded_rows(rows: int) -> int:
    return -(-rows // 128) * 128


def scales_bytes(rows: int, K: int) -> int:
    return padded_rows(rows) * (K // BLOCK)


def scale_offsets(rows: int, K: int, row_index=None) -> np.ndarray:
    """Byte offset of logical scale (r, kb) in the tiled buffer, shape [rows, K/16]
    (or [len(row_index), K/16] for the listed rows only)."""
    assert K % 64 == 0
    r = (np.arange(rows) if row_index is None else np.asarray(row_index, dtype=np.int64))[:, None]
    kb = np.arange(K // BLOCK)[None, :]
    atoms_per_row_tile = K // 64
    atom = (r // 128) * atoms_per_row_tile + kb // 4
    return atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4


def scales_from_tiled(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return np.asarray(buf, dtype=np.uint8).reshape(-1)[scale_offsets(rows, K)]


def scales_to_tiled(s: np.ndarray, rows: int, K: int) -> np.ndarray:
    out = np.zeros(scales_bytes(rows, K), dtype=np.uint8)
    out[scale_offsets(rows, K)] = s
    return out


def within_tolerance(y: np.ndarray, y_ref: np.ndarray, rms: float | None = None):
    """Output bar for the GEMMs: |y - y_ref| <= 8e-3 |y_ref| + 1e-3 rms(y_ref).

    Returns (ok, worst ratio |err| / bound)."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if rms is None:
        rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    bound = 8e-3 * np.abs(y_ref) + 1e-3 * rms
    err = np.abs(y - y_ref)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if y.size else 0.0
    return bool(np.all(err <= bound)), ratio
