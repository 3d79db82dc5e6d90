"""CPU oracle for INT4 group-128 weight-only quantization and the W4A16 GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  It shares
no code with the CUDA path.

What it computes (MARLIN page, abeam.tech: decode multiplies high-precision
activations by 4-bit weights that carry one scale per group of 128 weights,
"data handling" section; weights and group scales are reordered offline so the
kernel reads them regularly, "weight layout" section):

  s[n, g] = BF16_RNE(amax over w[n, 128g : 128g+128] / 7)
  q[n, k] = clamp(RNE_half_even(w[n, k] / s[n, g]), -8, 7)   (0 when s == 0)
  u[n, k] = q + 8 stored as a nibble, even k in the low nibble
  Y = X @ (s * q)^T in float64.

Exactness of the two roundings done through float64:
  * amax / 7: amax is a bf16 value.  Either 7 divides its significand (the
    quotient is exact) or the quotient's binary expansion repeats with period 3
    (1/7 = 0.001001...b), so it never lies within 2^-53 (relative) of a bf16
    midpoint, whose expansion ends in a single 1 after bit 8.  Rounding the
    float64 quotient to bf16 therefore gives the same result as rounding the
    exact quotient.
  * w / s: w and s are bf16 (8-bit significands) and |w / s| <= 8; if the exact
    quotient is not a half-integer it is at least about 2^-20 (relative) away
    from one, far above float64's 2^-53, so np.rint (half to even) of the
    float64 quotient decides as the exact quotient would.
"""
from __future__ import annotations

import numpy as np

GROUP = 128


def f64_to_bf16_bits_rne(v: np.ndarray) -> np.ndarray:
    """Round float64 values (normal bf16 range or zero) to bf16 bits, ties to even."""
    v = np.asarray(v, dtype=np.float64)
    b = v.view(np.uint64)
    sign = (b >> np.uint64(63)).astype(np.uint64)
    exp = ((b >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    man = (b & np.uint64((1 << 52) - 1)).astype(np.uint64)
    zero = (exp == 0) & (man == 0)
    # bf16 keeps 7 of the 52 stored mantissa bits; round the rest half to even.
    keep = man >> np.uint64(45)
    rest = man & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rest > half) | ((rest == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    keep = keep + up.astype(np.uint64)
    e32 = exp - 1023 + 127 + (keep >> np.uint64(7)).astype(np.int64)
    keep = keep & np.uint64(0x7F)
    assert np.all(zero | ((e32 >= 1) & (e32 <= 254))), "value outside the bf16 normal range"
    bits = (sign << np.uint64(15)) | (e32.clip(0, 255).astype(np.uint64) << np.uint64(7)) | keep
    bits = np.where(zero, sign << np.uint64(15), bits)
    return bits.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def quantize(w: np.ndarray):
    """INT4 g128 RTN of a [N, K] float64 array of bf16 values.

    Returns (u uint8 [N, K] offset-binary codes 0..15, scale bits uint16 [N, K/128])."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    assert K % GROUP == 0
    wg = w.reshape(N, K // GROUP, GROUP)
    amax = np.max(np.abs(wg), axis=-1)
    s_bits = f64_to_bf16_bits_rne(amax / 7.0)
    s = bf16_bits_to_f64(s_bits)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(wg / s[..., None])
    q = np.where(s[..., None] == 0, 0.0, q)
    q = np.clip(q, -8, 7).astype(np.int64)
    u = (q + 8).astype(np.uint8).reshape(N, K)
    return u, s_bits


def pack_nibbles(u: np.ndarray) -> np.ndarray:
    """[N, K] codes -> [N, K/2] bytes, even k in the low nibble."""
    u = np.asarray(u, dtype=np.uint8)
    return (u[:, 0::2] & 0xF) | ((u[:, 1::2] & 0xF) << 4)


def unpack_nibbles(p: np.ndarray) -> np.ndarray:
    p = np.asarray(p, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def dequantize(u: np.ndarray, s_bits: np.ndarray) -> np.ndarray:
    """s * (u - 8), exact in float64."""
    N, K = u.shape
    q = u.astype(np.float64).reshape(N, K // GROUP, GROUP) - 8.0
    return (q * bf16_bits_to_f64(s_bits)[..., None]).reshape(N, K)


def w4a16_ref(x: np.ndarray, what: np.ndarray) -> np.ndarray:
    """Y = X @ What^T in float64."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(what, dtype=np.float64).T


def bytes_ratio_bf16_over_int4_g128(group: int = GROUP, scale_bytes: int = 2) -> float:
    """Bytes per weight of a 16-bit dense weight over 4-bit codes plus one
    16-bit scale per group; the MARLIN page's scale-aware bound on the 4-bit
    speedup (about 3.87x, "weight layout" section)."""
    return 2.0 / (0.5 + scale_bytes / group)


# ---------------------------------------------------------------------------
# Offline reorder of codes and scales for the decode kernel ("weight layout"
# section of the MARLIN page: codes and group scales are permuted ahead of time
# so each thread's loads are regular and land in tensor-core fragment order).
#
# The unit is a tile of 32 weight rows x one 128-wide group: 2048 code bytes
# and 64 scale bytes, stored at unit index (n // 32) * (K / 128) + k // 128.
# The 32 rows are two 16-row tensor-core tiles tt = 0, 1 (rows 16 tt .. 16 tt + 15).
# Inside a unit, 512 little-endian 32-bit words; word (q, lane, comp) at index
# 128 q + 4 lane + comp holds k16-step j = 2 q + comp // 2 of tile tt = comp % 2
# for lane = 4 g + c.  K is permuted inside the group so that lane (g, c)
# covers k = 32c .. 32c+31:
#   nibble p (bits 4p..4p+3), with r = row in the 16-row tile, kk = k within the group:
#     p=0: (g,   32c+4j)    p=4: (g,   32c+4j+1)
#     p=1: (g+8, 32c+4j)    p=5: (g+8, 32c+4j+1)
#     p=2: (g,   32c+4j+2)  p=6: (g,   32c+4j+3)
#     p=3: (g+8, 32c+4j+2)  p=7: (g+8, 32c+4j+3)
# Scale word 2 g + tt (g = 0..7) of a unit holds rows 16 tt + g (low half) and
# 16 tt + g + 8 (high half).
# ---------------------------------------------------------------------------

UNIT_ROWS = 32
_NIBBLE_ROW = np.array([0, 8, 0, 8, 0, 8, 0, 8])     # row offset added to g
_NIBBLE_K = np.array([0, 0, 2, 2, 1, 1, 3, 3])       # k offset added to 32c+4j


def packed_code_index(N: int, K: int):
    """For every (unit, word, nibble) slot, the logical (n, k) it holds.

    Returns arrays n_idx, k_idx of shape [N*K/8, 8] indexed by packed word."""
    G = K // GROUP
    units = (N // UNIT_ROWS) * G
    word = np.arange(512)
    q, lane, comp = word // 128, (word // 4) % 32, word % 4
    j, tt = 2 * q + comp // 2, comp % 2
    g, c = lane // 4, lane % 4
    r = (16 * tt + g)[:, None] + _NIBBLE_ROW[None, :]              # [512, 8]
    kk = (32 * c + 4 * j)[:, None] + _NIBBLE_K[None, :]            # [512, 8]
    unit = np.arange(units)
    nt, gi = unit // G, unit % G
    n_idx = (UNIT_ROWS * nt)[:, None, None] + r[None]              # [units, 512, 8]
    k_idx = (GROUP * gi)[:, None, None] + kk[None]
    return n_idx.reshape(-1, 8), k_idx.reshape(-1, 8)


def _scale_rows(N: int, K: int):
    """Row of every 16-bit scale slot: [units, 32] (slot 2 w + h of scale word w)."""
    G = K // GROUP
    unit = np.arange((N // UNIT_ROWS) * G)
    nt = unit // G
    w = np.arange(16)
    g, tt = w // 2, w % 2
    slot_row = np.stack([16 * tt + g, 16 * tt + g + 8], axis=1).reshape(-1)   # [32]
    return (UNIT_ROWS * nt)[:, None] + slot_row[None, :], (unit % G)[:, None] + 0 * slot_row[None, :]


def unpack_weights(packed_codes: np.ndarray, packed_scales: np.ndarray, N: int, K: int):
    """Inverse of the offline reorder: returns (u [N, K] codes, scale bits [N, K/128])."""
    words = np.frombuffer(np.ascontiguousarray(packed_codes, dtype=np.uint8).tobytes(),
                          dtype="<u4")
    n_idx, k_idx = packed_code_index(N, K)
    u = np.zeros((N, K), dtype=np.uint8)
    for p in range(8):
        u[n_idx[:, p], k_idx[:, p]] = (words >> np.uint32(4 * p)) & np.uint32(0xF)
    G = K // GROUP
    sw = np.frombuffer(np.ascontiguousarray(packed_scales, dtype=np.uint8).tobytes(),
                       dtype="<u2").reshape((N // UNIT_ROWS) * G, 32)
    rows, gis = _scale_rows(N, K)
    s = np.zeros((N, G), dtype=np.uint16)
    s[rows, gis] = sw
    return u, s


def pack_weights(u: np.ndarray, s_bits: np.ndarray):
    """Forward reorder (used to check the GPU's reorder byte for byte)."""
    N, K = u.shape
    n_idx, k_idx = packed_code_index(N, K)
    words = np.zeros(n_idx.shape[0], dtype=np.uint32)
    for p in range(8):
        words |= u[n_idx[:, p], k_idx[:, p]].astype(np.uint32) << np.uint32(4 * p)
    rows, gis = _scale_rows(N, K)
    sw = s_bits[rows, gis].astype(np.uint16)
    return words.view(np.uint8).copy(), sw.reshape(-1).view(np.uint8).copy()