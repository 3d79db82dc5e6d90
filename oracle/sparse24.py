"""CPU oracle for the 2:4-sparse INT4 group-128 weight-only decode GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  It shares
no code with the CUDA path.

What it computes (MARLIN page, abeam.tech: the official implementation also
combines the INT4 group-128 weights with 2:4 structured sparsity, Sparse-MARLIN;
the decode GEMM itself is the W4A16 one of ``oracle/int4.py``):

  1. 2:4 pruning of the BF16 master W [N, K] (reading R17): in every run of 4
     consecutive k of a row keep the 2 entries of largest |w|; among equal
     magnitudes the lower k wins.  The other two become 0.
  2. INT4 group-128 RTN of the pruned W exactly as ``int4.quantize``.  A run's
     largest |w| is always kept, so each group's scale equals the dense one,
     and a kept entry's code equals its dense code.
  3. Logical sparse form: for each row and run r, the kept positions
     i0 < i1 (0..3) as the nibble i0 | i1 << 2, and the two kept codes u.
  4. Y = X @ (s * (u - 8) at the kept positions, 0 elsewhere)^T in float64.

Kernel order (``pack``): the 32-row x 128-k group "unit" of the decode kernel
is two 16-row tiles tt = 0, 1 (rows 16 tt .. 16 tt + 15), each 512 bytes of
codes then 256 bytes of metadata (1536 bytes per unit), and 64 bytes of
scales: 32-bit word 2 g + tt holds rows 16 tt + g (low half) and 16 tt + g + 8
(high half).  Inside a tile the m16n8k32 sparse MMA step s (0..3) reads the runs
G(s, j) = 8 s + j / 2 for even j and 8 s + 4 + (j - 1) / 2 for odd j (MMA
run j = 0..7); lane (g, c) holds, for step s, one 32-bit word whose nibble
i (bits 4i..4i+3) and nibble i + 4 are the two compressed values of its A
fragment register i: register 0 = row g, compressed k 2c and 2c + 1; register
1 = row g + 8, same k; registers 2 and 3 = the same rows at compressed k
2c + 8 and 2c + 9 (compressed k 2j, 2j + 1 = the two kept entries of MMA run
j).  Lanes c = 0, 1 also hold one metadata word per step: nibble n is the run
descriptor of row g + 8 (n // 4) and MMA run 4 c + n % 4.
"""
from __future__ import annotations

import numpy as np

from . import int4 as oint4

RUN = 4
UNIT_ROWS = 32
UNIT_CODE_BYTES = 512
UNIT_META_BYTES = 256


def prune24(w: np.ndarray):
    """Step 1: (pruned float64 array, keep mask bool) for w [N, K], K % 4 == 0."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    assert K % RUN == 0
    a = np.abs(w).reshape(N, K // RUN, RUN)
    keep = np.zeros(a.shape, dtype=bool)
    for r in range(a.shape[1]):
        blk = a[:, r, :]
        # stable sort by decreasing magnitude: equal magnitudes keep index order
        order = np.argsort(-blk, axis=1, kind="stable")
        rows = np.arange(N)
        keep[rows, r, order[:, 0]] = True
        keep[rows, r, order[:, 1]] = True
    keep = keep.reshape(N, K)
    return np.where(keep, w, 0.0), keep


def quantize(w: np.ndarray):
    """Steps 1-3: (u_kept [N, K/2], meta [N, K/4] nibbles, s_bits [N, K/128], keep [N, K])."""
    pruned, keep = prune24(w)
    u, s_bits = oint4.quantize(pruned)
    N, K = pruned.shape
    kr = keep.reshape(N, K // RUN, RUN)
    pos = np.argsort(~kr, axis=2, kind="stable")[:, :, :2]     # kept positions, ascending
    i0, i1 = pos[:, :, 0], pos[:, :, 1]
    meta = (i0 | (i1 << 2)).astype(np.uint8)
    ur = u.reshape(N, K // RUN, RUN)
    kept = np.stack([np.take_along_axis(ur, i0[..., None], 2)[..., 0],
                     np.take_along_axis(ur, i1[..., None], 2)[..., 0]], axis=2).reshape(N, K // 2)
    return kept.astype(np.uint8), meta, s_bits, keep


def dense_codes(u_kept: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """Logical sparse form -> dense codes [N, K] with u = 8 (value 0) at dropped positions."""
    N, half = u_kept.shape
    K = 2 * half
    u = np.full((N, K // RUN, RUN), 8, dtype=np.uint8)
    kr = u_kept.reshape(N, K // RUN, 2)
    i0, i1 = meta & 3, (meta >> 2) & 3
    np.put_along_axis(u, i0[..., None].astype(np.int64), kr[..., 0:1], 2)
    np.put_along_axis(u, i1[..., None].astype(np.int64), kr[..., 1:2], 2)
    return u.reshape(N, K)


def w4a16_ref(x: np.ndarray, u_kept: np.ndarray, meta: np.ndarray, s_bits: np.ndarray) -> np.ndarray:
    """Step 4."""
    return oint4.w4a16_ref(x, oint4.dequantize(dense_codes(u_kept, meta), s_bits))


def _mma_run(s: int, j: int) -> int:
    """Run (0..31) of the 128-k group read by MMA step s, MMA run j."""
    return 8 * s + (j // 2 if j % 2 == 0 else 4 + (j - 1) // 2)


def _tile_words(kr: np.ndarray, meta: np.ndarray, r0: int, gi: int):
    """Code words (32 lanes x 4 steps) and metadata words (16 lanes x 4 steps) of
    the 16-row tile starting at row r0, group gi."""
    codes = np.zeros(128, dtype=np.uint32)
    metaw = np.zeros(64, dtype=np.uint32)
    for lane in range(32):
        g, c = lane >> 2, lane & 3
        for s in range(4):
            w = 0
            for reg in range(4):
                row = r0 + g + (8 if reg & 1 else 0)
                kc = 2 * c + (8 if reg & 2 else 0)           # compressed k of the register's low half
                for half_i, kk in enumerate((kc, kc + 1)):
                    j, q = kk // 2, kk % 2
                    run = 128 // RUN * gi + _mma_run(s, j)
                    w |= int(kr[row, run, q]) << (4 * (reg + 4 * half_i))
            codes[4 * lane + s] = w
            if c < 2:
                m = 0
                for n in range(8):
                    row = r0 + g + 8 * (n // 4)
                    run = 128 // RUN * gi + _mma_run(s, 4 * c + n % 4)
                    m |= int(meta[row, run]) << (4 * n)
                metaw[4 * (2 * g + c) + s] = m
    return codes, metaw


def pack(u_kept: np.ndarray, meta: np.ndarray, s_bits: np.ndarray):
    """Kernel order: (codes_and_meta uint8 [units * 1536], scales uint8 [units * 64]),
    units in (32-row tile, 128-k group) order, tile-major."""
    N, half = u_kept.shape
    K = 2 * half
    assert N % UNIT_ROWS == 0 and K % 128 == 0
    G = K // 128
    kr = u_kept.reshape(N, K // RUN, 2)
    tb = UNIT_CODE_BYTES + UNIT_META_BYTES
    out = np.zeros((N // UNIT_ROWS, G, 2, tb), dtype=np.uint8)
    sc = np.zeros((N // UNIT_ROWS, G, 16, 2), dtype=np.uint16)
    for nt in range(N // UNIT_ROWS):
        for gi in range(G):
            for tt in range(2):
                codes, metaw = _tile_words(kr, meta, UNIT_ROWS * nt + 16 * tt, gi)
                out[nt, gi, tt, :UNIT_CODE_BYTES] = codes.view(np.uint8)
                out[nt, gi, tt, UNIT_CODE_BYTES:] = metaw.view(np.uint8)
                for g in range(8):
                    sc[nt, gi, 2 * g + tt, 0] = s_bits[UNIT_ROWS * nt + 16 * tt + g, gi]
                    sc[nt, gi, 2 * g + tt, 1] = s_bits[UNIT_ROWS * nt + 16 * tt + g + 8, gi]
    return out.reshape(-1), sc.reshape(-1).view(np.uint8).copy()


def unpack(packed: np.ndarray, packed_scales: np.ndarray, N: int, K: int):
    """Inverse of ``pack``: (u_kept, meta, s_bits)."""
    G = K // 128
    tb = UNIT_CODE_BYTES + UNIT_META_BYTES
    p = np.asarray(packed, dtype=np.uint8).reshape(N // UNIT_ROWS, G, 2, tb)
    u = np.zeros((N, K // RUN, 2), dtype=np.uint8)
    meta = np.zeros((N, K // RUN), dtype=np.uint8)
    for nt in range(N // UNIT_ROWS):
        for gi in range(G):
            for tt in range(2):
                r0 = UNIT_ROWS * nt + 16 * tt
                codes = p[nt, gi, tt, :UNIT_CODE_BYTES].copy().view(np.uint32)
                metaw = p[nt, gi, tt, UNIT_CODE_BYTES:].copy().view(np.uint32)
                for lane in range(32):
                    g, c = lane >> 2, lane & 3
                    for s in range(4):
                        w = int(codes[4 * lane + s])
                        for reg in range(4):
                            row = r0 + g + (8 if reg & 1 else 0)
                            kc = 2 * c + (8 if reg & 2 else 0)
                            for half_i, kk in enumerate((kc, kc + 1)):
                                j, q = kk // 2, kk % 2
                                run = 128 // RUN * gi + _mma_run(s, j)
                                u[row, run, q] = (w >> (4 * (reg + 4 * half_i))) & 0xF
                        if c < 2:
                            m = int(metaw[4 * (2 * g + c) + s])
                            for n in range(8):
                                row = r0 + g + 8 * (n // 4)
                                run = 128 // RUN * gi + _mma_run(s, 4 * c + n % 4)
                                meta[row, run] = (m >> (4 * n)) & 0xF
    sc = np.asarray(packed_scales, dtype=np.uint8).copy().view(np.uint16).reshape(N // UNIT_ROWS, G, 16, 2)
    s_bits = np.zeros((N, G), dtype=np.uint16)
    for nt in range(N // UNIT_ROWS):
        for w in range(16):
            g, tt = w // 2, w % 2
            s_bits[UNIT_ROWS * nt + 16 * tt + g] = sc[nt, :, w, 0]
            s_bits[UNIT_ROWS * nt + 16 * tt + g + 8] = sc[nt, :, w, 1]
    return u.reshape(N, K // 2), meta, s_bits
