"""Shared test plumbing: tensor <-> numpy conversion and oracle calls on inputs
drawn by the seeded generators.  Holds no quantization arithmetic."""
import numpy as np
import torch

from oracle import int4 as oint4
from oracle import nvfp4 as onv


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 tensor (sign of zero kept)."""
    bits = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return onv.bf16_bits_to_f64(bits)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint8)


def oracle_nvfp4(x: torch.Tensor, t_in=None):
    """Oracle quantization of a bf16 tensor: (packed codes [rows, K/2], logical scales, t)."""
    codes, s, t = onv.quantize(bf16_to_f64(x), t_in=t_in)
    return onv.pack_codes(codes), s, t


def oracle_int4(w: torch.Tensor):
    u, s_bits = oint4.quantize(bf16_to_f64(w))
    return u, s_bits
