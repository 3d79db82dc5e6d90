"""nvfp4_quantize_noalloc: the quantize entry point for callers that cannot
allocate device memory (an engine whose memory all belongs to its own pool, a
plugin that must not allocate behind its host).  It keeps its scratch in a
fixed device array inside the library.  Checked through the C ABI against the
ordinary entry point, bit for bit:

  * two computed-scale calls in a row, the second with fewer amax partials
    (but more than one) and a much smaller max|x| than the first, so a partial
    left over in the shared array from the first call would raise the second
    call's tensor scale;
  * a call with a caller-fixed tensor scale (no amax pre-pass);
  * a call with zero rows, which writes only the tensor scale.
"""
import ctypes

import numpy as np
import pytest
import torch

import phase_disaggregated_quantized_b200 as nvq
from phase_disaggregated_quantized_b200 import synth

pytestmark = pytest.mark.gpu


def _u8(t):
    return t.detach().cpu().numpy()


def _outputs(rows, K):
    return (torch.empty(rows, K // 2, dtype=torch.uint8, device="cuda"),
            torch.empty(max(nvq.nvfp4_scales_bytes(rows, K), 16), dtype=torch.uint8, device="cuda"),
            torch.empty(1, dtype=torch.float32, device="cuda"))


def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from phase_disaggregated_quantized_b200 import build_lib
    build_lib.build()
    L = nvq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L, stream


def _vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _same(L, stream, x, rows, K, t_in=None):
    c, s, t = _outputs(rows, K)
    st = L.nvfp4_quantize_noalloc(_vp(x), rows, K, _vp(t_in), _vp(c), _vp(s), _vp(t), stream)
    assert st == 0, L.nvq_last_error_detail()
    rc, rs, rt = nvq.nvfp4_quantize(x, t_in)
    nvq.check_device_error()
    np.testing.assert_array_equal(_u8(c), _u8(rc))
    np.testing.assert_array_equal(_u8(s)[:rs.numel()], _u8(rs))
    assert float(t.item()) == float(rt.item())
    return float(t.item())


def test_noalloc_matches_workspace_entry_point_twice():
    L, stream = _setup()
    # 2^22 elements (512 amax partials) with outliers x20, then 2^18 elements
    # (32 partials) scaled down 100x: a stale partial would show in t.
    x1 = synth.activations(4096, 1024, seed=7).cuda()
    t1 = _same(L, stream, x1, 4096, 1024)
    x2 = (synth.activations(256, 1024, seed=8).cuda().float() * 0.01).to(torch.bfloat16)
    t2 = _same(L, stream, x2, 256, 1024)
    assert t2 < t1 / 10


def test_noalloc_caller_scale_and_empty_tensor():
    L, stream = _setup()
    x = synth.activations(130, 512, seed=9).cuda()
    t_in = torch.tensor([0.004], dtype=torch.float32, device="cuda")
    _same(L, stream, x, 130, 512, t_in)
    # zero rows: nothing to quantize, the tensor scale is still written (1, or the caller's)
    empty = torch.zeros(0, 512, dtype=torch.bfloat16, device="cuda")
    t = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    st = L.nvfp4_quantize_noalloc(_vp(empty), 0, 512, None, None, None, _vp(t), stream)
    assert st == 0, L.nvq_last_error_detail()
    torch.cuda.synchronize()
    assert float(t.item()) == 1.0
    nvq.check_device_error()


def test_noalloc_rejects_sizes_beyond_its_limit():
    L = nvq.lib()
    # NULL pointers: the size check comes first, and nothing is launched either way.
    st = L.nvfp4_quantize_noalloc(None, 1 << 15, 1 << 16, None, None, None, None, None)
    assert st == 2
    assert b"2^30" in L.nvq_last_error_detail()
