"""nvfp4_quantize_noalloc: the quantize entry point for callers that cannot
allocate device memory (an engine whose memory all belongs to its own pool, a
plugin that must not allocate behind its host).  It keeps its scratch in a
fixed device array inside the library.  Checked through the C ABI against the
ordinary entry point on two calls in a row, the second smaller than the first,
so a partial left over in the shared array from the first call would show."""
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
            torch.empty(nvq.nvfp4_scales_bytes(rows, K), dtype=torch.uint8, device="cuda"),
            torch.empty(1, dtype=torch.float32, device="cuda"))


def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from phase_disaggregated_quantized_b200 import build_lib
    build_lib.build()
    L = nvq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    # 2^21 + 2^20 elements first (3 partials), then a small tensor (1 partial).
    for rows, K, seed in ((3 * 1024, 1024, 7), (130, 512, 8)):
        x = synth.activations(rows, K, seed=seed).cuda()
        c, s, t = _outputs(rows, K)
        st = L.nvfp4_quantize_noalloc(vp(x), rows, K, None, vp(c), vp(s), vp(t), stream)
        assert st == 0, L.nvq_last_error_detail()
        rc, rs, rt = nvq.nvfp4_quantize(x)
        nvq.check_device_error()
        np.testing.assert_array_equal(_u8(c), _u8(rc))
        np.testing.assert_array_equal(_u8(s), _u8(rs))
        assert float(t.item()) == float(rt.item())


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = nvq.lib()
    fake = ctypes.c_void_p(0x7F0000000000)
    st = L.nvfp4_quantize_noalloc(fake, 1 << 15, 1 << 16, None, fake, fake, fake, None)
    assert st == 2
    assert b"2^30" in L.nvq_last_error_detail()
