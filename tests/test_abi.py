"""The C-ABI library: loads without a GPU, exports every declared entry point,
and rejects bad arguments on the host before touching the device."""
import ctypes
import os

import pytest

import phase_disaggregated_quantized_b200 as nvq
from phase_disaggregated_quantized_b200 import build_lib


@pytest.fixture(scope="module")
def L():
    build_lib.build()
    return nvq.lib()


def test_header_lists_the_entry_points():
    names = nvq.header_functions()
    for must in ("nvfp4_quantize", "nvfp4_gemm_w4a4", "int4_pack_weights", "w4a16_gemm", "int4_quantize",
                 "nvq_check_device_error", "nvq_selftest_wait_timeout", "nvfp4_scales_bytes",
                 "nvfp4_amax", "nvfp4_scale_from_amax", "nvfp4_scale_offset", "nvq_workspace_bytes",
                 "w4a16_workspace_bytes"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in nvq.header_functions():
        assert hasattr(L, name), name


def test_abi_version_and_status_strings(L):
    assert L.nvq_abi_version() == 1
    for code, name in nvq.STATUS.items():
        assert L.nvq_status_string(code).decode() == name


def test_size_helpers(L):
    assert L.nvfp4_scales_bytes(1, 64) == 128 * 4
    assert L.nvfp4_scales_bytes(130, 512) == 256 * 32
    assert L.nvfp4_scales_bytes(10, 100) == 0          # K % 64 != 0
    assert L.nvfp4_quantize_workspace_bytes(0, 64) == 0
    assert L.nvfp4_quantize_workspace_bytes(128, 512) > 0
    assert L.w4a16_workspace_bytes(1, 4096, 4096) == 0          # partial sums stay on chip
    assert L.w4a16_workspace_bytes(4, 256, 4096) == 0
    assert L.w4a16_workspace_bytes(4096, 4096, 4096) == 0


def test_scale_offset_map_matches_the_oracles_layout(L):
    import numpy as np
    from oracle import nvfp4 as onv
    for rows, K in ((1, 64), (130, 512), (300, 192), (256, 1024)):
        want = onv.scale_offsets(rows, K)
        got = np.array([[L.nvfp4_scale_offset(r, kb, rows, K) for kb in range(K // 16)] for r in range(rows)])
        np.testing.assert_array_equal(got, want)
        assert sorted(got.ravel().tolist()) == sorted(set(got.ravel().tolist()))     # one byte per scale
        assert got.max() < L.nvfp4_scales_bytes(rows, K)
    for bad in ((-1, 0, 4, 64), (4, 0, 4, 64), (0, 4, 4, 64), (0, -1, 4, 64), (0, 0, 4, 100), (0, 0, 0, 64)):
        assert L.nvfp4_scale_offset(*bad) == -1


def test_workspace_bytes_by_operation(L):
    assert L.nvq_workspace_bytes(0, 8192, 0, 4096) == L.nvfp4_quantize_workspace_bytes(8192, 4096) > 0
    assert L.nvq_workspace_bytes(1, 8192, 4096, 4096) == 0
    assert L.nvq_workspace_bytes(2, 16, 4096, 4096) == L.w4a16_workspace_bytes(16, 4096, 4096) == 0
    assert L.nvq_workspace_bytes(3, 4096, 24576, 4096) == L.nvq_linear_workspace_bytes(4096, 24576, 4096, -1) > 0
    assert L.nvq_workspace_bytes(3, 1, 24576, 4096) == 0
    assert L.nvq_workspace_bytes(7, 1, 1, 64) == 2 ** 64 - 1


FAKE = 0x7F0000000000          # 16-byte aligned, never dereferenced: validation fails first
ODD = FAKE + 8


def _vp(v):
    return ctypes.c_void_p(v)


def test_quantize_rejects_bad_arguments(L):
    q = L.nvfp4_quantize
    assert q(_vp(FAKE), 4, 100, None, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, 0, None) == 2   # K % 64
    assert q(_vp(FAKE), -1, 64, None, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, 0, None) == 1
    assert q(_vp(FAKE), 4, 64, None, _vp(FAKE), _vp(FAKE), None, None, 0, None) == 1          # no t_out
    assert q(_vp(ODD), 4, 64, None, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, 0, None) == 3
    assert q(_vp(FAKE), 4, 64, None, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, 0, None) == 4     # workspace
    assert q(_vp(FAKE), 4, 64, None, _vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE), 2, None) == 4
    assert b"workspace" in L.nvq_last_error_detail()


def test_size_limits_keep_the_kernel_counters_from_wrapping(L):
    # rows * K / 16 = 2^31 blocks: one past the limit of one quantize call
    assert L.nvfp4_quantize(_vp(FAKE), 1 << 25, 1024, None, _vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE),
                            1 << 20, None) == 2
    assert L.nvfp4_quantize(_vp(FAKE), (1 << 25) - 1, 1024, None, _vp(FAKE), _vp(FAKE), _vp(FAKE), None,
                            0, None) == 4     # just inside: reaches the workspace check
    # (M / 128) * (N / 128) = 2^31 output blocks
    assert L.nvfp4_gemm_w4a4(*([_vp(FAKE)] * 7), 1 << 24, 1 << 21, 64, None) == 2


def test_gemm_rejects_bad_arguments(L):
    g = L.nvfp4_gemm_w4a4
    a = [_vp(FAKE)] * 7
    assert g(*a, 128, 12, 512, None) == 2            # N % 8
    assert g(*a, 128, 512, 96, None) == 2            # K % 64
    assert g(*a, -1, 512, 512, None) == 1
    b = list(a)
    b[6] = _vp(ODD)
    assert g(*b, 128, 512, 512, None) == 3
    b = list(a)
    b[0] = None
    assert g(*b, 128, 512, 512, None) == 1


def test_int4_calls_reject_bad_arguments(L):
    assert L.int4_quantize(_vp(FAKE), 16, 100, _vp(FAKE), _vp(FAKE), None) == 2
    assert L.int4_pack_weights(_vp(FAKE), _vp(FAKE), 48, 128, _vp(FAKE), _vp(FAKE), None) == 2   # N % 32
    assert L.int4_pack_weights(_vp(ODD), _vp(FAKE), 32, 128, _vp(FAKE), _vp(FAKE), None) == 3
    w = L.w4a16_gemm
    assert w(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE), 4, 24, 128, None, 0, None) == 2
    assert w(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE), 4, 48, 128, None, 0, None) == 2     # N % 32
    assert w(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(ODD), 4, 256, 4096, None, 0, None) == 3    # y misaligned
    assert w(_vp(FAKE), _vp(FAKE), None, _vp(FAKE), 4, 256, 4096, None, 0, None) == 1         # NULL scales


def test_row_shard_calls_reject_bad_arguments(L):
    a = L.nvfp4_amax
    assert a(_vp(FAKE), 4, 100, _vp(FAKE), _vp(FAKE), 1 << 20, None) == 2          # K % 64
    assert a(_vp(FAKE), -1, 64, _vp(FAKE), _vp(FAKE), 1 << 20, None) == 1
    assert a(_vp(FAKE), 4, 64, None, _vp(FAKE), 1 << 20, None) == 1                 # no amax_out
    assert a(_vp(ODD), 4, 64, _vp(FAKE), _vp(FAKE), 1 << 20, None) == 3
    assert a(_vp(FAKE), 4, 64, _vp(FAKE + 2), _vp(FAKE), 1 << 20, None) == 3        # amax_out not 4-aligned
    assert a(_vp(FAKE), 4, 64, _vp(FAKE), None, 0, None) == 4                       # workspace
    assert a(_vp(FAKE), 4, 64, _vp(FAKE), _vp(FAKE), 0, None) == 4
    f = L.nvfp4_scale_from_amax
    assert f(None, _vp(FAKE), None) == 1
    assert f(_vp(FAKE), None, None) == 1
    assert f(_vp(FAKE + 1), _vp(FAKE), None) == 3


def test_timeout_selftest_rejects_limits_out_of_range(L):
    assert L.nvq_selftest_wait_timeout(999, None) == 1              # below 1 us: nothing launched
    assert L.nvq_selftest_wait_timeout(100_000_001, None) == 1      # above 100 ms
    assert b"limit_ns" in L.nvq_last_error_detail()


def test_zero_sized_calls_are_noops(L):
    assert L.nvfp4_gemm_w4a4(*([_vp(FAKE)] * 7), 0, 512, 512, None) == 0
    assert L.w4a16_gemm(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE), 0, 512, 512, None, 0, None) == 0
    assert L.int4_quantize(_vp(FAKE), 0, 128, _vp(FAKE), _vp(FAKE), None) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(nvq, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(nvq, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        nvq.lib()


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.dirname(nvq.__file__)
    for root, _dirs, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_phase_dispatch_host_rules(L):
    """nvq_linear: path choice by M, workspace sizing and argument checks (no GPU)."""
    c = L.nvq_default_crossover_m()
    assert c >= 1
    assert L.nvq_linear_workspace_bytes(c, 24576, 4096, -1) == 0               # W4A16 side: no scratch
    big = L.nvq_linear_workspace_bytes(c + 1, 24576, 4096, -1)
    assert big >= (c + 1) * 4096 // 2 + L.nvfp4_scales_bytes(c + 1, 4096)       # codes + scales at least
    assert L.nvq_linear_workspace_bytes(64, 24576, 4096, 128) == 0              # caller's crossover wins
    f = L.nvq_linear
    # W4A16 side without the packed weights / W4A4 side without the NVFP4 weights
    assert f(_vp(FAKE), 1, 256, 4096, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, None, -1,
             _vp(FAKE), None, 0, None) == 1
    assert f(_vp(FAKE), 4096, 256, 4096, None, None, None, _vp(FAKE), _vp(FAKE), -1,
             _vp(FAKE), _vp(FAKE), 1 << 30, None) == 1
    # W4A4 side: workspace too small, misaligned, bad K
    assert f(_vp(FAKE), 4096, 256, 4096, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, None, -1,
             _vp(FAKE), _vp(FAKE), 16, None) == 4
    assert f(_vp(FAKE), 4096, 256, 4096, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, None, -1,
             _vp(FAKE), _vp(ODD), 1 << 30, None) == 3
    assert f(_vp(FAKE), 4096, 256, 4100, _vp(FAKE), _vp(FAKE), _vp(FAKE), None, None, -1,
             _vp(FAKE), _vp(FAKE), 1 << 30, None) == 2
    # W4A16 side keeps its own shape rules (N % 32)
    assert f(_vp(FAKE), 1, 48, 4096, None, None, None, _vp(FAKE), _vp(FAKE), -1,
             _vp(FAKE), None, 0, None) == 2


def test_prefill_streamed_host_rules(L):
    """nvq_prefill_streamed: workspace sizing and argument checks (no GPU)."""
    import phase_disaggregated_quantized_b200 as nvq
    def layers(*shapes, bad=None):
        arr = (nvq.StreamLayer * len(shapes))()
        for i, (N, K) in enumerate(shapes):
            arr[i] = nvq.StreamLayer(FAKE, FAKE, FAKE, FAKE, FAKE, N, K)
        if bad is not None:
            setattr(arr[0], bad, None)
        return arr
    one = L.nvq_prefill_streamed_workspace_bytes(layers((4096, 4096)), 1, 8192)
    two = L.nvq_prefill_streamed_workspace_bytes(layers((4096, 4096), (24576, 4096)), 2, 8192)
    assert one > 2 * 4096 * 2048 and two > one                      # two weight slots for the largest layer
    assert two >= 2 * 24576 * 2048 + 8192 * 2048
    s = L.nvq_prefill_streamed
    assert s(layers((4096, 4096)), 0, 8192, _vp(FAKE), 1 << 40, None, None) == 1     # no layers
    assert s(layers((4096, 4096), bad="w_t_host"), 1, 8192, _vp(FAKE), 1 << 40, None, None) == 1
    assert s(layers((4100, 4096)), 1, 8192, _vp(FAKE), 1 << 40, None, None) == 2    # N % 8
    assert s(layers((4096, 4100)), 1, 8192, _vp(FAKE), 1 << 40, None, None) == 2    # K % 64
    assert s(layers((4096, 4096)), 1, 8192, _vp(FAKE), 16, None, None) == 4         # workspace
    assert s(layers((4096, 4096)), 1, 8192, _vp(ODD), 1 << 40, None, None) == 3     # alignment


def test_swiglu_gemm_host_rules(L):
    f = L.nvfp4_gemm_w4a4_swiglu
    P = [_vp(FAKE)] * 9
    assert f(*P, 128, 384, 512, None) == 2                   # N % 256
    assert f(*P, 128, 512, 100, None) == 2                   # K % 64
    Pn = list(P)
    Pn[6] = None                                             # t_h
    assert f(*Pn, 128, 512, 512, None) == 1
    Pm = list(P)
    Pm[7] = _vp(ODD)                                         # h_codes misaligned
    assert f(*Pm, 128, 512, 512, None) == 3
    assert f(*P, 0, 512, 512, None) == 0                     # M = 0: nothing to do


def test_sparse24_host_rules(L):
    p = L.int4_pack_sparse24
    assert p(_vp(FAKE), _vp(FAKE), _vp(FAKE), 24, 128, _vp(FAKE), _vp(FAKE), None) == 2      # N % 32
    assert p(_vp(FAKE), _vp(FAKE), _vp(FAKE), 48, 128, _vp(FAKE), _vp(FAKE), None) == 2
    assert p(_vp(FAKE), _vp(FAKE), _vp(FAKE), 32, 100, _vp(FAKE), _vp(FAKE), None) == 2      # K % 128
    assert p(_vp(FAKE), None, _vp(FAKE), 32, 128, _vp(FAKE), _vp(FAKE), None) == 1
    assert p(_vp(FAKE), _vp(FAKE), _vp(FAKE), 32, 128, _vp(ODD), _vp(FAKE), None) == 3
    g = L.w4a16_sparse24_gemm
    assert g(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE), 4, 24, 128, None) == 2
    assert g(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE), 4, 48, 128, None) == 2
    assert g(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(ODD), 4, 256, 4096, None) == 3
    assert g(_vp(FAKE), None, _vp(FAKE), _vp(FAKE), 4, 256, 4096, None) == 1
    assert g(_vp(FAKE), _vp(FAKE), _vp(FAKE), _vp(FAKE), 0, 256, 4096, None) == 0
