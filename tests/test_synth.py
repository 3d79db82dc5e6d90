"""The seeded input generators follow the stated recipe and hold no method
arithmetic (they are the one module both the oracle and the CUDA path use)."""
import inspect

import torch

from phase_disaggregated_quantized_b200 import synth


def test_outlier_channel_counts():
    # 0.1 % of the channels, at least one, for the Qwen3-8B / -32B hidden sizes
    assert [synth.n_outlier_channels(K) for K in (4096, 12288, 5120, 8192, 25600, 512)] == [4, 12, 5, 8, 26, 1]


def test_activations_seeded_shapes_and_outliers():
    a = synth.activations(512, 4096, seed=7)
    b = synth.activations(512, 4096, seed=7)
    c = synth.activations(512, 4096, seed=8)
    assert a.dtype == torch.bfloat16 and a.shape == (512, 4096)
    assert torch.equal(a, b) and not torch.equal(a, c)
    std = a.float().std(dim=0)
    big = torch.nonzero(std > 5.0).flatten()
    assert big.numel() == 4                                   # the outlier channels
    assert torch.all((std[big] > 15.0) & (std[big] < 25.0))  # gain 20 on N(0, 1)
    rest = torch.ones(4096, dtype=torch.bool)
    rest[big] = False
    assert abs(float(std[rest].mean()) - 1.0) < 0.02


def test_weights_scale_and_seed():
    w = synth.weights(1024, 1024, seed=3)
    assert w.dtype == torch.bfloat16 and w.shape == (1024, 1024)
    assert abs(float(w.float().std()) - 0.02) < 0.001
    assert torch.equal(w, synth.weights(1024, 1024, seed=3))
    assert not torch.equal(w, synth.weights(1024, 1024, seed=4))


def test_tiny_case_shapes():
    x, w = synth.tiny_case()
    assert x.shape == (128, 512) and w.shape == (512, 512)


def test_generators_hold_no_method_code():
    src = inspect.getsource(synth)
    for word in ("import oracle", "from oracle", "libnvq", "nvq.", "e2m1", "e4m3", "quantiz("):
        assert word not in src, word
