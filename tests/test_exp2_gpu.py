"""The FMA-pipe exponential that the attention softmax uses for one
probability pair in four, evaluated on the device through its self-check
entry point and compared with exact values and with the hardware ex2.approx."""
import numpy as np
import pytest
import torch

from latent_attention_jagged_b200 import binding

pytestmark = pytest.mark.gpu


def _eval(x_np):
    x = torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).cuda()
    y, y_hw = binding.exp2_eval(x)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), y_hw.cpu().numpy().astype(np.float64)


def test_relative_error_over_the_softmax_range():
    # the softmax feeds s - m <= 8 (lazy rescale threshold); cover far beyond
    x = np.concatenate([np.linspace(-124.5, 64.0, 1_000_001),
                        np.random.default_rng(0).uniform(-30.0, 8.0, 200_001)]).astype(np.float32)
    y, y_hw = _eval(x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y / exact - 1.0)
    assert rel.max() < 1e-4, rel.max()
    # and against CUDA's own approximation of the same function
    rel_hw = np.abs(y / y_hw - 1.0)
    assert rel_hw.max() < 1.2e-4, rel_hw.max()


def test_integers_halves_and_odd_length():
    x = np.concatenate([np.arange(-124, 65), np.arange(-124, 64) + 0.5]).astype(np.float32)
    assert x.size % 2 == 1
    y, _ = _eval(x)
    exact = np.exp2(x.astype(np.float64))
    assert np.abs(y / exact - 1.0).max() < 1e-4


def test_very_negative_and_non_finite_inputs_give_zero():
    # a masked score reaches the exponential as -inf and must give exactly 0
    x = np.array([-125.0, -126.0, -200.0, -1e30, -np.inf, np.nan], dtype=np.float32)
    y, y_hw = _eval(x)
    assert np.all(y == 0.0)
    assert y_hw[4] == 0.0
    # just above the cut the value is the ordinary one
    y2, _ = _eval(np.array([-124.75, -124.0], dtype=np.float32))
    assert np.abs(y2 / np.exp2([-124.75, -124.0]) - 1.0).max() < 1e-4
