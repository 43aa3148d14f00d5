"""The softmax's FMA-pipe 2^x (range reduction + fitted cubic) against exp2."""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3

pytestmark = pytest.mark.gpu


def test_exp2_polynomial_error_bound():
    grid = np.linspace(-125.0, 8.0, 1 << 20, dtype=np.float32)
    edges = np.concatenate([np.arange(-125, 9, dtype=np.float32),                  # integers
                            np.arange(-125, 8, dtype=np.float32) + np.float32(0.5),  # rounding ties
                            np.array([0.0, -0.0, 1e-7, -1e-7, 7.999], np.float32)])
    x = np.concatenate([grid, edges]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    y = h3.selftest_exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 1e-4, (rel.max(), x[np.argmax(rel)])


def test_exp2_polynomial_clamps_tiny_inputs():
    x = np.array([-126.0, -200.0, -1e30, -125.0], np.float32)
    y = h3.selftest_exp2(torch.from_numpy(x).cuda()).cpu().numpy()
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y <= 2.0 ** -124)
