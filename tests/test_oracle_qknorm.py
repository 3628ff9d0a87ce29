"""Pins of the q/k RMS-norm oracle (CPU): torch's own fp64 rms_norm, and two closed forms
(a constant row normalises to +-1 times the weight; the mean square of a normalised row with
unit weight and eps = 0 is 1)."""
import numpy as np
import pytest
import torch

from oracle import bifocal_ref as R


@pytest.mark.parametrize("D,eps", [(8, 0.0), (64, 1e-6), (128, 1e-6), (128, 0.5)])
def test_matches_torch_rms_norm(D, eps):
    rng = np.random.default_rng(D)
    x = rng.standard_normal((5, 3, D))
    w = 1.0 + 0.1 * rng.standard_normal(D)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (D,), torch.from_numpy(w), eps).numpy()
    assert np.abs(R.qk_rms_norm(x, w, eps) - ref).max() < 1e-12


def test_closed_forms():
    w = np.linspace(0.5, 1.5, 16)
    assert np.allclose(R.qk_rms_norm(np.full(16, -3.0), w, 0.0), -w, atol=1e-15)
    x = np.random.default_rng(1).standard_normal((7, 16)) * 5.0
    y = R.qk_rms_norm(x, np.ones(16), 0.0)
    assert np.allclose(np.mean(y * y, axis=-1), 1.0, atol=1e-12)
