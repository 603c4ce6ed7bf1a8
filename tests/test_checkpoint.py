"""Saving and loading theta*: a bit-exact round trip, the shape recorded and
checked, and bad files or shapes rejected."""
import numpy as np
import pytest
import torch

from test_layer_reconstruction_b200 import checkpoint


def test_round_trip_is_bit_exact(tmp_path):
    theta = torch.randn(3 * 2 * 16 * 32, generator=torch.Generator().manual_seed(1))
    theta[5] = float("-0.0")
    p = tmp_path / "theta.npz"
    checkpoint.save_theta(p, theta, 2, 16, 32)
    back, shape = checkpoint.load_theta(p, heads=2, d=16, h=32)
    assert shape == (2, 16, 32)
    assert torch.equal(back.view(torch.int32), theta.view(torch.int32))


def test_shape_checks(tmp_path):
    p = tmp_path / "theta.npz"
    with pytest.raises(ValueError):
        checkpoint.save_theta(p, torch.zeros(10), 1, 16, 32)
    checkpoint.save_theta(p, torch.zeros(3 * 16 * 32), 1, 16, 32)
    with pytest.raises(ValueError):
        checkpoint.load_theta(p, d=64)
    np.savez(tmp_path / "bad.npz", theta=np.zeros(3, np.float32), heads=1, d=1, h=1, layout="other")
    with pytest.raises(ValueError):
        checkpoint.load_theta(tmp_path / "bad.npz")
