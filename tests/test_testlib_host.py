"""Host checks of the parity helpers (no GPU): the norm-wise error and the
float32 resolution allowance of the update diagnostic.

An update rounded to float32 after each step, with otherwise exact
arithmetic, must read as error-free beyond the resolution; a 3 % error in
the update must read as 3 %; the allowance must be no larger than the
rounding it stands for."""
import numpy as np

from ttt_testlib import delta_error, f32_resolution, normwise


def _steps_f32(theta0, grads, lr):
    th64, th32 = theta0.astype(np.float64), theta0.astype(np.float32)
    for g in grads:
        th64 = th64 - lr * g
        th32 = (th32.astype(np.float64) - lr * g).astype(np.float32)
    return th64, th32.astype(np.float64)


def test_f32_rounding_of_theta_is_within_the_allowance():
    rng = np.random.default_rng(0)
    theta0 = (rng.standard_normal(65536) * 0.08).astype(np.float32)
    grads = [rng.standard_normal(65536) * 1e-5 for _ in range(2)]
    exact, stored = _steps_f32(theta0, grads, 0.05)
    t0 = theta0.astype(np.float64)
    # the raw norm-wise error of delta is well above zero (a few percent) ...
    assert normwise(stored - t0, exact - t0) > 5e-3
    # ... and entirely the float32 rounding: nothing is left beyond the allowance
    assert delta_error(stored, exact, t0, steps=2) == 0.0


def test_a_planted_error_in_the_update_reads_at_its_size():
    rng = np.random.default_rng(1)
    theta0 = (rng.standard_normal(4096) * 0.08).astype(np.float64)
    d = rng.standard_normal(4096) * 1e-2        # far above the float32 resolution
    exact = theta0 + d
    wrong = theta0 + d * 1.03
    assert abs(delta_error(wrong, exact, theta0, steps=2) - 0.03) < 1e-3


def test_allowance_is_half_an_ulp_per_step():
    # |theta| in [0.25, 0.5): ulp = 2^-25
    assert f32_resolution(0.3, 1) == 0.5 * 2.0 ** -25
    assert f32_resolution(0.3, 2) == 2.0 ** -25
    assert f32_resolution(1.0, 1) == 0.5 * 2.0 ** -23
    assert f32_resolution(0.0, 2) == 0.0
    x = np.float32(0.3)
    assert f32_resolution(0.3, 1) == float(np.spacing(x)) / 2
