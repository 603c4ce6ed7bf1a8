"""Pins of the oracle's dot-product loss and Muon step against facts that do
not come from the oracle.

What fixes each expected value: brute force over tokens (the loss), central
finite differences and torch float64 autograd (the gradient), the singular
value decomposition (the Newton-Schulz iteration acts on each singular value
alone: s <- 1.5 s - 0.5 s^3 after dividing by the Frobenius norm), a rank-1
fixed point, the polar factor U V^T as the iteration's limit, and a linear
model whose Muon step has a closed form.  The mistakes these catch include:
a lost minus sign of the loss, a transposed product in the iteration
(X^T X X instead of X X^T X), normalising by the spectral instead of the
Frobenius norm, a wrong iteration count, applying the step with the wrong
sign, and orthogonalising the concatenated parameters instead of each matrix.
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc

rng = np.random.default_rng(2468)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_theta(d, h, scale=0.3, seed=0):
    r = np.random.default_rng(seed)
    return (r.normal(0, scale, (d, h)), r.normal(0, scale, (d, h)), r.normal(0, scale, (h, d)))


def _dot_loss_at(K, Vp, th):
    return orc.dot_loss(orc.swiglu_forward(K, *th)[0], Vp)


# ----------------------------------------------------------------- the loss

def test_dot_loss_brute_force():
    n, d = 7, 3
    Y = rng.normal(size=(n, d)); Vp = rng.normal(size=(n, d))
    want = 0.0
    for i in range(n):
        want -= sum(Y[i, j] * Vp[i, j] for j in range(d))
    assert orc.dot_loss(Y, Vp) == pytest.approx(want / n, rel=1e-14)
    # maximising the dot product is minimising the loss: T(k) = v' gives -mean ||v'||^2
    assert orc.dot_loss(Vp, Vp) == pytest.approx(-np.sum(Vp * Vp) / n, rel=1e-14)


@pytest.mark.parametrize("d,h,n", [(3, 5, 7), (4, 6, 10)])
def test_dot_grad_central_finite_differences(d, h, n):
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th = list(_rand_theta(d, h, scale=0.8, seed=d))
    g = orc.dot_grad(K, Vp, *th)
    eps = 1e-6
    for p in range(3):
        num = np.zeros_like(th[p])
        for idx in np.ndindex(th[p].shape):
            tp = [w.copy() for w in th]; tm = [w.copy() for w in th]
            tp[p][idx] += eps; tm[p][idx] -= eps
            num[idx] = (_dot_loss_at(K, Vp, tp) - _dot_loss_at(K, Vp, tm)) / (2 * eps)
        err = np.max(np.abs(num - g[p])) / np.max(np.abs(num))
        assert err < 1e-6, (p, err)


def test_dot_grad_matches_torch_autograd():
    d, h, n = 16, 32, 128
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th = _rand_theta(d, h, scale=0.2, seed=7)
    tt = [torch.from_numpy(w.copy()).requires_grad_(True) for w in th]
    Kt, Vt = torch.from_numpy(K), torch.from_numpy(Vp)
    Y = (torch.nn.functional.silu(Kt @ tt[0]) * (Kt @ tt[1])) @ tt[2]
    loss = -(Y * Vt).sum(dim=1).mean()
    loss.backward()
    g = orc.dot_grad(K, Vp, *th)
    for p in range(3):
        np.testing.assert_allclose(g[p], tt[p].grad.numpy(), rtol=1e-10, atol=1e-14)


def test_dot_grad_minibatch_decomposition_eq5():
    """Eq. 5: the gradient over all tokens is the token-weighted sum over any partition."""
    d, h, n = 5, 8, 40
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th = _rand_theta(d, h, seed=3)
    full = orc.dot_grad(K, Vp, *th)
    acc = [np.zeros_like(w) for w in th]
    for a, b in ((0, 13), (13, 14), (14, 40)):
        gp = orc.dot_grad(K[a:b], Vp[a:b], *th)
        for p in range(3):
            acc[p] += gp[p] * ((b - a) / n)
    for p in range(3):
        np.testing.assert_allclose(acc[p], full[p], rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------- Newton-Schulz

def _ns_by_svd(G, iters):
    """The iteration acts on each singular value: s <- 1.5 s - 0.5 s^3, starting from s / ||G||_F."""
    U, S, Vt = np.linalg.svd(G, full_matrices=False)
    s = S / np.sqrt(np.sum(S * S))
    for _ in range(iters):
        s = 1.5 * s - 0.5 * s ** 3
    return (U * s) @ Vt


@pytest.mark.parametrize("shape", [(4, 9), (9, 4), (16, 64), (64, 16)])
def test_newton_schulz_matches_singular_value_closed_form(shape):
    G = rng.normal(size=shape)
    for iters in (0, 1, 5):
        np.testing.assert_allclose(orc.newton_schulz(G, iters), _ns_by_svd(G, iters), rtol=0, atol=1e-12)


def test_newton_schulz_rank_one_is_fixed_point_and_zero_stays_zero():
    u = np.array([3.0, 4.0]) / 5.0
    v = np.array([2.0, -1.0, 2.0]) / 3.0
    np.testing.assert_allclose(orc.newton_schulz(7.5 * np.outer(u, v)), np.outer(u, v), rtol=0, atol=1e-15)
    assert not np.any(orc.newton_schulz(np.zeros((3, 5))))


def test_newton_schulz_converges_to_polar_factor():
    """Its limit is U V^T (all singular values to 1); five steps get most of the way."""
    G = rng.normal(size=(8, 24))
    U, _, Vt = np.linalg.svd(G, full_matrices=False)
    polar = U @ Vt
    np.testing.assert_allclose(orc.newton_schulz(G, 60), polar, rtol=0, atol=1e-10)
    errs = [np.max(np.abs(orc.newton_schulz(G, k) - polar)) for k in range(6)]
    assert all(b < a for a, b in zip(errs, errs[1:]))


def test_newton_schulz_is_odd_and_scale_free():
    G = rng.normal(size=(6, 10))
    np.testing.assert_array_equal(orc.newton_schulz(-G), -orc.newton_schulz(G))
    np.testing.assert_allclose(orc.newton_schulz(1e3 * G), orc.newton_schulz(G), rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------- the Muon write

def test_muon_linear_model_closed_form():
    """T(x) = x W: grad = -K^T V'/n, so one step is W1 = W0 + lr * NS(K^T V') (NS is odd and scale-free)."""
    n, d, lr = 50, 6, 0.1
    K = rng.normal(size=(n, d)); Vp = rng.normal(size=(n, d)); W0 = rng.normal(size=(d, d))
    (W1,), losses = orc.muon_write(K, Vp, (W0,), lr, 1, model=orc.DotLinearModel)
    np.testing.assert_allclose(W1, W0 + lr * _ns_by_svd(K.T @ Vp, 5), rtol=0, atol=1e-12)
    assert losses[0] == pytest.approx(-np.sum((K @ W0) * Vp) / n, rel=1e-13)


def test_muon_swiglu_step_is_ns_of_fd_gradient_per_matrix():
    """Two steps: each matrix moves by -lr * NS(its own finite-difference gradient)."""
    d, h, n, lr = 3, 4, 9, 0.1
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th0 = _rand_theta(d, h, scale=0.7, seed=3)
    th = [w.copy() for w in th0]
    eps = 1e-6
    for _ in range(2):
        nxt = []
        for p in range(3):
            num = np.zeros_like(th[p])
            for idx in np.ndindex(th[p].shape):
                tp = [w.copy() for w in th]; tm = [w.copy() for w in th]
                tp[p][idx] += eps; tm[p][idx] -= eps
                num[idx] = (_dot_loss_at(K, Vp, tp) - _dot_loss_at(K, Vp, tm)) / (2 * eps)
            nxt.append(th[p] - lr * _ns_by_svd(num, 5))
        th = nxt
    got, _ = orc.muon_write(K, Vp, th0, lr, 2)
    for p in range(3):
        np.testing.assert_allclose(got[p], th[p], rtol=0, atol=1e-7)


def test_muon_small_step_descends_and_lr_zero_keeps_theta():
    """<g, NS(g)> = sum_i s_i f(s_i) > 0, so a small Muon step lowers the loss."""
    d, h, n = 8, 16, 64
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th0 = _rand_theta(d, h, scale=0.3, seed=11)
    th1, losses = orc.muon_write(K, Vp, th0, 1e-3, 1)
    assert _dot_loss_at(K, Vp, th1) < losses[0]
    same, _ = orc.muon_write(K, Vp, th0, 0.0, 2)
    for a, b in zip(same, th0):
        np.testing.assert_array_equal(a, b)
