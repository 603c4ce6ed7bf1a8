"""Pins of the float64 oracle against facts that do not come from the oracle.

Each test names what fixes the expected value: a library routine (torch
conv2d, torch autograd), central finite differences, a closed form, brute
force on tiny inputs, or an invariant stated by the pages.  The mistakes
these catch include: a dropped term of d silu/dz, a sign error in the
update, a transposed operand, a wrong loss normalisation, conv orientation
or cross-view leakage, and special tokens being convolved.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def _rand_theta(d, h, scale=0.3, seed=0):
    r = np.random.default_rng(seed)
    return (r.normal(0, scale, (d, h)), r.normal(0, scale, (d, h)), r.normal(0, scale, (h, d)))


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ----------------------------------------------------------------- ShortConv2D

def test_conv_matches_torch_depthwise_conv2d():
    """Library special case: depthwise torch conv2d (cross-correlation, zero pad 1)."""
    dims = orc.Dims(n_views=3, grid_h=5, grid_w=7, n_special=2)
    C = 6
    V = rng.normal(size=(dims.n, C))
    w = rng.normal(size=(C, 3, 3))
    got = orc.shortconv2d(V, w, dims)
    T = dims.tokens_per_view
    for v in range(dims.n_views):
        grid = V[v * T + 2: (v + 1) * T].reshape(5, 7, C)
        x = torch.from_numpy(grid).permute(2, 0, 1)[None]            # [1, C, gh, gw]
        ref = torch.nn.functional.conv2d(x, torch.from_numpy(w)[:, None], padding=1, groups=C)
        ref = ref[0].permute(1, 2, 0).reshape(-1, C).numpy()
        np.testing.assert_allclose(got[v * T + 2:(v + 1) * T], ref, rtol=0, atol=1e-12)


def test_conv_special_tokens_pass_through():
    """[summary] App. A: camera/register tokens are not spatially mixed."""
    dims = orc.Dims(n_views=2, grid_h=3, grid_w=4, n_special=5)
    V = rng.normal(size=(dims.n, 3))
    out = orc.shortconv2d(V, rng.normal(size=(3, 3, 3)), dims)
    T = dims.tokens_per_view
    for v in range(2):
        np.testing.assert_array_equal(out[v * T:v * T + 5], V[v * T:v * T + 5])


def test_conv_identity_kernel_and_box_sum_brute_force():
    dims = orc.Dims(n_views=2, grid_h=4, grid_w=3, n_special=1)
    C = 2
    V = rng.normal(size=(dims.n, C))
    ident = np.zeros((C, 3, 3)); ident[:, 1, 1] = 1.0
    np.testing.assert_array_equal(orc.shortconv2d(V, ident, dims), V)
    ones = np.ones((C, 3, 3))
    out = orc.shortconv2d(V, ones, dims)
    T = dims.tokens_per_view
    for v in range(2):
        for y in range(4):
            for x in range(3):
                for c in range(C):
                    s = 0.0
                    for yy in range(y - 1, y + 2):
                        for xx in range(x - 1, x + 2):
                            if 0 <= yy < 4 and 0 <= xx < 3:
                                s += V[v * T + 1 + yy * 3 + xx, c]
                    assert abs(out[v * T + 1 + y * 3 + x, c] - s) < 1e-12


def test_conv_orientation_is_cross_correlation():
    """A single off-centre tap: out[y, x] = in[y - 1, x] for tap (row 0, col 1)."""
    dims = orc.Dims(n_views=1, grid_h=4, grid_w=4, n_special=0)
    V = rng.normal(size=(16, 1))
    w = np.zeros((1, 3, 3)); w[0, 0, 1] = 1.0
    out = orc.shortconv2d(V, w, dims).reshape(4, 4)
    g = V.reshape(4, 4)
    np.testing.assert_array_equal(out[1:], g[:-1])
    np.testing.assert_array_equal(out[0], 0.0)


def test_conv_never_crosses_views():
    """[blog]: the conv runs inside each image only."""
    dims = orc.Dims(n_views=3, grid_h=3, grid_w=3, n_special=0)
    V = rng.normal(size=(dims.n, 4)); w = rng.normal(size=(4, 3, 3))
    base = orc.shortconv2d(V, w, dims)
    V2 = V.copy(); V2[9:18] += 100.0                      # perturb view 1 only
    out = orc.shortconv2d(V2, w, dims)
    np.testing.assert_array_equal(out[:9], base[:9])
    np.testing.assert_array_equal(out[18:], base[18:])


# ----------------------------------------------------------------- SwiGLU, loss

def test_swiglu_forward_brute_force():
    d, h, n = 3, 4, 5
    W1, W3, W2 = _rand_theta(d, h, seed=1)
    X = rng.normal(size=(n, d))
    Y = orc.swiglu_forward(X, W1, W3, W2)[0]
    for i in range(n):
        for o in range(d):
            acc = 0.0
            for j in range(h):
                z1 = sum(X[i, k] * W1[k, j] for k in range(d))
                z3 = sum(X[i, k] * W3[k, j] for k in range(d))
                acc += (z1 / (1.0 + math.exp(-z1))) * z3 * W2[j, o]
            assert abs(Y[i, o] - acc) < 1e-12


def test_swiglu_matches_torch_silu():
    d, h, n = 8, 12, 20
    W1, W3, W2 = _rand_theta(d, h, scale=1.5, seed=2)
    X = rng.normal(size=(n, d))
    t = lambda a: torch.from_numpy(a)
    ref = (torch.nn.functional.silu(t(X) @ t(W1)) * (t(X) @ t(W3))) @ t(W2)
    np.testing.assert_allclose(orc.swiglu_forward(X, W1, W3, W2)[0], ref.numpy(), rtol=1e-13, atol=1e-13)


def test_mse_loss_brute_force():
    Y = rng.normal(size=(6, 3)); Vp = rng.normal(size=(6, 3))
    s = 0.0
    for i in range(6):
        s += sum((Y[i, c] - Vp[i, c]) ** 2 for c in range(3))
    assert abs(orc.mse_loss(Y, Vp) - s / 6) < 1e-13


# ----------------------------------------------------------------- gradient

def _loss_at(K, Vp, th):
    return orc.mse_loss(orc.swiglu_forward(K, *th)[0], Vp)


@pytest.mark.parametrize("d,h,n", [(3, 5, 7), (4, 6, 10)])
def test_grad_central_finite_differences(d, h, n):
    K = _unit_rows(rng.normal(size=(n, d)))
    Vp = rng.normal(size=(n, d))
    th = list(_rand_theta(d, h, scale=0.8, seed=d))
    g = orc.mse_grad(K, Vp, *th)
    eps = 1e-6
    for p in range(3):
        num = np.zeros_like(th[p])
        for idx in np.ndindex(th[p].shape):
            tp = [w.copy() for w in th]; tm = [w.copy() for w in th]
            tp[p][idx] += eps; tm[p][idx] -= eps
            num[idx] = (_loss_at(K, Vp, tp) - _loss_at(K, Vp, tm)) / (2 * eps)
        err = np.max(np.abs(num - g[p])) / np.max(np.abs(num))
        assert err < 1e-6, (p, err)


def test_grad_matches_torch_autograd():
    d, h, n = 16, 32, 128
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th = _rand_theta(d, h, scale=0.2, seed=7)
    tt = [torch.from_numpy(w.copy()).requires_grad_(True) for w in th]
    Kt, Vt = torch.from_numpy(K), torch.from_numpy(Vp)
    Y = (torch.nn.functional.silu(Kt @ tt[0]) * (Kt @ tt[1])) @ tt[2]
    loss = ((Y - Vt) ** 2).sum(dim=1).mean()
    loss.backward()
    g = orc.mse_grad(K, Vp, *th)
    for p in range(3):
        np.testing.assert_allclose(g[p], tt[p].grad.numpy(), rtol=1e-10, atol=1e-14)


def test_update_is_minus_lr_times_fd_gradient_each_step():
    """Two SGD steps: theta_{t+1} = theta_t - lr * (finite-difference gradient at theta_t)."""
    d, h, n, lr = 3, 4, 9, 0.37
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th0 = _rand_theta(d, h, scale=0.7, seed=3)
    th = [w.copy() for w in th0]
    eps = 1e-6
    for step in range(2):
        nxt = []
        for p in range(3):
            num = np.zeros_like(th[p])
            for idx in np.ndindex(th[p].shape):
                tp = [w.copy() for w in th]; tm = [w.copy() for w in th]
                tp[p][idx] += eps; tm[p][idx] -= eps
                num[idx] = (_loss_at(K, Vp, tp) - _loss_at(K, Vp, tm)) / (2 * eps)
            nxt.append(th[p] - lr * num)
        th = nxt
    got, _ = orc.sgd_write(K, Vp, th0, lr, 2)
    for p in range(3):
        np.testing.assert_allclose(got[p], th[p], rtol=0, atol=1e-8)


def test_linear_model_closed_form_single_step():
    """T(x) = x W: W1 = W0 - lr * (2/n) K^T (K W0 - V') (least-squares gradient by hand)."""
    n, d, lr = 50, 6, 0.2
    K = rng.normal(size=(n, d)); Vp = rng.normal(size=(n, d)); W0 = rng.normal(size=(d, d))
    got, losses = orc.sgd_write(K, Vp, (W0,), lr, 1, model=orc.LinearModel)
    expect = W0 - lr * (2.0 / n) * K.T @ (K @ W0 - Vp)
    np.testing.assert_allclose(got[0], expect, rtol=1e-13, atol=1e-13)
    assert abs(losses[0] - np.mean(np.sum((K @ W0 - Vp) ** 2, axis=1))) < 1e-12


# ----------------------------------------------------------------- invariants

def _layer_inputs(dims, H=2, d=4, h=6, seed=0):
    r = np.random.default_rng(seed)
    n = dims.n
    Q = _unit_rows(r.normal(size=(n, H, d))); K = _unit_rows(r.normal(size=(n, H, d)))
    V = r.normal(size=(n, H, d)); w = r.normal(0, 1 / 3, size=(H * d, 3, 3))
    W1 = r.normal(0, 0.4, size=(H, d, h)); W3 = r.normal(0, 0.4, size=(H, d, h))
    W2 = r.normal(0, 0.4, size=(H, h, d))
    return Q, K, V, w, W1, W3, W2


def test_lr_zero_and_steps_zero_keep_theta_and_read_theta0():
    dims = orc.Dims(2, 3, 3, 1)
    Q, K, V, w, W1, W3, W2 = _layer_inputs(dims)
    for lr, steps in [(0.0, 2), (0.5, 0)]:
        a1, a3, a2, O, _ = orc.layer(Q, K, V, w, W1, W3, W2, lr, steps, dims)
        np.testing.assert_array_equal(a1, W1); np.testing.assert_array_equal(a3, W3)
        np.testing.assert_array_equal(a2, W2)
        for hd in range(2):
            np.testing.assert_array_equal(O[:, hd], orc.swiglu_forward(Q[:, hd], W1[hd], W3[hd], W2[hd])[0])


def test_theta_invariant_to_view_permutation_and_O_permutes():
    dims = orc.Dims(4, 3, 4, 2)
    Q, K, V, w, W1, W3, W2 = _layer_inputs(dims, seed=5)
    T = dims.tokens_per_view
    perm = [2, 0, 3, 1]
    idx = np.concatenate([np.arange(p * T, (p + 1) * T) for p in perm])
    r1 = orc.layer(Q, K, V, w, W1, W3, W2, 0.3, 2, dims)
    r2 = orc.layer(Q[idx], K[idx], V[idx], w, W1, W3, W2, 0.3, 2, dims)
    for p in range(3):
        np.testing.assert_allclose(r2[p], r1[p], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r2[3], r1[3][idx], rtol=1e-12, atol=1e-15)


def test_minibatch_gradient_decomposition_eq5():
    """[summary] Eq. 5: sum_i dL_i/dtheta over all tokens = sum over chunks of chunk sums."""
    n, d, h = 37, 4, 6
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th = _rand_theta(d, h, seed=9)
    full = orc.mse_grad(K, Vp, *th)                  # = (1/n) sum_i grad of ||.||^2
    cuts = [0, 5, 6, 20, 37]
    acc = [np.zeros_like(w) for w in th]
    for a, b in zip(cuts[:-1], cuts[1:]):
        g = orc.mse_grad(K[a:b], Vp[a:b], *th)      # = (1/(b-a)) * chunk sum
        for p in range(3):
            acc[p] += g[p] * (b - a) / n
    for p in range(3):
        np.testing.assert_allclose(acc[p], full[p], rtol=1e-12, atol=1e-15)


def test_chunked_gradient_equals_full_gradient():
    """mse_grad_chunked (used on long sequences) restates Eq. 5: same values as mse_grad."""
    n, d, h = 101, 4, 6
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th = _rand_theta(d, h, seed=17)
    full = orc.mse_grad(K, Vp, *th)
    for chunk in (1, 7, 50, 101, 500):
        got = orc.mse_grad_chunked(K, Vp, *th, chunk=chunk)
        for p in range(3):
            np.testing.assert_allclose(got[p], full[p], rtol=1e-12, atol=1e-15)
    m = orc.ChunkedSwiGLUModel(13)
    a, _ = orc.sgd_write(K, Vp, th, 0.3, 2, model=m)
    b, _ = orc.sgd_write(K, Vp, th, 0.3, 2)
    for p in range(3):
        np.testing.assert_allclose(a[p], b[p], rtol=1e-12, atol=1e-15)


def test_fixed_point_zero_gradient():
    """If V' = T_theta0(K) the loss is 0, its gradient is 0 and theta stays put."""
    n, d, h = 30, 4, 8
    K = _unit_rows(rng.normal(size=(n, d)))
    th = _rand_theta(d, h, seed=11)
    Vp = orc.swiglu_forward(K, *th)[0]
    got, losses = orc.sgd_write(K, Vp, th, 0.5, 2)
    assert losses == [0.0, 0.0]
    for p in range(3):
        np.testing.assert_array_equal(got[p], th[p])


def test_small_step_descends():
    n, d, h = 64, 8, 16
    K = _unit_rows(rng.normal(size=(n, d))); Vp = rng.normal(size=(n, d))
    th = _rand_theta(d, h, seed=13)
    got, losses = orc.sgd_write(K, Vp, th, 0.05, 3)
    assert losses[0] > losses[1] > losses[2]


def test_heads_are_independent():
    dims = orc.Dims(2, 3, 3, 0)
    Q, K, V, w, W1, W3, W2 = _layer_inputs(dims, seed=21)
    base = orc.layer(Q, K, V, w, W1, W3, W2, 0.2, 2, dims)
    K2 = K.copy(); K2[:, 1] = _unit_rows(rng.normal(size=K2[:, 1].shape))
    V2 = V.copy(); V2[:, 1] += 1.0
    out = orc.layer(Q, K2, V2, w, W1, W3, W2, 0.2, 2, dims)
    for p in range(3):
        np.testing.assert_array_equal(out[p][0], base[p][0])
    np.testing.assert_array_equal(out[3][:, 0], base[3][:, 0])


# ----------------------------------------------------------------- layout (pages' numbers)

def test_token_layout_matches_pages_numbers():
    g = json.load(open(os.path.join(GOLDEN, "token_layout.json")))
    side = g["image_side_px"] // g["patch_px"]
    dims = orc.Dims(n_views=1, grid_h=side, grid_w=side, n_special=0)
    assert dims.n == g["patch_tokens_per_image"]
    assert orc.Dims(g["views_training_length"], side, side, 0).n == g["patch_tokens_at_training_length"]
    assert round(orc.Dims(g["views_1k"], side, side, 0).n / 1e6, 2) == g["approx_tokens_1k_millions"]
    assert round(orc.Dims(g["views_2k"], side, side, 0).n / 1e6, 2) == g["approx_tokens_2k_millions"]
