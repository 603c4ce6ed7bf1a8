"""Pins of the oracle's layer surround (QKV projections, Q/K L2
normalisation, output projection) against facts that do not come from the
oracle: torch's linear layers and vector norms (library routines), the unit
norm and scale invariance that define an L2 normalisation, brute force over
(token, head) rows, and the pages' statement that only Q and K are
normalised: scaling Wq or Wk leaves the layer's output unchanged, scaling Wv
does not.  The mistakes these catch include normalising over all heads at
once instead of per head, normalising V, and a transposed projection."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc

rng = np.random.default_rng(1357)


def test_l2_normalize_heads_unit_rows_brute_force_and_zero_rows():
    n, H, d = 5, 3, 4
    Y = rng.normal(size=(n, H * d))
    Y[2, d:2 * d] = 0.0
    got = orc.l2_normalize_heads(Y, H)
    for i in range(n):
        for hd in range(H):
            row = Y[i, hd * d:(hd + 1) * d]
            nrm = sum(x * x for x in row) ** 0.5
            want = row / nrm if nrm > 0 else row
            np.testing.assert_allclose(got[i, hd], want, rtol=1e-14, atol=0)
    np.testing.assert_array_equal(got[2, 1], np.zeros(d))
    t = torch.nn.functional.normalize(torch.from_numpy(Y.reshape(n, H, d)), dim=2)
    np.testing.assert_allclose(got, t.numpy(), rtol=1e-14, atol=1e-15)
    # scale-free per row, not per token
    scaled = Y.copy()
    scaled[:, :d] *= 7.0
    np.testing.assert_allclose(orc.l2_normalize_heads(scaled, H), got, rtol=1e-14, atol=1e-15)


def _setup(H=2, d=8, h=16, views=2, gh=3, gw=4, ns=1):
    dims = orc.Dims(views, gh, gw, ns)
    n, C = dims.n, H * d
    X = rng.normal(size=(n, C))
    Ws = [rng.normal(size=(C, C)) / np.sqrt(C) for _ in range(4)]
    conv_w = rng.normal(size=(C, 3, 3)) / 3.0
    th = [rng.normal(size=(H, d, h)) * 0.3, rng.normal(size=(H, d, h)) * 0.3, rng.normal(size=(H, h, d)) * 0.3]
    return dims, X, Ws, conv_w, th


@pytest.mark.parametrize("inner,lr", [("sgd", 0.5), ("muon", 0.1)])
def test_attention_matches_torch_projections_and_layer(inner, lr):
    dims, X, (Wq, Wk, Wv, Wo), conv_w, th = _setup()
    H, n = th[0].shape[0], X.shape[0]
    out, *_ = orc.ttt_attention(X, Wq, Wk, Wv, Wo, conv_w, *th, lr, 2, dims, inner)
    Xt = torch.from_numpy(X)
    lin = lambda W: torch.nn.functional.linear(Xt, torch.from_numpy(W).T).numpy()   # noqa: E731
    q = torch.nn.functional.normalize(torch.from_numpy(lin(Wq).reshape(n, H, -1)), dim=2).numpy()
    k = torch.nn.functional.normalize(torch.from_numpy(lin(Wk).reshape(n, H, -1)), dim=2).numpy()
    v = lin(Wv).reshape(n, H, -1)
    if inner == "sgd":
        O = orc.layer(q, k, v, conv_w, *th, lr, 2, dims)[3]
    else:
        d = v.shape[2]
        Vp = orc.shortconv2d(v.reshape(n, H * d), conv_w, dims).reshape(n, H, d)
        O = np.zeros_like(q)
        for hd in range(H):
            t, _ = orc.muon_write(k[:, hd], Vp[:, hd], [w[hd] for w in th], lr, 2)
            O[:, hd] = orc.read(q[:, hd], *t)
    want = torch.nn.functional.linear(torch.from_numpy(O.reshape(n, -1)), torch.from_numpy(Wo).T).numpy()
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-12)


def test_only_q_and_k_are_normalised():
    dims, X, (Wq, Wk, Wv, Wo), conv_w, th = _setup()
    base, *_ = orc.ttt_attention(X, Wq, Wk, Wv, Wo, conv_w, *th, 0.5, 2, dims)
    for scaled in ((3 * Wq, Wk, Wv), (Wq, 0.2 * Wk, Wv)):
        out, *_ = orc.ttt_attention(X, *scaled, Wo, conv_w, *th, 0.5, 2, dims)
        np.testing.assert_allclose(out, base, rtol=1e-10, atol=1e-12)
    out, *_ = orc.ttt_attention(X, Wq, Wk, 3 * Wv, Wo, conv_w, *th, 0.5, 2, dims)
    assert np.max(np.abs(out - base)) > 1e-3 * np.max(np.abs(base))
