"""Float64 CPU oracle of the VGG-T^3 test-time-training (TTT) layer.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA path and imports nothing from it.

Plain, slow, obviously-correct numpy in float64.  Pages cited below:

* [summary] "VGG-T$^3$: Offline Feed-Forward 3D Reconstruction at Scale"
  (paper-graph summary of arXiv 2602.23361), Sec. 3.4:
    - "The Test-Time Training (TTT) Framework ...": Eq. 3 (write:
      theta* = argmin_theta sum_i L(T_theta(k_i), v_i)) and Eq. 4 (read:
      o_i = T_theta(q_i)).
    - "Non-Linear Spatial Mixing via ShortConv2D": reshape the value sequence
      to (N, H/p, W/p, d), apply a 3x3 convolution, flatten back to V';
      "Implementation detail (Appendix A)": camera and register tokens pass
      through without spatial mixing.
    - "TTT MLP Architecture and Inner Optimization": SwiGLU fast-weight MLP.
    - "Large-Scale Inference Strategies": Eq. 5, the gradient of the summed
      loss is the sum of per-minibatch gradients.
* [blog] VGG-T^3 blog post (neteralex.cn), section on why a trivial mapping
  is not enough: ShortConv2D is a depthwise 3x3 convolution applied within
  a single image only.

Readings taken where the pages are silent or disagree:

* Loss: mean over all n tokens (special tokens included) of ||T(k) - v'||^2.
* Inner optimiser: plain SGD, theta <- theta - lr * grad, each step a
  full-batch gradient at the current theta, V' computed once.
* SwiGLU: T(x) = (silu(x W1) * (x W3)) W2, no biases, one MLP per head.
* Conv: cross-correlation (the torch conv2d convention), zero padding, no
  bias, depthwise over all heads*d channels, weights shared by all views.
* Special tokens are the first ``n_special`` tokens of each view.

The pages' own inner loop (dot-product loss and Muon) takes these readings:

* Dot-product loss ([summary] Sec. 3.4, "The dot product loss": the per-token
  loss is T(k)^T v, and the arg-min form implies a minus sign):
  L = -(1/n) sum_i <T(k_i), v'_i>, on V' as for the mean-squared loss.  The
  1/n is immaterial under Muon, whose step is scale-invariant.
* Muon ("TTT MLP Architecture and Inner Optimization": 5 Newton-Schulz
  iterations, learning rate 0.1; the pages give no polynomial, momentum or
  shape factor): per weight matrix of a head, X_0 = G / ||G||_F and the cubic
  Newton-Schulz iteration for the orthogonal polar factor,
  X <- 1.5 X - 0.5 X X^T X, five times; then theta <- theta - lr * X_5.  No
  momentum (one or two steps), no shape factor.

The layer's surround (QKV projections, Q/K normalisation, output projection)
takes these readings:

* Projections (Eq. 1 of [summary] Sec. 3, "QKV projection with
  normalization"), in row-vector form: q = x Wq, k = x Wk, v = x Wv with
  [C, C] matrices, C = heads * d, split into heads of d channels; the output
  projection ("the output projection matrices that follow the attention
  operation") is out = o Wo.  No biases (none are given).
* LN_q and LN_k are replaced by L2 normalisation ("The LayerNorm removal":
  k_hat = k / ||k||_2) of each (token, head) row of length d; V is not
  normalised.  A zero row stays zero.

Every function here is pinned by tests in ``tests/test_oracle_*.py`` against
facts that do not come from this file (library routines, finite differences,
closed forms, brute force, invariants).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence, Tuple

import numpy as np

__all__ = [
    "Dims", "shortconv2d", "sigmoid", "swiglu_forward", "mse_loss", "mse_grad", "mse_grad_chunked",
    "sgd_write", "read", "layer", "LinearModel", "SwiGLUModel", "ChunkedSwiGLUModel",
    "dot_loss", "dot_grad", "newton_schulz", "muon_write", "DotSwiGLUModel", "DotLinearModel",
    "l2_normalize_heads", "ttt_attention",
]


@dataclass(frozen=True)
class Dims:
    """Token layout: each view holds ``n_special`` tokens, then a grid_h x grid_w grid."""
    n_views: int
    grid_h: int
    grid_w: int
    n_special: int

    @property
    def tokens_per_view(self) -> int:
        return self.n_special + self.grid_h * self.grid_w

    @property
    def n(self) -> int:
        return self.n_views * self.tokens_per_view


# ---------------------------------------------------------------------------
# ShortConv2D  ([summary] "Non-Linear Spatial Mixing via ShortConv2D" + App. A;
#               [blog] depthwise 3x3 within one image)
# ---------------------------------------------------------------------------

def shortconv2d(V: np.ndarray, conv_w: np.ndarray, dims: Dims) -> np.ndarray:
    """V' from V.

    V: [n, C] (C = heads * d channels, token-major).  conv_w: [C, 3, 3].
    For every view: reshape its patch tokens to (grid_h, grid_w, C), take
    out[y, x, c] = sum_{a,b in 0..2} w[c, a, b] * in[y + a - 1, x + b - 1, c]
    with zeros outside the grid, flatten back.  Special tokens are copied.
    """
    V = np.asarray(V, dtype=np.float64)
    w = np.asarray(conv_w, dtype=np.float64)
    n, C = V.shape
    assert n == dims.n and w.shape == (C, 3, 3)
    gh, gw, T = dims.grid_h, dims.grid_w, dims.tokens_per_view
    out = V.copy()                      # special tokens pass through unchanged
    for v in range(dims.n_views):
        first = v * T + dims.n_special
        grid = V[first:first + gh * gw].reshape(gh, gw, C)
        padded = np.zeros((gh + 2, gw + 2, C))
        padded[1:gh + 1, 1:gw + 1] = grid
        acc = np.zeros((gh, gw, C))
        for a in range(3):
            for b in range(3):
                acc += w[:, a, b] * padded[a:a + gh, b:b + gw]
        out[first:first + gh * gw] = acc.reshape(gh * gw, C)
    return out


# ---------------------------------------------------------------------------
# SwiGLU fast-weight MLP ([summary] "TTT MLP Architecture and Inner Optimization")
# ---------------------------------------------------------------------------

def sigmoid(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def swiglu_forward(X, W1, W3, W2):
    """T(X) = (silu(X W1) * (X W3)) W2 for X [n, d]; returns (Y, Z1, Z3, A)."""
    Z1 = X @ W1
    Z3 = X @ W3
    A = Z1 * sigmoid(Z1) * Z3
    return A @ W2, Z1, Z3, A


class SwiGLUModel:
    """theta = (W1 [d,h], W3 [d,h], W2 [h,d]) of one head."""

    @staticmethod
    def forward(X, theta):
        return swiglu_forward(X, *theta)[0]

    @staticmethod
    def grad(X, Vp, theta):
        return mse_grad(X, Vp, *theta)


class LinearModel:
    """T(x) = x W, used only to pin the write loop against a closed form."""

    @staticmethod
    def forward(X, theta):
        return X @ theta[0]

    @staticmethod
    def grad(X, Vp, theta):
        n = X.shape[0]
        R = X @ theta[0] - Vp
        return (X.T @ ((2.0 / n) * R),)


def mse_loss(Y: np.ndarray, Vp: np.ndarray) -> float:
    """(1/n) * sum_i ||y_i - v'_i||^2 over all n tokens."""
    n = Y.shape[0]
    R = Y - Vp
    return float(np.sum(R * R) / n)


def mse_grad(K, Vp, W1, W3, W2) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradient of mse_loss(T(K), V') with respect to (W1, W3, W2).

    Backward through the SwiGLU by the chain rule:
      G = (2/n)(Y - V'),  dW2 = A^T G,  dA = G W2^T,
      with S = sigmoid(Z1):  d silu(z)/dz = S (1 + Z1 (1 - S)),
      dZ1 = dA * Z3 * S * (1 + Z1 (1 - S)),  dZ3 = dA * Z1 * S,
      dW1 = K^T dZ1,  dW3 = K^T dZ3.
    """
    n = K.shape[0]
    Y, Z1, Z3, A = swiglu_forward(K, W1, W3, W2)
    S = sigmoid(Z1)
    G = (2.0 / n) * (Y - Vp)
    dW2 = A.T @ G
    dA = G @ W2.T
    dZ1 = dA * Z3 * S * (1.0 + Z1 * (1.0 - S))
    dZ3 = dA * Z1 * S
    return K.T @ dZ1, K.T @ dZ3, dW2


def mse_grad_chunked(K, Vp, W1, W3, W2, chunk: int):
    """mse_grad summed over token chunks ([summary] Eq. 5: the gradient of the
    total loss is the sum of the per-minibatch gradients), to bound memory on
    long sequences.  Each chunk's gradient is normalised by its own length, so
    it is weighted by len(chunk)/n."""
    n = K.shape[0]
    acc = [np.zeros_like(W1, dtype=np.float64), np.zeros_like(W3, dtype=np.float64),
           np.zeros_like(W2, dtype=np.float64)]
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        g = mse_grad(K[a:b], Vp[a:b], W1, W3, W2)
        for p in range(3):
            acc[p] += g[p] * ((b - a) / n)
    return tuple(acc)


class ChunkedSwiGLUModel:
    """SwiGLU with the Eq. 5 chunked gradient (same values, bounded memory)."""

    def __init__(self, chunk: int):
        self.chunk = chunk

    def forward(self, X, theta):
        out = np.empty((X.shape[0], theta[2].shape[1]))
        for a in range(0, X.shape[0], self.chunk):
            out[a:a + self.chunk] = swiglu_forward(X[a:a + self.chunk], *theta)[0]
        return out

    def grad(self, X, Vp, theta):
        return mse_grad_chunked(X, Vp, *theta, chunk=self.chunk)


# ---------------------------------------------------------------------------
# Write (Eq. 3 with plain SGD) and read (Eq. 4), per head
# ---------------------------------------------------------------------------

def sgd_write(K, Vp, theta0: Sequence[np.ndarray], lr: float, steps: int,
              model=SwiGLUModel) -> Tuple[List[np.ndarray], List[float]]:
    """theta_{t+1} = theta_t - lr * grad L(theta_t), t = 0..steps-1, full batch.

    Returns (theta_steps, losses) where losses[t] is the loss at theta_t.
    """
    theta = [np.array(w, dtype=np.float64, copy=True) for w in theta0]
    losses = []
    for _ in range(steps):
        losses.append(mse_loss(model.forward(K, theta), Vp))
        g = model.grad(K, Vp, theta)
        theta = [w - lr * gw for w, gw in zip(theta, g)]
    return theta, losses


# ---------------------------------------------------------------------------
# The pages' own inner loop: dot-product loss and Muon ([summary] Sec. 3.4,
# "The dot product loss"; "TTT MLP Architecture and Inner Optimization")
# ---------------------------------------------------------------------------

def dot_loss(Y: np.ndarray, Vp: np.ndarray) -> float:
    """-(1/n) * sum_i <y_i, v'_i> over all n tokens."""
    n = Y.shape[0]
    return float(-np.sum(Y * Vp) / n)


def dot_grad(K, Vp, W1, W3, W2) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradient of dot_loss(T(K), V') with respect to (W1, W3, W2).

    The chain rule of mse_grad with dL/dY = G = -V'/n (the loss is linear in
    Y, so G does not depend on theta):
      dW2 = A^T G,  dA = G W2^T,  dZ1 = dA * Z3 * S * (1 + Z1 (1 - S)),
      dZ3 = dA * Z1 * S,  dW1 = K^T dZ1,  dW3 = K^T dZ3.
    """
    n = K.shape[0]
    _, Z1, Z3, A = swiglu_forward(K, W1, W3, W2)
    S = sigmoid(Z1)
    G = -Vp / n
    dW2 = A.T @ G
    dA = G @ W2.T
    dZ1 = dA * Z3 * S * (1.0 + Z1 * (1.0 - S))
    dZ3 = dA * Z1 * S
    return K.T @ dZ1, K.T @ dZ3, dW2


def newton_schulz(G: np.ndarray, iters: int = 5) -> np.ndarray:
    """Muon's orthogonalised update of one matrix: X_0 = G / ||G||_F, then
    X <- 1.5 X - 0.5 X X^T X, ``iters`` times (zero for G = 0)."""
    G = np.asarray(G, np.float64)
    nrm = np.sqrt(np.sum(G * G))
    if nrm == 0.0:
        return np.zeros_like(G)
    X = G / nrm
    for _ in range(iters):
        X = 1.5 * X - 0.5 * (X @ X.T) @ X
    return X


class DotSwiGLUModel:
    """SwiGLU fast weights under the dot-product loss."""

    @staticmethod
    def forward(X, theta):
        return swiglu_forward(X, *theta)[0]

    @staticmethod
    def loss(Y, Vp):
        return dot_loss(Y, Vp)

    @staticmethod
    def grad(X, Vp, theta):
        return dot_grad(X, Vp, *theta)


class DotLinearModel:
    """T(x) = x W under the dot-product loss, used only to pin the Muon loop
    against a closed form."""

    @staticmethod
    def forward(X, theta):
        return X @ theta[0]

    @staticmethod
    def loss(Y, Vp):
        return dot_loss(Y, Vp)

    @staticmethod
    def grad(X, Vp, theta):
        return (-(X.T @ Vp) / X.shape[0],)


def muon_write(K, Vp, theta0: Sequence[np.ndarray], lr: float, steps: int, model=DotSwiGLUModel,
               ns_iters: int = 5) -> Tuple[List[np.ndarray], List[float]]:
    """theta_{t+1} = theta_t - lr * NS(grad L(theta_t)) per weight matrix,
    t = 0..steps-1, full batch.  Returns (theta_steps, losses[t] at theta_t)."""
    theta = [np.array(w, dtype=np.float64, copy=True) for w in theta0]
    losses = []
    for _ in range(steps):
        losses.append(model.loss(model.forward(K, theta), Vp))
        g = model.grad(K, Vp, theta)
        theta = [w - lr * newton_schulz(gw, ns_iters) for w, gw in zip(theta, g)]
    return theta, losses


def read(Q, W1, W3, W2) -> np.ndarray:
    """o_i = T_theta(q_i) for every row of Q [n, d]."""
    return swiglu_forward(Q, W1, W3, W2)[0]


# ---------------------------------------------------------------------------
# The layer's surround ([summary] Sec. 3 "QKV projection with normalization",
# Eq. 1; Sec. 3.2 / "The LayerNorm removal"; the output projection)
# ---------------------------------------------------------------------------

def l2_normalize_heads(Y: np.ndarray, heads: int) -> np.ndarray:
    """Y [n, heads*d] with every (token, head) row of length d scaled to unit
    L2 norm; rows of norm zero stay zero.  Returns [n, heads, d]."""
    Y = np.asarray(Y, np.float64)
    n = Y.shape[0]
    R = Y.reshape(n, heads, -1)
    nrm = np.sqrt(np.sum(R * R, axis=2, keepdims=True))
    return np.divide(R, nrm, out=np.zeros_like(R), where=nrm > 0)


def ttt_attention(X, Wq, Wk, Wv, Wo, conv_w, W1, W3, W2, lr: float, steps: int, dims: Dims, inner: str = "sgd"):
    """The global attention layer with the TTT layer in place of softmax
    attention: q_hat = L2(X Wq), k_hat = L2(X Wk) per head, v = X Wv; the
    layer on (q_hat, k_hat, v) with ``inner`` = "sgd" (mean-squared loss, SGD)
    or "muon" (dot-product loss, Muon); out = O Wo.

    X: [n, C]; Wq, Wk, Wv, Wo: [C, C]; the rest as for ``layer``.
    Returns (out [n, C], W1*, W3*, W2*)."""
    X = np.asarray(X, np.float64)
    H = np.asarray(W1).shape[0]
    n = X.shape[0]
    Q = l2_normalize_heads(X @ Wq, H)
    K = l2_normalize_heads(X @ Wk, H)
    V = (X @ Wv).reshape(n, H, -1)
    if inner == "sgd":
        W1s, W3s, W2s, O, _ = layer(Q, K, V, conv_w, W1, W3, W2, lr, steps, dims)
    elif inner == "muon":
        d = V.shape[2]
        Vp = shortconv2d(V.reshape(n, H * d), conv_w, dims).reshape(n, H, d)
        W1s, W3s, W2s = [], [], []
        O = np.zeros_like(Q)
        for hd in range(H):
            th, _ = muon_write(K[:, hd], Vp[:, hd], (np.asarray(W1[hd], np.float64), np.asarray(W3[hd], np.float64),
                                                     np.asarray(W2[hd], np.float64)), lr, steps)
            W1s.append(th[0]); W3s.append(th[1]); W2s.append(th[2])
            O[:, hd] = read(Q[:, hd], *th)
        W1s, W3s, W2s = np.stack(W1s), np.stack(W3s), np.stack(W2s)
    else:
        raise ValueError(f"unknown inner loop {inner!r}")
    return O.reshape(n, -1) @ Wo, W1s, W3s, W2s


def layer(Q, K, V, conv_w, W1, W3, W2, lr: float, steps: int, dims: Dims):
    """The whole layer: V' = ShortConv2D(V); per head, fit theta on K -> V'
    with ``steps`` SGD steps; read O = T_theta*(Q).

    Q, K, V: [n, heads, d]; conv_w: [heads*d, 3, 3]; W1, W3: [heads, d, h];
    W2: [heads, h, d].  Returns (W1*, W3*, W2*, O [n, heads, d], losses [heads, steps]).
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    n, H, d = K.shape
    Vp = shortconv2d(V.reshape(n, H * d), conv_w, dims).reshape(n, H, d)
    W1s, W3s, W2s, losses = [], [], [], []
    O = np.zeros_like(Q)
    for hd in range(H):
        th, ls = sgd_write(K[:, hd], Vp[:, hd],
                           (np.asarray(W1[hd], np.float64), np.asarray(W3[hd], np.float64),
                            np.asarray(W2[hd], np.float64)), lr, steps)
        W1s.append(th[0]); W3s.append(th[1]); W2s.append(th[2]); losses.append(ls)
        O[:, hd] = read(Q[:, hd], *th)
    return np.stack(W1s), np.stack(W3s), np.stack(W2s), O, np.array(losses)
