"""Shared helpers of the parity tests: run the oracle and compare.

Tolerance reading (norm-wise "max relative error"): err(a, ref) =
max|a - ref| / max|ref|, per tensor and per head.  The GPU path must meet
O <= 2e-2 and theta* <= 1e-2; the stricter diagnostic on the update itself,
delta = theta* - theta0, must meet <= 2e-2.

theta* is returned in float32, and each step rounds theta to it: the stored
theta* differs from the exact theta_t - lr * g by up to half an ulp of
|theta| per step, whatever the arithmetic before it.  At the workloads' step
sizes one step moves theta by ~1e-6 while half an ulp of |theta| ~ 0.3 is
1.5e-8, so that resolution alone is a few percent of delta on the largest
workloads.  The delta diagnostic is therefore measured beyond it:
    (max|delta_gpu - delta_ref| - steps * ulp32(max|theta|) / 2) / max|delta_ref|.
The gradient itself (``ttt_grad``, float32 with no theta added) carries no
such term and is compared plainly.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from oracle import ttt_oracle as orc
from test_layer_reconstruction_b200 import inputs as tin

TOL_O = 2e-2
TOL_THETA = 1e-2
TOL_DELTA = 2e-2


def normwise(a, ref) -> float:
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.max(np.abs(ref))
    num = np.max(np.abs(a - ref))
    return float(num / den) if den > 0 else float(num)


def dims_of(cfg: tin.LayerConfig) -> orc.Dims:
    return orc.Dims(cfg.n_views, cfg.grid_h, cfg.grid_w, cfg.n_special)


def bf16_inputs(inp):
    """The GPU path takes bf16 token tensors; the oracle parity run gets the same rounded values."""
    out = dict(inp)
    for k in ("Q", "K", "V"):
        out[k] = tin.bf16_round(inp[k])
    return out


def to_device(inp, device="cuda"):
    d = {k: inp[k].to(device=device, dtype=torch.bfloat16).contiguous() for k in ("Q", "K", "V") if k in inp}
    if "conv_w" in inp:
        d["conv_w"] = inp["conv_w"].to(device=device, dtype=torch.float32).contiguous()
    if "W1" in inp:
        d["theta"] = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).to(device)
    return d


def oracle_layer(cfg: tin.LayerConfig, inp, heads=None, steps=None, lr=None):
    """Oracle (float64) over the selected heads; returns dict of per-head arrays."""
    heads = list(range(cfg.heads)) if heads is None else list(heads)
    steps = cfg.steps if steps is None else steps
    lr = cfg.lr if lr is None else lr
    n, H, d = inp["K"].shape
    res = {"W1": {}, "W3": {}, "W2": {}, "O": {}, "losses": {}}
    dims = dims_of(cfg)
    for hd in heads:
        ch = slice(hd * d, (hd + 1) * d)
        V = inp["V"][:, hd].double().numpy()
        Vp = orc.shortconv2d(V, inp["conv_w"][ch].double().numpy(), dims)
        th0 = (inp["W1"][hd].double().numpy(), inp["W3"][hd].double().numpy(), inp["W2"][hd].double().numpy())
        th, ls = orc.sgd_write(inp["K"][:, hd].double().numpy(), Vp, th0, lr, steps)
        res["W1"][hd], res["W3"][hd], res["W2"][hd] = th
        res["O"][hd] = orc.read(inp["Q"][:, hd].double().numpy(), *th)
        res["losses"][hd] = ls
    return res


def f32_resolution(theta_max: float, steps: int) -> float:
    """Largest error that rounding theta to float32 after each of `steps`
    steps can leave on theta*: half an ulp of the largest |theta| per step."""
    if theta_max <= 0 or steps <= 0:
        return 0.0
    ulp = 2.0 ** (np.floor(np.log2(theta_max)) - 23)
    return steps * 0.5 * float(ulp)


def delta_error(g, r, t0, steps) -> float:
    """Norm-wise error of delta = theta* - theta0 beyond the float32 resolution of theta*."""
    g, r, t0 = (np.asarray(x, np.float64) for x in (g, r, t0))
    dr = r - t0
    den = np.max(np.abs(dr))
    q = f32_resolution(max(np.max(np.abs(r)), np.max(np.abs(t0))), steps)
    num = max(0.0, float(np.max(np.abs((g - t0) - dr))) - q)
    return num / den if den > 0 else num


def compare_theta(cfg, inp, theta_gpu: torch.Tensor, ref, heads=None, steps=None):
    """Return worst (theta err, delta err) over heads and the three matrices;
    the delta error is measured beyond the float32 resolution of theta*."""
    steps = cfg.steps if steps is None else steps
    W1g, W3g, W2g = tin.unpack_theta(theta_gpu.detach().cpu(), cfg.heads, cfg.d, cfg.h)
    gpu = {"W1": W1g, "W3": W3g, "W2": W2g}
    heads = list(ref["W1"].keys()) if heads is None else heads
    worst_t, worst_d = 0.0, 0.0
    for hd in heads:
        for name in ("W1", "W3", "W2"):
            g = gpu[name][hd].double().numpy()
            r = ref[name][hd]
            t0 = inp[name][hd].double().numpy()
            worst_t = max(worst_t, normwise(g, r))
            worst_d = max(worst_d, delta_error(g, r, t0, steps))
    return worst_t, worst_d


def compare_O(O_gpu: torch.Tensor, ref, heads=None, rows=None):
    heads = list(ref["O"].keys()) if heads is None else heads
    Og = O_gpu.detach().float().cpu()
    worst = 0.0
    for hd in heads:
        r = ref["O"][hd]
        g = Og[:, hd].double().numpy()
        if rows is not None:
            r, g = r[rows], g[rows]
        worst = max(worst, normwise(g, r))
    return worst


# ---------------------------------------------------------------- guard bands
GUARD = 4096          # bytes of canary on each side (keeps the payload 256-byte aligned)
CANARY = 0xA5


def guarded(shape, dtype, device, fill=None):
    """A tensor of `shape` inside a byte buffer with GUARD canary bytes on both
    sides.  Returns (payload view, whole buffer).  `fill` poisons the payload
    (e.g. NaN for outputs)."""
    nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device=device)
    view = buf[GUARD:GUARD + nbytes].view(dtype).reshape(shape)
    if fill is not None:
        view.fill_(fill)
    return view, buf


def guards_intact(buf) -> bool:
    """True when both canary bands of a `guarded` buffer are untouched."""
    b = buf.cpu()
    return bool((b[:GUARD] == CANARY).all()) and bool((b[-GUARD:] == CANARY).all())


def report(test: str, **values) -> None:
    """Append the measured errors of a parity test as one JSON line to the file
    named by TTT_PARITY_REPORT (nothing when it is unset)."""
    path = os.environ.get("TTT_PARITY_REPORT")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, **{k: (float(v) if isinstance(v, (float, np.floating)) else v)
                                              for k, v in values.items()}}) + "\n")


def oracle_grad_sum(K, Vp, th0, chunk=None):
    """d/dtheta of (1/2) sum_i ||T(k_i) - v'_i||^2 by the oracle (one head), the
    quantity ttt_grad returns: n/2 times the gradient of the mean-squared loss."""
    n = K.shape[0]
    if chunk is None or chunk >= n:
        g = orc.mse_grad(K, Vp, *th0)
    else:
        g = orc.mse_grad_chunked(K, Vp, *th0, chunk=chunk)
    return tuple(x * (n / 2.0) for x in g)
