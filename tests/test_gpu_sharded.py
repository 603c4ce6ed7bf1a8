"""GPU parity of the entry points of the view-sharded write: ttt_grad and
ttt_sgd_update, through the C ABI.

* ttt_grad at theta0 against the oracle's gradient (n/2 times the mean-loss
  gradient of Eq. 3), every head of 6 views of 37x37+5.
* One shard: the sharded write (sharded.write_sharded with a one-rank gather)
  equals ttt_write bit for bit: same kernels, same reduction order, the same
  single-precision step size.
* Two shards emulated on one GPU (10 + 14 of 24 views, in lockstep, their
  gradient sums stacked in rank order as an all-gather would): one step at a
  large step size matches ttt_write on all views up to summation order; at
  the workload's step size theta* is within two units in the last place
  (plus the step's summation-order difference) of ttt_write's and within the
  parity tolerances of the oracle's full-batch write; each shard's read
  equals ttt_read of its queries with theta*.
* ttt_sgd_update sums its gradients in index order (bit for bit against the
  single-precision sum in that order), rounds the step once, and accepts
  theta_out aliasing theta_in.
* The wide-head path's ttt_grad: one update with it equals ttt_write's one step.
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc
from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import sharded, ttt
from ttt_testlib import TOL_DELTA, TOL_O, TOL_THETA, compare_O, compare_theta, dims_of, normwise, oracle_layer

pytestmark = pytest.mark.gpu

BASE = tin.CONFIGS["views24_37x37p5_h16_d64_h256"]


def _device_inputs(cfg, views=None):
    inp = tin.make_inputs(cfg, views=views)
    dev = {k: inp[k].to(torch.bfloat16).contiguous().cuda() for k in ("Q", "K", "V")}
    dev["conv_w"] = inp["conv_w"].float().contiguous().cuda()
    dev["theta"] = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).cuda()
    return inp, dev


def test_grad_matches_oracle():
    cfg = BASE.with_views(6)
    inp, dev = _device_inputs(cfg)
    Vp = ttt.shortconv2d(dev["V"], dev["conv_w"], cfg)
    g = ttt.grad(dev["K"], Vp, dev["theta"], cfg)
    torch.cuda.synchronize()
    G1, G3, G2 = (t.double().cpu().numpy() for t in tin.unpack_theta(g.cpu(), cfg.heads, cfg.d, cfg.h))
    dims = dims_of(cfg)
    n, H, d = inp["K"].shape
    for hd in range(H):
        ch = slice(hd * d, (hd + 1) * d)
        vp = orc.shortconv2d(inp["V"][:, hd].double().numpy(), inp["conv_w"][ch].double().numpy(), dims)
        ref = orc.mse_grad(inp["K"][:, hd].double().numpy(), vp, inp["W1"][hd].double().numpy(),
                           inp["W3"][hd].double().numpy(), inp["W2"][hd].double().numpy())
        for got, r in zip((G1[hd], G3[hd], G2[hd]), ref):
            assert normwise(got, r * (n / 2.0)) <= TOL_DELTA


def test_one_shard_equals_write_bitwise():
    cfg = BASE
    _, dev = _device_inputs(cfg)
    full = ttt.write(dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, 2, cfg)
    sh = sharded.write_sharded(dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, 2, cfg, cfg.n,
                               gather=lambda t: t.reshape(1, -1))
    torch.cuda.synchronize()
    assert torch.equal(full, sh)


def _two_shard_write(cfg, dev, lr, steps, parts=((0, 10), (10, 24))):
    """The sharded write of two ranks emulated in lockstep on one GPU."""
    tpv = cfg.tokens_per_view
    shards = []
    for a, b in parts:
        loc = cfg.with_views(b - a)
        rows = slice(a * tpv, b * tpv)
        K, V, Q = (dev[k][rows].contiguous() for k in ("K", "V", "Q"))
        shards.append((loc, K, ttt.shortconv2d(V, dev["conv_w"], loc), Q))
    scale = sharded.step_scale(lr, cfg.n)
    theta = dev["theta"]
    for _ in range(steps):
        grads = torch.stack([ttt.grad(K, Vp, theta, loc) for loc, K, Vp, _ in shards])
        theta = ttt.sgd_update(theta, grads, scale, cfg)
    return theta, shards


def test_two_shards_on_one_gpu_match_full_batch():
    cfg = BASE
    inp, dev = _device_inputs(cfg)
    th0 = dev["theta"].double().cpu().numpy()
    # One step far above theta's single-precision resolution: the sum of the
    # shards' gradient sums equals the full one up to summation order.
    big, _ = _two_shard_write(cfg, dev, 50.0, 1)
    full_big = ttt.write(dev["K"], dev["V"], dev["conv_w"], dev["theta"], 50.0, 1, cfg)
    torch.cuda.synchronize()
    assert normwise(big.double().cpu().numpy() - th0, full_big.double().cpu().numpy() - th0) <= 5e-4
    # The workload's own step size: the update is ~1e-4 of theta, so the two
    # orders may round theta* apart by a unit in the last place, plus the
    # summation-order difference of the step itself.
    theta, shards = _two_shard_write(cfg, dev, cfg.lr, 2)
    full = ttt.write(dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, 2, cfg)
    torch.cuda.synchronize()
    diff = (theta - full).abs()
    step = (full - dev["theta"]).abs().max()
    assert bool((diff <= full.abs() * 2.0 ** -22 + 1e-4 * step).all())
    ref = oracle_layer(cfg, inp, steps=2, lr=cfg.lr)
    t_err, d_err = compare_theta(cfg, inp, theta, ref)
    assert t_err <= TOL_THETA and d_err <= TOL_DELTA, (t_err, d_err)
    O = torch.cat([ttt.read(Q, theta, loc) for loc, _, _, Q in shards])
    assert torch.equal(O, ttt.read(dev["Q"], theta, cfg))
    assert compare_O(O, ref) <= TOL_O


def test_sgd_update_sums_in_order_and_in_place():
    cfg = BASE
    count = 3 * cfg.heads * cfg.d * cfg.h
    g = torch.Generator().manual_seed(5)
    theta = torch.randn(count, generator=g)
    # magnitudes far apart, so another summation order rounds differently
    grads = torch.randn(3, count, generator=g) * torch.tensor([1.0, 1e3, 1e-3]).reshape(3, 1)
    # theta = 0, scale = -1: the result is the single-precision sum itself, bit for bit
    s = (grads[0] + grads[1]) + grads[2]
    assert not torch.equal(s, grads[0] + (grads[1] + grads[2]))
    sums = ttt.sgd_update(torch.zeros(count, device="cuda"), grads.cuda(), -1.0, cfg)
    out = ttt.sgd_update(theta.cuda(), grads.cuda(), 0.25, cfg)
    th_dev = theta.cuda()
    ttt.sgd_update(th_dev, grads.cuda(), 0.25, cfg, theta_out=th_dev)
    torch.cuda.synchronize()
    assert torch.equal(sums.cpu(), s)
    assert torch.equal(out, th_dev)
    exp = theta.double() - 0.25 * s.double()
    assert bool(((out.cpu().double() - exp).abs() <= exp.abs() * 2 ** -23 + 1e-30).all())


def test_wide_grad_step_equals_write_step():
    cfg = tin.LayerConfig("wide_small", 3, 9, 11, 2, 2, 128, 192, 1, 0.1, 21)
    _, dev = _device_inputs(cfg)
    Vp = ttt.shortconv2d(dev["V"], dev["conv_w"], cfg)
    g = ttt.grad(dev["K"], Vp, dev["theta"], cfg)
    one = ttt.sgd_update(dev["theta"], g.reshape(1, -1), sharded.step_scale(cfg.lr, cfg.n), cfg)
    full = ttt.write(dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, 1, cfg)
    torch.cuda.synchronize()
    th0 = dev["theta"].double().cpu().numpy()
    assert normwise(one.double().cpu().numpy() - th0, full.double().cpu().numpy() - th0) <= 1e-6
