"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Sizes span several 128-token tiles with ragged tails, both hidden slices,
every supported head width, special tokens and none, 1 and 2 steps.  The
workloads' own sizes are covered in test_gpu_workloads.py.
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc
from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import ttt
from ttt_testlib import (TOL_DELTA, TOL_O, TOL_THETA, bf16_inputs, compare_O, compare_theta, dims_of,
                         normwise, oracle_layer, to_device)

pytestmark = pytest.mark.gpu


def _cfg(n_views, gh, gw, ns, H, d, h, steps=1, lr=0.1, seed=7, name="case"):
    return tin.LayerConfig(name, n_views, gh, gw, ns, H, d, h, steps, lr, seed)


CONV_CASES = [
    _cfg(2, 8, 8, 0, 1, 16, 32),
    _cfg(3, 37, 37, 5, 2, 64, 256),
    _cfg(1, 1, 1, 0, 1, 32, 64),
    _cfg(2, 5, 7, 2, 16, 64, 256),
    _cfg(1, 2, 3, 5, 1, 64, 256),
    _cfg(2, 41, 41, 1, 1, 32, 64),      # 41 rows: the last 3-row band is ragged (41 = 13 * 3 + 2)
    _cfg(3, 37, 37, 5, 1, 16, 32),      # 16 channels: 4 threads per row, most of the block idle
    _cfg(2, 2, 300, 1, 1, 32, 64),      # 300 columns: many passes of the 8-column shared-memory ring
]


@pytest.mark.parametrize("cfg", CONV_CASES, ids=lambda c: f"{c.n_views}v{c.grid_h}x{c.grid_w}+{c.n_special}_H{c.heads}d{c.d}")
def test_shortconv2d_matches_oracle(cfg):
    inp = tin.make_inputs(cfg)
    dev = to_device(inp)
    out = ttt.shortconv2d(dev["V"], dev["conv_w"], cfg)
    torch.cuda.synchronize()
    n, H, d = inp["V"].shape
    ref = orc.shortconv2d(inp["V"].reshape(n, H * d).double().numpy(), inp["conv_w"].double().numpy(), dims_of(cfg))
    got = out.float().cpu().reshape(n, H * d).double().numpy()
    # fp32 accumulation, one bf16 rounding of the result: within a bf16 half-ulp plus fp32 noise
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5)
    T = cfg.tokens_per_view
    for v in range(cfg.n_views):
        np.testing.assert_array_equal(got[v * T:v * T + cfg.n_special], inp["V"].reshape(n, H * d)[v * T:v * T + cfg.n_special].double().numpy())


READ_CASES = [
    _cfg(2, 8, 8, 0, 1, 16, 32),
    _cfg(3, 5, 7, 2, 2, 64, 256),
    _cfg(4, 37, 37, 5, 3, 64, 256),
    _cfg(2, 9, 9, 1, 2, 32, 100),
    _cfg(1, 1, 1, 0, 1, 64, 128),
]


@pytest.mark.parametrize("cfg", READ_CASES, ids=lambda c: f"n{c.n}_H{c.heads}d{c.d}h{c.h}")
def test_read_matches_oracle(cfg):
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    O = ttt.read(dev["Q"], dev["theta"], cfg)
    torch.cuda.synchronize()
    ref = oracle_layer(cfg, inp, steps=0)
    assert compare_O(O, ref) <= TOL_O


WRITE_CASES = [
    _cfg(2, 8, 8, 0, 1, 16, 32, steps=1, lr=0.1),
    _cfg(3, 5, 7, 2, 2, 64, 256, steps=1),
    _cfg(4, 37, 37, 5, 3, 64, 256, steps=2, lr=0.1),
    _cfg(2, 9, 9, 1, 2, 32, 100, steps=2, lr=0.3),
    _cfg(3, 11, 13, 0, 1, 64, 128, steps=1, lr=0.5),
]


@pytest.mark.parametrize("cfg", WRITE_CASES, ids=lambda c: f"n{c.n}_H{c.heads}d{c.d}h{c.h}_s{c.steps}")
def test_layer_matches_oracle(cfg):
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    theta, O = ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, cfg.steps, cfg)
    torch.cuda.synchronize()
    ref = oracle_layer(cfg, inp)
    t_err, d_err = compare_theta(cfg, inp, theta, ref)
    assert t_err <= TOL_THETA, t_err
    assert d_err <= TOL_DELTA, d_err
    assert compare_O(O, ref) <= TOL_O


def test_write_alone_matches_layer_and_in_place():
    cfg = _cfg(3, 6, 6, 1, 2, 64, 256, steps=2)
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    th_w = ttt.write(dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, cfg.steps, cfg)
    th_l, _ = ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, cfg.steps, cfg)
    inplace = dev["theta"].clone()
    ttt.write(dev["K"], dev["V"], dev["conv_w"], inplace, cfg.lr, cfg.steps, cfg, theta_out=inplace)
    torch.cuda.synchronize()
    assert torch.equal(th_w, th_l)
    assert torch.equal(th_w, inplace)


def test_steps0_and_lr0_keep_theta_exactly():
    cfg = _cfg(2, 5, 5, 0, 2, 64, 256)
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    for lr, steps in [(0.1, 0), (0.0, 2)]:
        th, O = ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], lr, steps, cfg)
        torch.cuda.synchronize()
        assert torch.equal(th, dev["theta"])
        O_read = ttt.read(dev["Q"], dev["theta"], cfg)
        torch.cuda.synchronize()
        assert torch.equal(O, O_read)


def test_deterministic_bitwise():
    cfg = _cfg(5, 37, 37, 5, 4, 64, 256, steps=2)
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    r1 = ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, cfg.steps, cfg)
    r2 = ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, cfg.steps, cfg)
    torch.cuda.synchronize()
    assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])


def test_view_permutation_invariance_on_gpu():
    """theta* does not depend on view order (only the fp32 summation order changes)."""
    cfg = _cfg(6, 9, 9, 2, 2, 64, 256, steps=2)
    T = cfg.tokens_per_view
    perm = [4, 1, 5, 0, 3, 2]
    a = bf16_inputs(tin.make_inputs(cfg))
    b = bf16_inputs(tin.make_inputs(cfg, views=perm))
    da, db = to_device(a), to_device(b)
    tha, Oa = ttt.layer(da["Q"], da["K"], da["V"], da["conv_w"], da["theta"], cfg.lr, cfg.steps, cfg)
    thb, Ob = ttt.layer(db["Q"], db["K"], db["V"], db["conv_w"], db["theta"], cfg.lr, cfg.steps, cfg)
    torch.cuda.synchronize()
    d0 = (tha - da["theta"]).double().cpu().numpy()
    d1 = (thb - db["theta"]).double().cpu().numpy()
    assert normwise(d1, d0) <= 2e-3
    idx = torch.cat([torch.arange(p * T, (p + 1) * T) for p in perm])
    assert normwise(Ob.float().cpu().numpy(), Oa.float().cpu()[idx].numpy()) <= 1e-2


def test_status_ok_after_runs():
    cfg = _cfg(2, 8, 8, 0, 1, 64, 256)
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    ws = ttt.make_workspace(cfg, ttt.OP_LAYER)
    ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, cfg.steps, cfg, workspace=ws)
    assert ttt.check_status(ws) == 0


def test_device_errors_reported():
    cfg = _cfg(2, 8, 8, 0, 1, 64, 256)
    inp = bf16_inputs(tin.make_inputs(cfg))
    dev = to_device(inp)
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(ttt.TTTError) as e:
        ttt.layer(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], cfg.lr, 1, cfg, workspace=small)
    assert e.value.status == -4
