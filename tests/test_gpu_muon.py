"""GPU parity of the pages' own inner loop (dot-product loss, Muon steps),
through the C ABI: ttt_write_muon / ttt_layer_muon and the sharded pieces
ttt_grad_dot / ttt_muon_update.

Tolerances.  The Newton-Schulz step is checked against the oracle on the same
gradient (FP32 iteration against float64: 1e-4 of the step).  The dot-product
gradient has the mean-squared path's error (bf16 operands, FP32
accumulation): 2e-2, as for the SGD update.  The oracle shows that NS5
magnifies an elementwise relative gradient perturbation about 3x on these
gradients (1e-2 noise moves the step by 3.1e-2), so the Muon update itself
is held to 3 x 2e-2 = 6e-2 of its size and theta* to what that implies; the
read O is held to the layer's own 2e-2.
"""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc
from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import sharded, ttt
from ttt_testlib import TOL_DELTA, TOL_O, dims_of, normwise, report

pytestmark = pytest.mark.gpu

TOL_MUON_DELTA = 3 * TOL_DELTA
LR = 0.1          # the pages' inner learning rate


def _device(cfg):
    inp = tin.make_inputs(cfg)
    dev = {k: inp[k].to(torch.bfloat16).contiguous().cuda() for k in ("Q", "K", "V")}
    dev["conv_w"] = inp["conv_w"].float().contiguous().cuda()
    dev["theta"] = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).cuda()
    return inp, dev


def _oracle_muon(cfg, inp, steps, heads):
    dims = dims_of(cfg)
    out = {}
    n, H, d = inp["K"].shape
    for hd in heads:
        ch = slice(hd * d, (hd + 1) * d)
        vp = orc.shortconv2d(inp["V"][:, hd].double().numpy(), inp["conv_w"][ch].double().numpy(), dims)
        th0 = [inp[k][hd].double().numpy() for k in ("W1", "W3", "W2")]
        th, _ = orc.muon_write(inp["K"][:, hd].double().numpy(), vp, th0, LR, steps)
        out[hd] = (th0, th, orc.read(inp["Q"][:, hd].double().numpy(), *th))
    return out


@pytest.mark.parametrize("heads,d,h", [(2, 64, 256), (3, 16, 32), (1, 32, 192)])
def test_muon_update_matches_oracle_newton_schulz(heads, d, h):
    cfg = tin.LayerConfig("muon_ns", 1, 4, 4, 0, heads, d, h, 1, LR, 0)
    g = torch.Generator().manual_seed(d + h)
    count = 3 * heads * d * h
    theta = torch.randn(count, generator=g) * 0.1
    grads = torch.randn(2, count, generator=g)
    out = ttt.muon_update(theta.cuda(), grads.cuda(), LR, cfg)
    torch.cuda.synchronize()
    Gs = tin.unpack_theta((grads[0] + grads[1]).double(), heads, d, h)
    Ts = tin.unpack_theta(theta.double(), heads, d, h)
    Os = tin.unpack_theta(out.double().cpu(), heads, d, h)
    for m in range(3):
        for hd in range(heads):
            ns = orc.newton_schulz(Gs[m][hd].numpy())
            step = (Ts[m][hd].numpy() - Os[m][hd].numpy()) / LR
            assert normwise(step, ns) <= 1e-4, (m, hd)


def test_grad_dot_matches_oracle():
    cfg = tin.CONFIGS["views24_37x37p5_h16_d64_h256"].with_views(6)
    inp, dev = _device(cfg)
    Vp = ttt.shortconv2d(dev["V"], dev["conv_w"], cfg)
    g = ttt.grad_dot(dev["K"], Vp, dev["theta"], cfg)
    torch.cuda.synchronize()
    G = [t.double().numpy() for t in tin.unpack_theta(g.cpu(), cfg.heads, cfg.d, cfg.h)]
    dims = dims_of(cfg)
    n, H, d = inp["K"].shape
    for hd in range(H):
        ch = slice(hd * d, (hd + 1) * d)
        vp = orc.shortconv2d(inp["V"][:, hd].double().numpy(), inp["conv_w"][ch].double().numpy(), dims)
        ref = orc.dot_grad(inp["K"][:, hd].double().numpy(), vp, inp["W1"][hd].double().numpy(),
                           inp["W3"][hd].double().numpy(), inp["W2"][hd].double().numpy())
        for m in range(3):
            assert normwise(G[m][hd], ref[m] * n) <= TOL_DELTA, (hd, m)


@pytest.mark.parametrize("name,heads", [("tiny_2v_8x8_d16_h32", [0]), ("views24_37x37p5_h16_d64_h256", [0, 7, 15])])
def test_layer_muon_matches_oracle(name, heads):
    cfg = tin.CONFIGS[name]
    inp, dev = _device(cfg)
    if cfg.fp32_inputs:   # the GPU takes bf16 tokens; give the oracle the same values
        for k in ("Q", "K", "V"):
            inp[k] = tin.bf16_round(inp[k])
    theta, O = ttt.layer_muon(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], LR, 2, cfg)
    torch.cuda.synchronize()
    W = [t.double().numpy() for t in tin.unpack_theta(theta.cpu(), cfg.heads, cfg.d, cfg.h)]
    Og = O.double().cpu().numpy()
    worst_d, worst_t, worst_o = 0.0, 0.0, 0.0
    for hd, (th0, th_ref, O_ref) in _oracle_muon(cfg, inp, 2, heads).items():
        for m in range(3):
            d_ref = th_ref[m] - th0[m]
            e_d = normwise(W[m][hd] - th0[m], d_ref)
            e_t = normwise(W[m][hd], th_ref[m])
            worst_d, worst_t = max(worst_d, e_d), max(worst_t, e_t)
            assert e_d <= TOL_MUON_DELTA, (hd, m)
            # theta* moves by at most the step's error
            assert e_t <= TOL_MUON_DELTA * np.max(np.abs(d_ref)) / np.max(np.abs(th_ref[m]))
        worst_o = max(worst_o, normwise(Og[:, hd], O_ref))
    report(f"muon_{name}", delta=worst_d, theta=worst_t, O=worst_o)
    assert worst_o <= TOL_O, worst_o


def test_muon_write_equals_its_pieces_bitwise():
    """ttt_write_muon = ttt_shortconv2d, then per step ttt_grad_dot + ttt_muon_update
    (what one rank of the sharded write runs)."""
    cfg = tin.CONFIGS["views24_37x37p5_h16_d64_h256"].with_views(5)
    _, dev = _device(cfg)
    full = ttt.write_muon(dev["K"], dev["V"], dev["conv_w"], dev["theta"], LR, 2, cfg)
    pieces = sharded.write_sharded(dev["K"], dev["V"], dev["conv_w"], dev["theta"], LR, 2, cfg, cfg.n,
                                   gather=lambda t: t.reshape(1, -1), ops=sharded.cuda_ops(cfg, "muon"))
    zero = ttt.write_muon(dev["K"], dev["V"], dev["conv_w"], dev["theta"], LR, 0, cfg)
    torch.cuda.synchronize()
    assert torch.equal(full, pieces)
    assert torch.equal(zero, dev["theta"])


# The wide-head path (d, h multiples of 64 beyond the fused kernels): the
# gradient on the tensor-core GEMM with V' in place of the residual, and
# Newton-Schulz on the GEMM with each FP32 operand split into a bf16 pair
# (about 2^-16 relative per product), FP32 accumulation.
WIDE_CASES = [tin.LayerConfig("muon_wide_small", 3, 9, 10, 2, 2, 128, 192, 2, LR, 51),
              tin.CONFIGS["views2000_37x37p5_h1_d1024_h2048"].with_views(4)]


@pytest.mark.parametrize("cfg", WIDE_CASES, ids=["d128_h192", "d1024_h2048"])
def test_wide_layer_muon_matches_oracle(cfg):
    inp, dev = _device(cfg)
    theta, O = ttt.layer_muon(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], LR, 2, cfg)
    torch.cuda.synchronize()
    W = [t.double().numpy() for t in tin.unpack_theta(theta.cpu(), cfg.heads, cfg.d, cfg.h)]
    Og = O.double().cpu().numpy()
    worst_d, worst_o = 0.0, 0.0
    for hd, (th0, th_ref, O_ref) in _oracle_muon(cfg, inp, 2, list(range(cfg.heads))).items():
        for m in range(3):
            worst_d = max(worst_d, normwise(W[m][hd] - th0[m], th_ref[m] - th0[m]))
        worst_o = max(worst_o, normwise(Og[:, hd], O_ref))
    report(f"muon_wide_{cfg.d}_{cfg.h}", delta=worst_d, O=worst_o)
    assert worst_d <= TOL_MUON_DELTA, worst_d
    assert worst_o <= TOL_O, worst_o


def test_wide_grad_dot_matches_oracle():
    cfg = WIDE_CASES[0]
    inp, dev = _device(cfg)
    Vp = ttt.shortconv2d(dev["V"], dev["conv_w"], cfg)
    g = ttt.grad_dot(dev["K"], Vp, dev["theta"], cfg)
    torch.cuda.synchronize()
    G = [t.double().numpy() for t in tin.unpack_theta(g.cpu(), cfg.heads, cfg.d, cfg.h)]
    dims = dims_of(cfg)
    n, H, d = inp["K"].shape
    worst = 0.0
    for hd in range(H):
        ch = slice(hd * d, (hd + 1) * d)
        vp = orc.shortconv2d(inp["V"][:, hd].double().numpy(), inp["conv_w"][ch].double().numpy(), dims)
        ref = orc.dot_grad(inp["K"][:, hd].double().numpy(), vp, inp["W1"][hd].double().numpy(),
                           inp["W3"][hd].double().numpy(), inp["W2"][hd].double().numpy())
        worst = max(worst, *(normwise(G[m][hd], ref[m] * n) for m in range(3)))
    report("muon_wide_grad_dot", grad=worst)
    assert worst <= TOL_DELTA, worst


def test_wide_muon_write_is_deterministic_and_lr0_keeps_theta():
    cfg = WIDE_CASES[0]
    _, dev = _device(cfg)
    a = ttt.write_muon(dev["K"], dev["V"], dev["conv_w"], dev["theta"], LR, 2, cfg)
    b = ttt.write_muon(dev["K"], dev["V"], dev["conv_w"], dev["theta"], LR, 2, cfg)
    z = ttt.write_muon(dev["K"], dev["V"], dev["conv_w"], dev["theta"], 0.0, 2, cfg)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(z, dev["theta"])
