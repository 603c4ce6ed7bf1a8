"""Canary and poison checks of the entry points on a GPU (compute-sanitizer is
not available here).  Every input, output and the workspace sit inside
4 KiB canary bands; outputs start as NaN.  After the call: the canaries are
intact (nothing written out of bounds), inputs are unchanged, no output
element is left unwritten, and the device status word is clear.  Shapes are
ragged on purpose: 3 views of 5x7 + 2 special tokens (the last 128-token tile
partial), two heads, d=64, h=192 (hidden padded to 256 inside), and a 1x1 /
2x3 grid for the conv."""
import pytest
import torch

from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import ttt
from ttt_testlib import guarded, guards_intact

pytestmark = pytest.mark.gpu

CFG = tin.LayerConfig("guards_3v_5x7p2_h2_d64_h192", 3, 5, 7, 2, 2, 64, 192, 2, 0.1, 51)
NAN = float("nan")


def _guarded_inputs(cfg):
    inp = tin.make_inputs(cfg)
    out, keep = {}, {}
    for k in ("Q", "K", "V"):
        t = inp[k].to(torch.bfloat16).contiguous()
        out[k], keep[k + "_buf"] = guarded(tuple(t.shape), torch.bfloat16, "cuda")
        out[k].copy_(t.cuda())
    w = inp["conv_w"].float().contiguous()
    out["conv_w"], keep["conv_w_buf"] = guarded(tuple(w.shape), torch.float32, "cuda")
    out["conv_w"].copy_(w.cuda())
    th = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"])
    out["theta"], keep["theta_buf"] = guarded(tuple(th.shape), torch.float32, "cuda")
    out["theta"].copy_(th.cuda())
    ref = {k: out[k].clone() for k in ("Q", "K", "V", "conv_w", "theta")}
    return out, keep, ref


def _workspace(cfg, op):
    ws, ws_buf = guarded((ttt.workspace_bytes(cfg, op),), torch.uint8, "cuda")
    return ws, ws_buf


def _check(dev, keep, ref, outs, ws_buf, ws):
    torch.cuda.synchronize()
    assert ttt.check_status(ws) == 0
    assert all(guards_intact(b) for b in keep.values())
    assert guards_intact(ws_buf)
    for k, v in ref.items():
        assert torch.equal(dev[k], v), k
    for name, (t, buf) in outs.items():
        assert guards_intact(buf), name
        assert not torch.isnan(t.float()).any(), name


@pytest.mark.parametrize("which", ["layer", "layer_muon"])
def test_layer_guards_and_poison(which):
    dev, keep, ref = _guarded_inputs(CFG)
    theta_out, th_buf = guarded(tuple(dev["theta"].shape), torch.float32, "cuda", fill=NAN)
    O, o_buf = guarded(tuple(dev["Q"].shape), torch.bfloat16, "cuda", fill=NAN)
    ws, ws_buf = _workspace(CFG, ttt.OP_LAYER)
    fn = ttt.layer if which == "layer" else ttt.layer_muon
    fn(dev["Q"], dev["K"], dev["V"], dev["conv_w"], dev["theta"], CFG.lr, CFG.steps, CFG, theta_out=theta_out, O=O,
       workspace=ws)
    _check(dev, keep, ref, {"theta_out": (theta_out, th_buf), "O": (O, o_buf)}, ws_buf, ws)


def test_write_read_grad_guards_and_poison():
    dev, keep, ref = _guarded_inputs(CFG)
    theta_out, th_buf = guarded(tuple(dev["theta"].shape), torch.float32, "cuda", fill=NAN)
    ws, ws_buf = _workspace(CFG, ttt.OP_WRITE)
    ttt.write(dev["K"], dev["V"], dev["conv_w"], dev["theta"], CFG.lr, CFG.steps, CFG, theta_out=theta_out,
              workspace=ws)
    _check(dev, keep, ref, {"theta_out": (theta_out, th_buf)}, ws_buf, ws)
    Vp, vp_buf = guarded(tuple(dev["V"].shape), torch.bfloat16, "cuda", fill=NAN)
    ttt.shortconv2d(dev["V"], dev["conv_w"], CFG, out=Vp)
    g, g_buf = guarded(tuple(dev["theta"].shape), torch.float32, "cuda", fill=NAN)
    ttt.grad(dev["K"], Vp, dev["theta"], CFG, out=g, workspace=ws)
    _check(dev, keep, ref, {"Vp": (Vp, vp_buf), "grad": (g, g_buf)}, ws_buf, ws)
    O, o_buf = guarded(tuple(dev["Q"].shape), torch.bfloat16, "cuda", fill=NAN)
    wsr, wsr_buf = _workspace(CFG, ttt.OP_READ)
    ttt.read(dev["Q"], dev["theta"], CFG, O=O, workspace=wsr)
    _check(dev, keep, ref, {"O": (O, o_buf)}, wsr_buf, wsr)


@pytest.mark.parametrize("gh,gw,ns", [(1, 1, 0), (1, 1, 5), (2, 3, 5)])
def test_conv_tiny_grids_guards_and_poison(gh, gw, ns):
    cfg = tin.LayerConfig("guards_conv", 2, gh, gw, ns, 2, 16, 32, 1, 0.1, 52)
    dev, keep, ref = _guarded_inputs(cfg)
    Vp, vp_buf = guarded(tuple(dev["V"].shape), torch.bfloat16, "cuda", fill=NAN)
    ttt.shortconv2d(dev["V"], dev["conv_w"], cfg, out=Vp)
    torch.cuda.synchronize()
    assert all(guards_intact(b) for b in keep.values()) and guards_intact(vp_buf)
    assert not torch.isnan(Vp.float()).any()
    for k, v in ref.items():
        assert torch.equal(dev[k], v), k
