"""GPU parity of the layer's surround (ttt_attention) through the C ABI:
q = L2(X Wq), k = L2(X Wk) per (token, head) row, v = X Wv on the tensor-core
GEMM with the normalisation in its epilogue, the TTT layer (both inner
loops), and out = O Wo, against the oracle's ttt_attention on the same bf16
values.

Tolerances: theta* <= 1e-2 and out <= 2e-2 (norm-wise, as for the layer);
the update delta <= 2e-2 beyond the float32 resolution of theta* for the
mean-squared inner loop, and the Muon update within 3 x 2e-2 (NS5 magnifies
a relative gradient error about 3x, as in the Muon tests).  q and k are
rounded to bf16 after the normalisation on the GPU, which these bounds
cover."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc
from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import ttt
from ttt_testlib import TOL_DELTA, TOL_O, TOL_THETA, delta_error, dims_of, normwise, report

pytestmark = pytest.mark.gpu


def _run(cfg, inner, lr):
    inp = tin.make_surround(cfg)
    dev = {k: inp[k].to(torch.bfloat16).contiguous().cuda() for k in ("X", "Wq", "Wk", "Wv", "Wo")}
    conv_w = inp["conv_w"].contiguous().cuda()
    theta0 = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).cuda()
    theta, out = ttt.attention(dev["X"], dev["Wq"], dev["Wk"], dev["Wv"], dev["Wo"], conv_w, theta0, lr,
                               cfg.steps, cfg, inner=inner)
    torch.cuda.synchronize()
    ref_out, r1, r3, r2 = orc.ttt_attention(
        inp["X"].double().numpy(), inp["Wq"].double().numpy(), inp["Wk"].double().numpy(),
        inp["Wv"].double().numpy(), inp["Wo"].double().numpy(), inp["conv_w"].double().numpy(),
        inp["W1"].double().numpy(), inp["W3"].double().numpy(), inp["W2"].double().numpy(), lr, cfg.steps,
        dims_of(cfg), inner="sgd" if inner == ttt.INNER_SGD else "muon")
    g1, g3, g2 = (t.double().numpy() for t in tin.unpack_theta(theta.cpu(), cfg.heads, cfg.d, cfg.h))
    t0 = (inp["W1"].double().numpy(), inp["W3"].double().numpy(), inp["W2"].double().numpy())
    return inp, out, ref_out, (g1, g3, g2), (r1, r3, r2), t0


@pytest.mark.parametrize("cfg", [tin.LayerConfig("surround_small", 3, 9, 10, 2, 4, 64, 256, 2, 0.1, 31),
                                 tin.CONFIGS["views24_37x37p5_h16_d64_h256"]],
                         ids=["small", "views24"])
def test_attention_sgd_matches_oracle(cfg):
    inp, out, ref_out, g, r, t0 = _run(cfg, ttt.INNER_SGD, cfg.lr)
    t_err = max(normwise(a, b) for a, b in zip(g, r))
    d_err = max(delta_error(a, b, c, cfg.steps) for a, b, c in zip(g, r, t0))
    o_err = normwise(out.double().cpu().numpy(), ref_out)
    report(f"attention_sgd_{cfg.name}", theta=t_err, delta=d_err, out=o_err)
    assert t_err <= TOL_THETA and d_err <= TOL_DELTA, (t_err, d_err)
    assert o_err <= TOL_O, o_err


def test_attention_muon_matches_oracle():
    cfg = tin.CONFIGS["views24_37x37p5_h16_d64_h256"]
    inp, out, ref_out, g, r, t0 = _run(cfg, ttt.INNER_MUON, 0.1)
    d_err = max(normwise(a - c, b - c) for a, b, c in zip(g, r, t0))
    o_err = normwise(out.double().cpu().numpy(), ref_out)
    report("attention_muon_views24", delta=d_err, out=o_err)
    assert d_err <= 3 * TOL_DELTA, d_err
    assert o_err <= TOL_O, o_err


def test_projection_alone_gives_unit_rows():
    """With lr = 0 the layer reads T_theta0(q); the projection's q and k rows are
    unit rows: checked through steps = 0, where out = T_theta0(L2(X Wq)) Wo."""
    cfg = tin.LayerConfig("surround_lr0", 2, 5, 6, 1, 2, 64, 128, 0, 0.0, 32)
    inp, out, ref_out, g, r, t0 = _run(cfg, ttt.INNER_SGD, 0.0)
    for a, c in zip(g, t0):
        assert np.array_equal(a, c.astype(np.float32).astype(np.float64))
    assert normwise(out.double().cpu().numpy(), ref_out) <= TOL_O


def test_attention_refuses_other_head_widths():
    cfg = tin.LayerConfig("surround_d32", 1, 2, 2, 0, 2, 32, 64, 1, 0.1, 33)
    X = torch.zeros(cfg.n, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    conv_w = torch.zeros(64, 3, 3, device="cuda")
    theta0 = torch.zeros(3 * 2 * 32 * 64, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(ttt.TTTError) as e:
        ttt.attention(X, W, W, W, W, conv_w, theta0, 0.1, 1, cfg, workspace=ws)
    assert e.value.status == -3
