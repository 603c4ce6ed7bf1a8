"""The control flow of the host-streamed layer on CPU, with float64 oracle
operations in place of the kernels: the write over chunks of whole views
equals the oracle's single-pass full-batch write (Eq. 5), for both inner
loops and for chunkings that do and do not divide the views; the streamed
read equals the oracle read; steps = 0 returns theta0."""
import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc
from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import sharded, stream
from test_multirank_sharded import _odims, _pack, _unpack, oracle_muon_ops, oracle_ops

CFG = tin.LayerConfig("stream_cpu_5v_6x7p2_h2_d16_h32", 5, 6, 7, 2, 2, 16, 32, 2, 0.5, 41)


def _with_out(ops: sharded.ShardOps) -> sharded.ShardOps:
    base = ops.grad

    def grad(K, Vp, theta, cfg, out=None):
        g = base(K, Vp, theta, cfg)
        if out is not None:
            out.copy_(g)
            return out
        return g

    return sharded.ShardOps(conv=ops.conv, grad=grad, update=ops.update, read=ops.read, step_size=ops.step_size)


def test_view_chunks():
    assert stream.view_chunks(5, 2) == [(0, 2), (2, 4), (4, 5)]
    assert stream.view_chunks(5, 9) == [(0, 5)]
    with pytest.raises(ValueError):
        stream.view_chunks(5, 0)


@pytest.mark.parametrize("inner,lr", [("sgd", 0.5), ("muon", 0.1)])
@pytest.mark.parametrize("chunk_views", [1, 2, 5])
def test_streamed_write_and_read_match_oracle(inner, lr, chunk_views):
    inp = tin.make_inputs(CFG)
    K, V, Q = (inp[k].double() for k in ("K", "V", "Q"))
    th0 = _pack(*(inp[k].double().numpy() for k in ("W1", "W3", "W2")))
    ops = _with_out(oracle_ops() if inner == "sgd" else oracle_muon_ops())
    theta = stream.write_streamed(K, V, inp["conv_w"], th0, lr, CFG.steps, CFG, chunk_views, inner, ops)
    O = stream.read_streamed(Q, theta, CFG, chunk_views, ops=ops)
    assert torch.equal(stream.write_streamed(K, V, inp["conv_w"], th0, lr, 0, CFG, chunk_views, inner, ops), th0)

    Kn, Vn, Qn = K.numpy(), V.numpy(), Q.numpy()
    n, H, d = Kn.shape
    Vp = orc.shortconv2d(Vn.reshape(n, H * d), inp["conv_w"].double().numpy(), _odims(CFG)).reshape(n, H, d)
    W0 = [inp[k].double().numpy() for k in ("W1", "W3", "W2")]
    ref = [np.zeros_like(w) for w in W0]
    write = orc.sgd_write if inner == "sgd" else orc.muon_write
    for hd in range(H):
        th, _ = write(Kn[:, hd], Vp[:, hd], [w[hd] for w in W0], lr, CFG.steps)
        for m in range(3):
            ref[m][hd] = th[m]
    ref_flat = _pack(*ref).numpy()
    delta_ref = ref_flat - th0.numpy()
    tol = 1e-6 if inner == "sgd" else 1e-10   # SGD's step size is rounded to single precision
    assert np.max(np.abs(theta.numpy() - ref_flat)) <= tol * np.max(np.abs(delta_ref))
    W = _unpack(theta, CFG)
    O_ref = np.stack([orc.read(Qn[:, hd], W[0][hd], W[1][hd], W[2][hd]) for hd in range(H)], axis=1)
    np.testing.assert_allclose(O.numpy(), O_ref, rtol=0, atol=1e-12 * np.max(np.abs(O_ref)))
