"""The view-sharded write on two gloo ranks on CPU.

test_layer_reconstruction_b200.sharded holds the control flow of the write
split by views over processes: convolve the rank's views, then per step its
gradient sum, an all-gather, and one fixed-order update.  Here that control
flow runs on two spawned gloo ranks with float64 oracle operations in place
of the kernels, on a collection of 5 views split 2 + 3.  Checked:

* theta* equals the oracle's single-process full-batch write over all views
  (the gradient over all tokens is the sum of the shards' sums, Eq. 5);
* theta* is bit-identical on both ranks (same gathered sums, same order);
* each rank's read equals the oracle read of its own queries with theta*;
* steps = 0 returns theta0;
* the pages' inner loop (dot-product loss, Muon on the summed gradient) run
  the same way equals the oracle's single-process Muon write.
"""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import ttt_oracle as orc
from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import sharded

CFG = tin.LayerConfig("shard_cpu_5v_6x7p2_h2_d16_h32", 5, 6, 7, 2, 2, 16, 32, 2, 0.5, 31)
SPLIT = ((0, 2), (2, 5))   # views of rank 0 and rank 1


def _odims(cfg):
    return orc.Dims(cfg.n_views, cfg.grid_h, cfg.grid_w, cfg.n_special)


def _unpack(theta, cfg):
    return [t.numpy() for t in tin.unpack_theta(theta, cfg.heads, cfg.d, cfg.h)]


def _pack(W1, W3, W2):
    """theta's packed layout in float64 (pack_theta itself stores float32)."""
    return torch.from_numpy(np.concatenate([np.asarray(w, np.float64).reshape(-1) for w in (W1, W3, W2)]))


def oracle_ops() -> sharded.ShardOps:
    """float64 oracle operations with the kernels' contracts (ttt_grad returns the
    gradient of (1/2) sum ||T(k) - v'||^2, i.e. n/2 times the mean-loss gradient)."""

    def conv(V, conv_w, cfg):
        n, H, d = V.shape
        out = orc.shortconv2d(V.reshape(n, H * d).numpy(), conv_w.double().numpy(), _odims(cfg))
        return torch.from_numpy(out).reshape(n, H, d)

    def grad(K, Vp, theta, cfg):
        W1, W3, W2 = _unpack(theta, cfg)
        g = [np.zeros_like(W1), np.zeros_like(W3), np.zeros_like(W2)]
        n = K.shape[0]
        for hd in range(cfg.heads):
            gh = orc.mse_grad(K[:, hd].numpy(), Vp[:, hd].numpy(), W1[hd], W3[hd], W2[hd])
            for m in range(3):
                g[m][hd] = gh[m] * (n / 2.0)
        return _pack(*g)

    def update(theta, grads, scale, cfg):
        total = grads[0].clone()
        for r in range(1, grads.shape[0]):
            total += grads[r]
        return theta - scale * total

    def read(Q, theta, cfg):
        W1, W3, W2 = _unpack(theta, cfg)
        return torch.from_numpy(np.stack([orc.read(Q[:, hd].numpy(), W1[hd], W3[hd], W2[hd])
                                          for hd in range(cfg.heads)], axis=1))

    return sharded.ShardOps(conv=conv, grad=grad, update=update, read=read)


def oracle_muon_ops() -> sharded.ShardOps:
    """The dot-product loss and Muon with the kernels' contracts (ttt_grad_dot returns
    the gradient of -sum <T(k), v'>, n times the mean loss's; ttt_muon_update takes lr)."""
    base = oracle_ops()

    def grad(K, Vp, theta, cfg):
        W1, W3, W2 = _unpack(theta, cfg)
        g = [np.zeros_like(W1), np.zeros_like(W3), np.zeros_like(W2)]
        n = K.shape[0]
        for hd in range(cfg.heads):
            gh = orc.dot_grad(K[:, hd].numpy(), Vp[:, hd].numpy(), W1[hd], W3[hd], W2[hd])
            for m in range(3):
                g[m][hd] = gh[m] * n
        return _pack(*g)

    def update(theta, grads, lr, cfg):
        total = grads[0].clone()
        for r in range(1, grads.shape[0]):
            total += grads[r]
        G = _unpack(total, cfg)
        W = _unpack(theta, cfg)
        new = [np.stack([W[m][hd] - lr * orc.newton_schulz(G[m][hd]) for hd in range(cfg.heads)]) for m in range(3)]
        return _pack(*new)

    return sharded.ShardOps(conv=base.conv, grad=grad, update=update, read=base.read,
                            step_size=sharded.muon_step_size)


def _gloo_gather(t):
    parts = [torch.empty_like(t.reshape(-1)) for _ in range(dist.get_world_size())]
    dist.all_gather(parts, t.reshape(-1).contiguous())
    return torch.stack(parts)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        a, b = SPLIT[rank]
        local = CFG.with_views(b - a)
        inp = tin.make_inputs(CFG, views=range(a, b))
        Q, K, V = (inp[k].double() for k in ("Q", "K", "V"))
        th0 = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).double()
        ops = oracle_ops()
        theta, O = sharded.layer_sharded(Q, K, V, inp["conv_w"], th0, CFG.lr, CFG.steps, local, CFG.n,
                                         _gloo_gather, ops)
        theta_ranks = _gloo_gather(theta)
        th_zero = sharded.write_sharded(K, V, inp["conv_w"], th0, CFG.lr, 0, local, CFG.n, _gloo_gather, ops)
        th_muon = sharded.write_sharded(K, V, inp["conv_w"], th0, 0.1, 2, local, CFG.n, _gloo_gather,
                                        oracle_muon_ops())
        q.put((rank, theta.numpy(), O.numpy(), theta_ranks.numpy(), bool(torch.equal(th_zero, th0)),
               th_muon.numpy()))
    finally:
        dist.destroy_process_group()


def test_sharded_write_two_gloo_ranks_matches_single_process_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    # the single-process reference: full-batch SGD over all 5 views
    inp = tin.make_inputs(CFG)
    K, V, Qall = (inp[k].double().numpy() for k in ("K", "V", "Q"))
    n, H, d = K.shape
    Vp = orc.shortconv2d(V.reshape(n, H * d), inp["conv_w"].double().numpy(), _odims(CFG)).reshape(n, H, d)
    th0 = [t.double().numpy() for t in (inp["W1"], inp["W3"], inp["W2"])]
    ref = [np.zeros_like(w) for w in th0]
    for hd in range(H):
        th, _ = orc.sgd_write(K[:, hd], Vp[:, hd], [w[hd] for w in th0], CFG.lr, CFG.steps)
        for m in range(3):
            ref[m][hd] = th[m]
    ref_flat = _pack(*ref).numpy()
    th0_flat = _pack(*th0).numpy()

    (_, th_a, O_a, ranks_a, zero_a, mu_a), (_, th_b, O_b, ranks_b, zero_b, mu_b) = results
    assert np.array_equal(th_a, th_b) and np.array_equal(ranks_a[0], ranks_a[1])
    assert zero_a and zero_b
    delta, delta_ref = th_a - th0_flat, ref_flat - th0_flat
    # the update's scale is rounded to single precision, as the kernels take it
    assert np.max(np.abs(delta - delta_ref)) <= 1e-6 * np.max(np.abs(delta_ref))
    assert np.max(np.abs(delta_ref)) > 1e-3                     # the write moved theta
    W = [w for w in _unpack(torch.from_numpy(th_a), CFG)]
    tpv = CFG.tokens_per_view
    for (a, b), O in zip(SPLIT, (O_a, O_b)):
        Qr = Qall[a * tpv:b * tpv]
        O_ref = np.stack([orc.read(Qr[:, hd], W[0][hd], W[1][hd], W[2][hd]) for hd in range(H)], axis=1)
        assert np.max(np.abs(O - O_ref)) <= 1e-12 * np.max(np.abs(O_ref))

    # the pages' inner loop, sharded the same way: the oracle's Muon write over all views
    assert np.array_equal(mu_a, mu_b)
    mref = [np.zeros_like(w) for w in th0]
    for hd in range(H):
        th, _ = orc.muon_write(K[:, hd], Vp[:, hd], [w[hd] for w in th0], 0.1, 2)
        for m in range(3):
            mref[m][hd] = th[m]
    mref_flat = _pack(*mref).numpy()
    assert np.max(np.abs(mu_a - mref_flat)) <= 1e-10 * np.max(np.abs(mref_flat - th0_flat))


def _failing_worker(rank: int, world: int, port: int, q) -> None:
    """Rank 1 leaves after its gradient, before the first exchange; rank 0 must
    get an error from the exchange, not hang."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
    a, b = SPLIT[rank]
    local = CFG.with_views(b - a)
    inp = tin.make_inputs(CFG, views=range(a, b))
    K, V = (inp[k].double() for k in ("K", "V"))
    th0 = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).double()
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()   # the message is out before the process vanishes
        os._exit(0)       # gone without a word: no destroy, no collective
    try:
        sharded.write_sharded(K, V, inp["conv_w"], th0, CFG.lr, 2, local, CFG.n, _gloo_gather, oracle_ops())
        q.put((rank, "no error"))
    except RuntimeError as exc:
        q.put((rank, str(exc)))
    q.close()
    q.join_thread()
    os._exit(0)


def test_sharded_write_reports_a_rank_that_left():
    import time
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    t0 = time.monotonic()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert results[1] == "left"
    assert "gradient exchange of step 0 failed" in results[0], results[0]
    assert time.monotonic() - t0 < 120

