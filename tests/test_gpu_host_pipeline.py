"""ttt_layer_host against ttt_layer on the same inputs, bit for bit.

The host entry point copies its inputs up and its outputs back in a pipeline:
Q and O move in chunks of whole 128-token tiles on helper streams, and each
chunk of Q is read as soon as it has landed.  The kernels and their inputs
are those of ttt_layer, and the read computes every tile on its own, so
theta* and O must equal the device entry point's exactly.

Covered: one chunk (tiny workload); five chunks with a ragged last tile
(24 views of 37x37+5, 258 tiles); pageable host memory; a caller stream other
than the default one; the wide-head path, which copies in order.
"""
import contextlib

import pytest
import torch

from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import ttt

pytestmark = pytest.mark.gpu


def _host_vs_device(cfg, pinned=True, stream=None):
    inp = tin.make_inputs(cfg)
    Q, K, V = (inp[k].to(torch.bfloat16).contiguous() for k in ("Q", "K", "V"))
    w = inp["conv_w"].float().contiguous()
    th0 = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).float().contiguous()
    theta_d, O_d = ttt.layer(Q.cuda(), K.cuda(), V.cuda(), w.cuda(), th0.cuda(), cfg.lr, cfg.steps, cfg)
    torch.cuda.synchronize()

    def host(t):
        return t.pin_memory() if pinned else t.clone()

    hq, hk, hv, hw, ht0 = (host(t) for t in (Q, K, V, w, th0))
    hth, ho = host(torch.full_like(th0, float("nan"))), host(torch.zeros_like(Q))
    ws = ttt.make_workspace(cfg, ttt.OP_LAYER_HOST)
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        ttt.layer_host(hq, hk, hv, hw, ht0, cfg.lr, cfg.steps, cfg, hth, ho, ws)
        assert ttt.check_status(ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(hth, theta_d.cpu())
    assert torch.equal(ho.view(torch.int16), O_d.cpu().view(torch.int16))
    # inputs are never modified
    assert torch.equal(hq, Q) and torch.equal(hk, K) and torch.equal(hv, V) and torch.equal(ht0, th0)


def test_host_pipeline_one_chunk():
    _host_vs_device(tin.CONFIGS["tiny_2v_8x8_d16_h32"])


def test_host_pipeline_ragged_chunks():
    cfg = tin.CONFIGS["views24_37x37p5_h16_d64_h256"]
    assert (cfg.n + 127) // 128 == 258          # 4 chunks of 64 tiles and one of 2; last tile 80 tokens
    _host_vs_device(cfg)


def test_host_pipeline_pageable_memory_and_own_stream():
    cfg = tin.CONFIGS["views24_37x37p5_h16_d64_h256"].with_views(7)
    _host_vs_device(cfg, pinned=False)
    _host_vs_device(cfg, stream=torch.cuda.Stream())


def test_host_wide_path():
    cfg = tin.LayerConfig("wide_small", 3, 9, 11, 2, 2, 128, 192, 2, 0.1, 21)
    _host_vs_device(cfg)
