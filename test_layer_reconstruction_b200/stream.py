"""The layer for collections whose tokens do not fit in device memory,
streamed from pinned host memory.

The gradient of the TTT loss is a sum of per-token terms, so it can be built
a minibatch of tokens at a time (VGG-T$^3$: Offline Feed-Forward 3D
Reconstruction at Scale, Sec. 3.4, Eq. 5 and "Large-Scale Inference
Strategies": load a minibatch, compute its gradient, accumulate, move on, and
apply the accumulated gradient once).  Here a minibatch is a chunk of whole
views, so ShortConv2D stays inside it.  Per step, for every chunk:

* K and V of the chunk are copied from host memory into one of two device
  buffers on a copy stream, one chunk ahead of the compute;
* ShortConv2D of its views, then its gradient sum (``ttt_grad``, or
  ``ttt_grad_dot`` for the pages' inner loop) into the chunk's row of a
  per-step gradient buffer;

and then one update from all rows, added in chunk order (``ttt_sgd_update``
or ``ttt_muon_update``), so the result does not depend on the chunking's
timing.  With one chunk this is ``ttt_write`` (``ttt_write_muon``).  V' is
recomputed each step: the conv costs far less than the copy it would save.
The read streams Q the same way and copies each chunk of O back.  Device
memory holds two chunks of K, V, V' (and Q, O), theta and chunks x theta of
gradient rows.

This module holds only the control flow and the copies; the arithmetic runs
in the library's kernels (``sharded.cuda_ops``).
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch

from . import sharded, ttt


def view_chunks(n_views: int, chunk_views: int) -> List[Tuple[int, int]]:
    """Contiguous ranges of whole views, chunk_views each (the last may be shorter)."""
    if chunk_views < 1:
        raise ValueError("chunk_views must be >= 1")
    return [(a, min(a + chunk_views, n_views)) for a in range(0, n_views, chunk_views)]


class _Stager:
    """Two device buffers per host tensor, filled on a copy stream one chunk ahead."""

    def __init__(self, hosts, rows_max: int, device):
        self.hosts = hosts
        self.device = torch.device(device)
        self.cuda = self.device.type == "cuda"
        self.bufs = [[torch.empty((rows_max,) + tuple(h.shape[1:]), dtype=h.dtype, device=self.device)
                      for h in hosts] for _ in range(2)]
        self.copy_stream = torch.cuda.Stream(self.device) if self.cuda else None
        self.copied = [torch.cuda.Event() if self.cuda else None for _ in range(2)]
        self.freed = [torch.cuda.Event() if self.cuda else None for _ in range(2)]
        self.used = [False, False]

    def issue(self, slot: int, r0: int, r1: int) -> None:
        """Start copying host rows [r0, r1) into buffer `slot`."""
        if not self.cuda:
            for buf, h in zip(self.bufs[slot], self.hosts):
                buf[:r1 - r0].copy_(h[r0:r1])
            return
        with torch.cuda.stream(self.copy_stream):
            if self.used[slot]:
                self.copy_stream.wait_event(self.freed[slot])   # the compute is done with it
            for buf, h in zip(self.bufs[slot], self.hosts):
                buf[:r1 - r0].copy_(h[r0:r1], non_blocking=True)
            self.copied[slot].record(self.copy_stream)
        self.used[slot] = True

    def take(self, slot: int, rows: int):
        """The buffers of `slot` (first `rows` rows), once their copy has landed."""
        if self.cuda:
            torch.cuda.current_stream(self.device).wait_event(self.copied[slot])
        return [buf[:rows] for buf in self.bufs[slot]]

    def release(self, slot: int) -> None:
        if self.cuda:
            self.freed[slot].record(torch.cuda.current_stream(self.device))


def write_streamed(K, V, conv_w, theta0, lr: float, steps: int, cfg, chunk_views: int,
                   inner: str = "sgd", ops: Optional[sharded.ShardOps] = None) -> torch.Tensor:
    """theta* of the collection `cfg` whose K, V ([n, heads, d], pinned host
    memory for overlap) stay on the host; conv_w and theta0 are on the device."""
    if steps < 0:
        raise ValueError("steps must be >= 0")
    device = theta0.device
    T = cfg.tokens_per_view
    chunks = view_chunks(cfg.n_views, chunk_views)
    ops = ops or sharded.cuda_ops(cfg.with_views(min(chunk_views, cfg.n_views)), inner)
    if steps == 0:
        return theta0.clone()
    scale = ops.step_size(lr, cfg.n)
    stager = _Stager([K, V], min(chunk_views, cfg.n_views) * T, device)
    grads = torch.empty((len(chunks), theta0.numel()), dtype=theta0.dtype, device=device)
    seq = [(s, i) for s in range(steps) for i in range(len(chunks))]
    a0, b0 = chunks[0]
    stager.issue(0, a0 * T, b0 * T)
    theta = theta0
    for k, (s, i) in enumerate(seq):
        if k + 1 < len(seq):
            a1, b1 = chunks[seq[k + 1][1]]
            stager.issue((k + 1) % 2, a1 * T, b1 * T)
        a, b = chunks[i]
        loc = cfg.with_views(b - a)
        Kc, Vc = stager.take(k % 2, (b - a) * T)
        Vp = ops.conv(Vc, conv_w, loc)
        ops.grad(Kc, Vp, theta, loc, out=grads[i])
        stager.release(k % 2)
        if i == len(chunks) - 1:
            theta = ops.update(theta, grads, scale, cfg)
    return theta


def read_streamed(Q, theta, cfg, chunk_views: int, O=None, ops: Optional[sharded.ShardOps] = None) -> torch.Tensor:
    """O = T_theta*(Q) for host-resident Q, chunk by chunk; O is returned in
    host memory (pinned if Q is)."""
    device = theta.device
    T = cfg.tokens_per_view
    chunks = view_chunks(cfg.n_views, chunk_views)
    rows_max = min(chunk_views, cfg.n_views) * T
    if ops is None:
        ws = ttt.make_workspace(cfg.with_views(min(chunk_views, cfg.n_views)), ttt.OP_READ)
        read = lambda q, th, dm, out: ttt.read(q, th, dm, O=out, workspace=ws)   # noqa: E731
    else:
        read = lambda q, th, dm, out: out.copy_(ops.read(q, th, dm))   # noqa: E731
    if O is None:
        O = torch.empty_like(Q, pin_memory=Q.is_pinned())
    stager = _Stager([Q], rows_max, device)
    # O of a chunk goes back on the compute stream, so the read two chunks
    # later (which reuses the buffer) is ordered after that copy
    outs = [torch.empty((rows_max,) + tuple(Q.shape[1:]), dtype=Q.dtype, device=device) for _ in range(2)]
    stager.issue(0, chunks[0][0] * T, chunks[0][1] * T)
    for i, (a, b) in enumerate(chunks):
        if i + 1 < len(chunks):
            stager.issue((i + 1) % 2, chunks[i + 1][0] * T, chunks[i + 1][1] * T)
        rows = (b - a) * T
        (Qc,) = stager.take(i % 2, rows)
        out = outs[i % 2][:rows]
        read(Qc, theta, cfg.with_views(b - a), out)
        stager.release(i % 2)
        O[a * T:b * T].copy_(out, non_blocking=stager.cuda)
    if stager.cuda:
        torch.cuda.current_stream(device).synchronize()
    return O
