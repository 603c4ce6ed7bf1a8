"""The write of one collection sharded by views over several processes.

The TTT loss of a collection (VGG-T$^3$: Offline Feed-Forward 3D
Reconstruction at Scale, Sec. 3.4, Eq. 3) is a mean over all n tokens, and its
gradient is a sum of per-token terms (Eq. 5).  ShortConv2D never crosses
views, so the views can be split between ranks with no halo:

* each rank convolves its own views once (V' = ShortConv2D(V));
* per SGD step, each rank evaluates its gradient sum on its views
  (``ttt_grad``: d/dtheta of (1/2) sum_i ||T(k_i) - v'_i||^2), the ranks
  all-gather these sums (3 * heads * d * h floats per rank), and every rank
  applies the same step theta <- theta - lr (2/n) sum_r g_r with the sums
  added in rank order (``ttt_sgd_update``), so theta* is the same on every
  rank bit for bit, and the same from run to run;
* the read of each rank's queries is local.

With one rank this computes what ``ttt_write`` computes.  The same control
flow runs the pages' own inner loop (dot-product loss, Muon steps:
``ttt_grad_dot`` and ``ttt_muon_update``, which orthogonalises the summed
gradient), ``cuda_ops(dims, inner="muon")``; with one rank that is
``ttt_write_muon``.

The exchange is the only collective.  This module holds only the per-step
control flow; every arithmetic step runs in the library's kernels
(``cuda_ops``).  ``ShardOps`` lets the multi-process tests drive the same
control flow with other operations on CPU ranks.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Tuple

import numpy as np
import torch

from . import ttt


def step_scale(lr: float, n_total: int) -> float:
    """lr * 2 / n_total in single precision, rounded as the single-process write rounds it."""
    return float(np.float32(np.float32(lr) * np.float32(2.0)) / np.float32(n_total))


def muon_step_size(lr: float, n_total: int) -> float:
    """Muon's step is scale-free in the gradient: its size is lr itself."""
    return float(lr)


@dataclass
class ShardOps:
    """The per-rank operations of the sharded layer."""
    conv: Callable[..., torch.Tensor]     # (V, conv_w, dims) -> V'
    grad: Callable[..., torch.Tensor]     # (K, Vp, theta, dims, out=None) -> gradient sum of the tokens
    update: Callable[..., torch.Tensor]   # (theta, grads [world, numel], size, dims) -> theta'
    read: Callable[..., torch.Tensor]     # (Q, theta, dims) -> O
    step_size: Callable[[float, int], float] = step_scale   # (lr, n_total) -> the update's size argument


def cuda_ops(dims, inner: str = "sgd") -> ShardOps:
    """The library's kernels, with one write workspace reused by every gradient pass.
    inner = "sgd": mean-squared loss, SGD; "muon": dot-product loss, Muon."""
    ws = ttt.make_workspace(dims, ttt.OP_WRITE)
    if inner == "sgd":
        grad, update, size = ttt.grad, ttt.sgd_update, step_scale
    elif inner == "muon":
        grad, update, size = ttt.grad_dot, ttt.muon_update, muon_step_size
    else:
        raise ValueError(f"unknown inner loop {inner!r}")
    return ShardOps(
        conv=lambda V, conv_w, dm: ttt.shortconv2d(V, conv_w, dm),
        grad=lambda K, Vp, theta, dm, out=None: grad(K, Vp, theta, dm, out=out, workspace=ws),
        update=lambda theta, grads, s, dm: update(theta, grads, s, dm),
        read=lambda Q, theta, dm: ttt.read(Q, theta, dm),
        step_size=size,
    )


def all_gather_rows(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """Gather of a flat tensor from every rank into [world, numel], in rank order
    (torch.distributed; NCCL on GPUs)."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        flat = t.reshape(-1).contiguous()
        out = torch.empty((dist.get_world_size(group), flat.numel()), dtype=flat.dtype, device=flat.device)
        dist.all_gather_into_tensor(out, flat, group=group)
        return out

    return gather


def write_sharded(K, V, conv_w, theta0, lr: float, steps: int, dims, n_total: int,
                  gather: Callable[[torch.Tensor], torch.Tensor], ops: Optional[ShardOps] = None) -> torch.Tensor:
    """theta* of the collection whose views are split over the ranks.

    K, V hold this rank's views (``dims`` describes them); ``n_total`` is the
    collection's token count over all ranks; ``gather`` returns every rank's
    tensor stacked in rank order.  Every rank must call this with the same
    ``theta0``, ``lr``, ``steps`` and ``n_total``.  If the exchange fails (a
    rank has left, or the process group's timeout ran out), the call raises
    RuntimeError naming the step; no collective is left half-issued on the
    ranks that remain, since each step issues exactly one.
    """
    if steps < 0:
        raise ValueError("steps must be >= 0")
    ops = ops or cuda_ops(dims)
    Vp = ops.conv(V, conv_w, dims)
    scale = ops.step_size(lr, n_total)
    theta = theta0
    for step in range(steps):
        g = ops.grad(K, Vp, theta, dims)
        try:
            gathered = gather(g)
        except Exception as exc:   # a rank that left, or the process group's timeout
            raise RuntimeError(f"sharded write: the gradient exchange of step {step} failed: {exc}") from exc
        theta = ops.update(theta, gathered, scale, dims)
    return theta.clone() if steps == 0 else theta


def layer_sharded(Q, K, V, conv_w, theta0, lr: float, steps: int, dims, n_total: int,
                  gather: Callable[[torch.Tensor], torch.Tensor],
                  ops: Optional[ShardOps] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The whole layer on this rank's views: the sharded write, then the local read of Q."""
    ops = ops or cuda_ops(dims)
    theta = write_sharded(K, V, conv_w, theta0, lr, steps, dims, n_total, gather, ops)
    return theta, ops.read(Q, theta, dims)
