"""Saving and loading the fast weights theta*.

After the write, theta* is the whole state of a TTT layer for its
collection: a few MB that can be kept and read from later (query mode) or
shipped to another device (VGG-T$^3$: Offline Feed-Forward 3D
Reconstruction at Scale, Sec. 3.4: the fast weights are transient, computed
for the current input and then discarded or frozen).  The file is a numpy
.npz holding theta in its packed FP32 layout [W1 | W3 | W2] (per head W1, W3
[d][h], W2 [h][d]) with heads, d and h, so a load can check the shape it is
given back against.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np
import torch

LAYOUT = "W1|W3|W2 per head; W1, W3 [d][h], W2 [h][d]; float32"


def save_theta(path, theta: torch.Tensor, heads: int, d: int, h: int) -> None:
    """Write theta (f32, 3*heads*d*h elements) and its shape to `path` (.npz)."""
    t = theta.detach().to("cpu", torch.float32).contiguous().reshape(-1)
    if t.numel() != 3 * heads * d * h:
        raise ValueError(f"theta has {t.numel()} elements, expected 3*{heads}*{d}*{h}")
    np.savez(path, theta=t.numpy(), heads=heads, d=d, h=h, layout=LAYOUT)


def load_theta(path, device="cpu", heads: int = None, d: int = None, h: int = None) -> Tuple[torch.Tensor, Tuple[int, int, int]]:
    """Read theta back; returns (theta on `device`, (heads, d, h)).  Any of
    heads, d, h given must match the file."""
    with np.load(path, allow_pickle=False) as z:
        if str(z["layout"]) != LAYOUT:
            raise ValueError(f"{path}: unknown theta layout {z['layout']!r}")
        shape = (int(z["heads"]), int(z["d"]), int(z["h"]))
        for name, want, got in zip(("heads", "d", "h"), (heads, d, h), shape):
            if want is not None and want != got:
                raise ValueError(f"{path}: {name} = {got}, expected {want}")
        theta = torch.from_numpy(np.array(z["theta"], dtype=np.float32))
    if theta.numel() != 3 * shape[0] * shape[1] * shape[2]:
        raise ValueError(f"{path}: theta has {theta.numel()} elements for shape {shape}")
    return theta.to(device), shape
