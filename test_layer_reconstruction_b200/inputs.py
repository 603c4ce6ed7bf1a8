"""Seeded synthetic inputs for the VGG-T^3 test-time-training layer.

This module holds shapes, layouts and random draws only; none of the layer's
arithmetic lives here.  Both the float64 oracle (through the tests) and the
CUDA path take their inputs from it.

Workloads (token layout per view: ``n_special`` camera/register tokens first,
then the ``grid_h x grid_w`` patch grid in row-major order):

* VGG-T^3 paper, Sec. 3.1 "Tokenization": a 518x518 image with patch size 14
  gives a 37x37 = 1369 patch grid; camera and register tokens are appended.
* VGG-T^3 paper, Sec. 3.2 / App. A: per-head width 64 (VGGT width 1024 = 16 x 64),
  SwiGLU fast-weight MLP, 1 inner step for short collections and 2 at 1k views.

Distributions.  The workloads' own draws ("stated", the default): every
(token, head) row of K and of Q is an N(0, I_d) draw divided by its Euclidean
norm (the pages' L2 normalisation of queries and keys, Sec. 3.4 "The
LayerNorm removal"), V ~ N(0, 1) elementwise, all three independent, each then
rounded to bfloat16 (round-to-nearest-even).  Depthwise 3x3 weights ~
N(0, 1/9); fast weights Xavier-normal with std sqrt(2 / (d + h)).

A second family ("correlated") gives the tokens the structure of projections
of one token feature, as in the attention layer the TTT layer replaces: every
(token, head) row has one latent x ~ N(0, I_d), and with per-head projections
P_Q, P_K, P_V ~ N(0, 1/d) (d x d, one draw per sequence)
    K = x P_K / ||x P_K||,  Q = x P_Q / ||x P_Q||,  V = x P_V,
so V at a token is linearly predictable from K at that token.  It is an extra
parity case, selected per workload with ``LayerConfig.draws``.

Every view's rows are drawn from their own generator, seeded by a SplitMix64
mix of (seed, tensor id, view index), so any subset or permutation of views
reproduces the same values.  Held-out views use the held-out seed (with the
correlated family they draw new latents and share the sequence's projections).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional, Sequence

import torch

__all__ = [
    "LayerConfig", "CONFIGS", "make_inputs", "make_surround", "pack_theta", "unpack_theta",
    "theta_numel", "bf16_round", "view_token_index",
]

_MASK64 = (1 << 64) - 1

# tensor ids of the counter-based seeding
_TID_K, _TID_Q, _TID_V, _TID_CONV, _TID_W1, _TID_W3, _TID_W2, _TID_X = range(8)
_TID_TOKENS, _TID_WQ, _TID_WK, _TID_WV, _TID_WO = range(8, 13)


def _splitmix64(x: int) -> int:
    """SplitMix64 output function (Steele, Lea, Flood, OOPSLA 2014)."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def _stream_seed(seed: int, tensor_id: int, view: int) -> int:
    s = _splitmix64(seed & _MASK64)
    s = _splitmix64(s ^ (tensor_id & _MASK64))
    s = _splitmix64(s ^ (view & _MASK64))
    return s & ((1 << 63) - 1)


def _randn(shape, seed, tensor_id, view, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(_stream_seed(seed, tensor_id, view))
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """One workload of the TTT layer.

    tokens per view = n_special + grid_h * grid_w; n = n_views * tokens per view.
    """
    name: str
    n_views: int
    grid_h: int
    grid_w: int
    n_special: int
    heads: int
    d: int
    h: int
    steps: int
    lr: float
    seed: int
    fp32_inputs: bool = False      # the tiny case draws fp32 Q/K/V
    heldout_views: int = 0         # frozen-theta read of extra views
    heldout_seed: int = 0
    draws: str = "stated"          # "stated" (independent) or "correlated"

    @property
    def tokens_per_view(self) -> int:
        return self.n_special + self.grid_h * self.grid_w

    @property
    def n(self) -> int:
        return self.n_views * self.tokens_per_view

    def with_views(self, n_views: int) -> "LayerConfig":
        return dataclasses.replace(self, n_views=n_views)

    def with_draws(self, draws: str) -> "LayerConfig":
        return dataclasses.replace(self, draws=draws)

    def flops(self) -> float:
        """Algorithmic FLOPs of conv-free layer math: (14*steps + 6) * d * h per token and head."""
        return float(14 * self.steps + 6) * self.d * self.h * self.n * self.heads

    def dims(self) -> Dict[str, int]:
        return dict(n_views=self.n_views, grid_h=self.grid_h, grid_w=self.grid_w,
                    n_special=self.n_special, heads=self.heads, d=self.d, h=self.h)


CONFIGS: Dict[str, LayerConfig] = {
    c.name: c for c in [
        # 2 views of an 8x8 grid, 1 head, d=16, h=32, fp32 draws, 1 step, lr 0.1, seed 0
        LayerConfig("tiny_2v_8x8_d16_h32", 2, 8, 8, 0, 1, 16, 32, 1, 0.1, 0, fp32_inputs=True),
        # 24 views of 37x37 + 5 special tokens (32,976 tokens), 16 heads, d=64, h=256, 1 step
        LayerConfig("views24_37x37p5_h16_d64_h256", 24, 37, 37, 5, 16, 64, 256, 1, 0.1, 1),
        # 100 views (137,400 tokens), 2 steps
        LayerConfig("views100_37x37p5_h16_d64_h256", 100, 37, 37, 5, 16, 64, 256, 2, 0.1, 2),
        # 1000 views (1,374,000 tokens), 2 steps, lr 0.05
        LayerConfig("views1000_37x37p5_h16_d64_h256", 1000, 37, 37, 5, 16, 64, 256, 2, 0.05, 3),
        # 2000 views, one fast-weight MLP d=1024, h=2048, 2 steps, lr 0.02, + 200 held-out views
        LayerConfig("views2000_37x37p5_h1_d1024_h2048", 2000, 37, 37, 5, 1, 1024, 2048, 2, 0.02, 4,
                    heldout_views=200, heldout_seed=1004),
    ]
}


def bf16_round(x: torch.Tensor) -> torch.Tensor:
    """Round to bfloat16 (round-to-nearest-even) and return float32 values."""
    return x.to(torch.bfloat16).to(torch.float32)


def view_token_index(cfg: LayerConfig, view: int, y: int, x: int) -> int:
    """Token index of patch (y, x) of a view; special tokens come first in each view."""
    return view * cfg.tokens_per_view + cfg.n_special + y * cfg.grid_w + x


def _latents(cfg, views, device, seed) -> torch.Tensor:
    """One N(0, I_d) latent per (token, head) row, drawn view by view."""
    parts = [_randn((cfg.tokens_per_view, cfg.heads, cfg.d), seed, _TID_X, v, device) for v in views]
    return torch.cat(parts, 0) if parts else torch.zeros(0, cfg.heads, cfg.d, device=device)


def _projection(cfg, tensor_id, device) -> torch.Tensor:
    """Per-head d x d projection ~ N(0, 1/d), drawn from the sequence seed."""
    return _randn((cfg.heads, cfg.d, cfg.d), cfg.seed, tensor_id, 0, device) * (1.0 / math.sqrt(cfg.d))


def _project(X, P, normalise) -> torch.Tensor:
    out = torch.empty_like(X)
    step = 1 << 16   # bounded temporaries on long sequences
    for a in range(0, X.shape[0], step):
        r = torch.einsum("thd,hde->the", X[a:a + step], P)
        if normalise:
            r = r / torch.linalg.vector_norm(r, dim=-1, keepdim=True)
        out[a:a + step] = r
    return out


def _unit_rows(cfg, views, device, seed, tensor_id) -> torch.Tensor:
    """N(0, I_d) rows divided by their norm, drawn view by view."""
    parts = []
    for v in views:
        r = _randn((cfg.tokens_per_view, cfg.heads, cfg.d), seed, tensor_id, v, device)
        parts.append(r / torch.linalg.vector_norm(r, dim=-1, keepdim=True))
    return torch.cat(parts, 0) if parts else torch.zeros(0, cfg.heads, cfg.d, device=device)


def _normal_rows(cfg, views, device, seed, tensor_id) -> torch.Tensor:
    parts = [_randn((cfg.tokens_per_view, cfg.heads, cfg.d), seed, tensor_id, v, device) for v in views]
    return torch.cat(parts, 0) if parts else torch.zeros(0, cfg.heads, cfg.d, device=device)


def make_inputs(cfg: LayerConfig, device="cpu", views: Optional[Sequence[int]] = None,
                heldout: bool = False) -> Dict[str, torch.Tensor]:
    """Draw the layer's inputs.

    Returns float32 tensors (values already rounded to bfloat16 unless
    ``cfg.fp32_inputs``): Q, K, V of shape [n, heads, d]; conv_w [heads*d, 3, 3];
    W1, W3 [heads, d, h]; W2 [heads, h, d].  ``views`` selects (and orders) the
    views drawn; ``heldout`` draws the held-out query views instead (Q only).
    """
    if cfg.draws not in ("stated", "correlated"):
        raise ValueError(f"unknown draws {cfg.draws!r}")
    if views is None:
        views = range(cfg.heldout_views if heldout else cfg.n_views)
    views = list(views)
    seed = cfg.heldout_seed if heldout else cfg.seed
    out: Dict[str, torch.Tensor] = {}
    rnd = (lambda t: t) if cfg.fp32_inputs else bf16_round
    if cfg.draws == "stated":
        out["Q"] = rnd(_unit_rows(cfg, views, device, seed, _TID_Q))
        if heldout:
            return out
        out["K"] = rnd(_unit_rows(cfg, views, device, seed, _TID_K))
        out["V"] = rnd(_normal_rows(cfg, views, device, seed, _TID_V))
    else:
        X = _latents(cfg, views, device, seed)
        out["Q"] = rnd(_project(X, _projection(cfg, _TID_Q, device), True))
        if heldout:
            return out
        out["K"] = rnd(_project(X, _projection(cfg, _TID_K, device), True))
        out["V"] = rnd(_project(X, _projection(cfg, _TID_V, device), False))
        del X
    C = cfg.heads * cfg.d
    out["conv_w"] = _randn((C, 3, 3), seed, _TID_CONV, 0, device) * (1.0 / 3.0)
    std = math.sqrt(2.0 / (cfg.d + cfg.h))
    out["W1"] = _randn((cfg.heads, cfg.d, cfg.h), seed, _TID_W1, 0, device) * std
    out["W3"] = _randn((cfg.heads, cfg.d, cfg.h), seed, _TID_W3, 0, device) * std
    out["W2"] = _randn((cfg.heads, cfg.h, cfg.d), seed, _TID_W2, 0, device) * std
    return out


def make_surround(cfg: LayerConfig, device="cpu", views: Optional[Sequence[int]] = None) -> Dict[str, torch.Tensor]:
    """Inputs of the attention layer around the TTT layer: token features
    X [n, C] ~ N(0, 1) and projections Wq, Wk, Wv, Wo [C, C] ~ N(0, 1/C)
    (C = heads * d; row-vector form x W), all rounded to bfloat16 and returned
    as float32; plus the layer's conv_w, W1, W3, W2 as in ``make_inputs``."""
    if views is None:
        views = range(cfg.n_views)
    views = list(views)
    C = cfg.heads * cfg.d
    parts = [_randn((cfg.tokens_per_view, C), cfg.seed, _TID_TOKENS, v, device) for v in views]
    out: Dict[str, torch.Tensor] = {"X": bf16_round(torch.cat(parts, 0))}
    for name, tid in (("Wq", _TID_WQ), ("Wk", _TID_WK), ("Wv", _TID_WV), ("Wo", _TID_WO)):
        out[name] = bf16_round(_randn((C, C), cfg.seed, tid, 0, device) * (1.0 / math.sqrt(C)))
    out["conv_w"] = _randn((C, 3, 3), cfg.seed, _TID_CONV, 0, device) * (1.0 / 3.0)
    std = math.sqrt(2.0 / (cfg.d + cfg.h))
    out["W1"] = _randn((cfg.heads, cfg.d, cfg.h), cfg.seed, _TID_W1, 0, device) * std
    out["W3"] = _randn((cfg.heads, cfg.d, cfg.h), cfg.seed, _TID_W3, 0, device) * std
    out["W2"] = _randn((cfg.heads, cfg.h, cfg.d), cfg.seed, _TID_W2, 0, device) * std
    return out


def theta_numel(heads: int, d: int, h: int) -> int:
    return 3 * heads * d * h


def pack_theta(W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor) -> torch.Tensor:
    """Flat float32 fast-weight buffer [W1: H*d*h | W3: H*d*h | W2: H*h*d], row-major."""
    return torch.cat([W1.reshape(-1), W3.reshape(-1), W2.reshape(-1)]).to(torch.float32).contiguous()


def unpack_theta(theta: torch.Tensor, heads: int, d: int, h: int):
    """Inverse of :func:`pack_theta`; returns (W1, W3, W2) views."""
    s = heads * d * h
    t = theta.reshape(-1)
    return (t[:s].reshape(heads, d, h), t[s:2 * s].reshape(heads, d, h),
            t[2 * s:3 * s].reshape(heads, h, d))
