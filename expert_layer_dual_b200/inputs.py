"""Seeded synthetic inputs, shared by the CUDA path's tests, the benchmark and
the oracle's callers.

This module only draws random numbers in the shapes and distributions of the
workloads; it holds none of the layer's arithmetic (no weight split, no
quantisation, no routing).  Every tensor has its own generator, seeded from
the workload seed and a fixed per-tensor index, so any tensor can be redrawn
alone and the order of draws never matters.

Recipe (one row per tensor, index in brackets):
  x [0]          N(0, 1) rounded to bf16, [T, d]
  router_w [1]   N(0, 1/d) float32, [E, d]
  w_gu [2]       N(0, 1/d) bf16, [E, 2I, d]   (gate rows first, then up rows)
  w_d [3]        N(0, 1/I) bf16, [E, d, I]
  ws_gu [4]      N(0, 1/d) bf16, [2Is, d]     (shared expert, when Is > 0)
  ws_d [5]       N(0, 1/Is) bf16, [d, Is]
  router_bias [6] skewed workload only: b_e = 0.38 * ln p_r(e), p_r ~ r^-1.2
                 over ranks r = 1..E given by a seeded permutation; the 8
                 lowest-ranked experts get -1e4 so they never receive tokens.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from .configs import MoEConfig


def _gen(seed: int, idx: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + idx)
    return g


def _normal(shape, std: float, seed: int, idx: int, device, dtype) -> torch.Tensor:
    g = _gen(seed, idx, device)
    out = torch.empty(shape, dtype=dtype, device=device)
    if len(shape) == 3 and shape[0] > 1:
        # one expert at a time keeps the float32 temporary small on the device
        for e in range(shape[0]):
            out[e] = (torch.randn(shape[1:], generator=g, device=device) * std).to(dtype)
    else:
        out.copy_((torch.randn(shape, generator=g, device=device) * std).to(dtype))
    return out


def zipf_bias(E: int, seed: int, s: float = 1.2, alpha: float = 0.38,
              n_masked: int = 8) -> torch.Tensor:
    g = _gen(seed, 6, "cpu")
    rank = torch.randperm(E, generator=g).to(torch.float64) + 1.0
    p = rank ** (-s)
    p = p / p.sum()
    b = alpha * torch.log(p)
    b[rank > E - n_masked] = -1.0e4
    return b.to(torch.float32)


def make_layer(cfg: MoEConfig, device="cpu", T: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All inputs of one layer forward, drawn on `device` (CPU and CUDA
    generators give different streams for the same seed)."""
    T = cfg.T if T is None else T
    s, d, E, I, Is = cfg.seed, cfg.d, cfg.E, cfg.I, cfg.Is
    bf = torch.bfloat16
    out = {
        "x": _normal((T, d), 1.0, s, 0, device, bf),
        "router_w": _normal((E, d), d ** -0.5, s, 1, device, torch.float32),
        "w_gu": _normal((E, 2 * I, d), d ** -0.5, s, 2, device, bf),
        "w_d": _normal((E, d, I), I ** -0.5, s, 3, device, bf),
        "ws_gu": None,
        "ws_d": None,
        "router_bias": None,
    }
    if Is > 0:
        out["ws_gu"] = _normal((2 * Is, d), d ** -0.5, s, 4, device, bf)
        out["ws_d"] = _normal((d, Is), Is ** -0.5, s, 5, device, bf)
    if cfg.zipf_bias:
        out["router_bias"] = zipf_bias(E, s).to(device)
    return out


def random_logits(T: int, E: int, seed: int, ties: bool = True) -> torch.Tensor:
    """float32 [T, E] ~ N(0, 1); with `ties`, every fourth row repeats some of
    its values exactly so equal logits occur inside and at the top-k edge."""
    g = _gen(seed, 10, "cpu")
    l = torch.randn((T, E), generator=g)
    if ties and E >= 4:
        for t in range(0, T, 4):
            j = torch.randperm(E, generator=g)[: max(2, E // 4)]
            l[t, j[1:]] = float(l[t, j[0]])
    return l


def random_ids(T: int, E: int, k: int, seed: int) -> torch.Tensor:
    """int32 [T, k]: k distinct experts per token, uniformly at random."""
    g = _gen(seed, 11, "cpu")
    keys = torch.rand((T, E), generator=g)
    return torch.argsort(keys, dim=1)[:, :k].to(torch.int32).contiguous()


def random_bf16(shape, seed: int, idx: int, std: float = 1.0) -> torch.Tensor:
    return _normal(tuple(shape), std, seed, 20 + idx, "cpu", torch.bfloat16)


def random_weights(T: int, k: int, seed: int) -> torch.Tensor:
    """float32 [T, k] positive weights summing to 1 per token."""
    g = _gen(seed, 12, "cpu")
    w = torch.rand((T, k), generator=g) + 0.05
    return (w / w.sum(dim=1, keepdim=True)).to(torch.float32)
