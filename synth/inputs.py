"""Seeded draws of the layer's inputs and weights.

Every tensor is drawn from its own ``torch.Generator`` whose seed is a stable
hash of (workload name, base seed, tensor tag, expert index), so any single
expert's weights can be regenerated on demand without drawing the others.  The
draws are device-specific: a tensor drawn on ``cuda`` differs from the one drawn
on ``cpu`` for the same seed, so a consumer that needs the host copy of a
device-drawn tensor copies it back.

Distributions (std, not variance):

* x ~ N(0, 1);
* W_r ~ N(0, router_std) (router_std <= 0 means 1/sqrt(H)); on skewed workloads
  the rows of ``skew_experts`` seeded-random experts are multiplied by
  ``skew_factor``;
* bias ~ U(-bias_range, bias_range), fp32;
* W1, W3 [I, H] ~ N(0, 1/sqrt(H)); W2 [H, I] ~ N(0, 1/sqrt(I)); the shared
  expert uses the same rule with I_shared;
* dy (the gradient of a loss with respect to the layer's output, the
  backward's input) ~ N(0, 1).

All matrices are returned in bf16 (bias in fp32), row-major.
"""

import zlib

import torch

from .configs import MoEShape


def _seed(cfg: MoEShape, tag: str, index: int = 0) -> int:
    key = f"{cfg.name}/{cfg.seed}/{tag}/{index}".encode()
    return zlib.crc32(key) & 0x7FFFFFFF


def _gen(cfg: MoEShape, tag: str, index: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(cfg, tag, index))
    return g


def _normal(shape, std, g, device) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def gen_x(cfg: MoEShape, device="cpu", T: int = None) -> torch.Tensor:
    T = cfg.T if T is None else T
    return _normal((T, cfg.H), 1.0, _gen(cfg, "x", 0, device), device)


def gen_dy(cfg: MoEShape, device="cpu") -> torch.Tensor:
    return _normal((cfg.T, cfg.H), 1.0, _gen(cfg, "dy", 0, device), device)


def gen_router(cfg: MoEShape, device="cpu"):
    """Returns (W_r [E, H] bf16, bias [E] fp32)."""
    std = cfg.router_std if cfg.router_std > 0 else cfg.H ** -0.5
    g = _gen(cfg, "w_router", 0, device)
    w = torch.randn(cfg.E, cfg.H, generator=g, device=device, dtype=torch.float32) * std
    if cfg.skew_experts > 0:
        gs = torch.Generator(device="cpu")
        gs.manual_seed(_seed(cfg, "skew", 0))
        hot = torch.randperm(cfg.E, generator=gs)[: cfg.skew_experts]
        w[hot.to(device)] *= cfg.skew_factor
    gb = _gen(cfg, "bias", 0, device)
    bias = (torch.rand(cfg.E, generator=gb, device=device, dtype=torch.float32) * 2.0 - 1.0) * cfg.bias_range
    return w.to(torch.bfloat16), bias


def gen_expert_weights(cfg: MoEShape, e: int, device="cpu"):
    """Returns (W1 [I, H], W3 [I, H], W2 [H, I]) of routed expert ``e``, bf16."""
    H, I = cfg.H, cfg.I
    w1 = _normal((I, H), H ** -0.5, _gen(cfg, "w1", e, device), device)
    w3 = _normal((I, H), H ** -0.5, _gen(cfg, "w3", e, device), device)
    w2 = _normal((H, I), I ** -0.5, _gen(cfg, "w2", e, device), device)
    return w1, w3, w2


def gen_shared_weights(cfg: MoEShape, device="cpu"):
    """Returns (Ws1 [I_s, H], Ws3 [I_s, H], Ws2 [H, I_s]) bf16, or None."""
    if cfg.I_shared <= 0:
        return None
    H, I = cfg.H, cfg.I_shared
    w1 = _normal((I, H), H ** -0.5, _gen(cfg, "ws1", 0, device), device)
    w3 = _normal((I, H), H ** -0.5, _gen(cfg, "ws3", 0, device), device)
    w2 = _normal((H, I), I ** -0.5, _gen(cfg, "ws2", 0, device), device)
    return w1, w3, w2


def gen_all(cfg: MoEShape, device="cpu") -> dict:
    """All inputs of a workload, with routed weights stacked as [E, ...]."""
    x = gen_x(cfg, device)
    w_r, bias = gen_router(cfg, device)
    w1 = torch.empty(cfg.E, cfg.I, cfg.H, dtype=torch.bfloat16, device=device)
    w3 = torch.empty_like(w1)
    w2 = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.bfloat16, device=device)
    for e in range(cfg.E):
        a, b, c = gen_expert_weights(cfg, e, device)
        w1[e], w3[e], w2[e] = a, b, c
    out = dict(x=x, w_router=w_r, bias=bias, w1=w1, w3=w3, w2=w2)
    sh = gen_shared_weights(cfg, device)
    if sh is not None:
        out["ws1"], out["ws3"], out["ws2"] = sh
    return out
