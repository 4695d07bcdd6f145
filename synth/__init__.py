"""Seeded synthetic workloads for the LightTransfer-Test prefill path.

This module is shared by the oracle-side tests and by the CUDA path's tests and
benchmark; it holds none of the method's arithmetic, only random numbers and the
shapes of the workloads.  The pages measure on LongBench, AIME24/25 and MathOAI
with 32B checkpoints, none of which exists here: these tensors stand in for the
per-layer Q/K/V of such a prefill.

Recipe (per configuration, layer and tensor a separate seeded torch generator):
  * Q [T, hq, d], K/V [T, hkv, d] ~ N(0, 1) in fp32.
  * Sink bias: a seeded unit vector u (shared by all heads of the layer) times
    alpha is added to every query row and to key rows 0..S-1 of every sequence.
    tiny: alpha = 4 on layers 1 and 3, 0 elsewhere; other configs alpha ~ U(0, 6).
  * Recency bias (configs that ask for it): beta ~ U(0, 3) per layer, realised as
    random Fourier features a * r(t) added to q_t and k_t (t = position inside the
    sequence), r(t)_c = sqrt(2/d) cos(w_c t + phi_c), w_c ~ Cauchy(0, 1/64),
    phi_c ~ U(0, 2 pi), a^2 = beta sqrt(d); the expected extra score
    a^2 r(i).r(j) / sqrt(d) is then beta exp(-|i-j| / 64).
  * The sum is rounded to bf16 (round to nearest even).
The bits depend on the device that draws them; tests always hand the oracle a
host copy of the very tensors the kernels read.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    layers: int
    seqlens: tuple
    hq: int
    hkv: int
    d: int
    S: int
    W: int
    n_obs: int
    budget: int
    recency: bool
    seed: int
    lazy_layers: Optional[tuple] = None   # tiny: the layers given a fixed sink bias
    tiny_alpha: float = 4.0
    online: bool = False

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens))

    def cu_seqlens(self) -> List[int]:
        cu = [0]
        for n in self.seqlens:
            cu.append(cu[-1] + int(n))
        return cu

    def causal_pairs(self) -> int:
        """Sum over sequences of N(N+1)/2 (query, key) pairs of one head."""
        return int(sum(n * (n + 1) // 2 for n in self.seqlens))


def _batched_lengths(seed: int, n: int, lo: int, hi: int) -> tuple:
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


CONFIGS = {
    "tiny": Config("tiny", 4, (256,), 2, 1, 64, 4, 32, 16, 2, False, 1001, lazy_layers=(1, 3)),
    "gqa1p2b": Config("gqa1p2b", 16, (4096,), 32, 8, 64, 4, 1020, 64, 8, False, 1002),
    "qwen32b": Config("qwen32b", 64, (32768,), 40, 8, 128, 4, 2044, 128, 32, True, 1003),
    "long128k": Config("long128k", 32, (131072,), 32, 8, 128, 4, 4092, 128, 16, True, 1004, online=True),
    "batched": Config("batched", 32, _batched_lengths(1005, 8, 8192, 32768), 32, 8, 128, 4, 1020, 64, 16, True,
                      1005),
}


def custom(name="custom", layers=1, seqlens=(256,), hq=2, hkv=1, d=64, S=4, W=32, n_obs=16, budget=0,
           recency=False, seed=7, lazy_layers=None) -> Config:
    """A configuration with arbitrary shapes (used for ragged/edge-case tests)."""
    return Config(name, layers, tuple(int(n) for n in seqlens), hq, hkv, d, S, W, n_obs, budget, recency, seed,
                  lazy_layers=lazy_layers)


def _gen(device, *key) -> torch.Generator:
    seed = 0
    for k in key:
        seed = (seed * 1000003 + int(k)) % (2**61 - 1)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def layer_params(cfg: Config, layer: int):
    """(alpha, u [d], beta) of one layer, drawn on the host."""
    g = _gen("cpu", cfg.seed, layer, 7)
    u = torch.randn(cfg.d, generator=g, dtype=torch.float64)
    u = u / u.norm()
    if cfg.lazy_layers is not None:
        alpha = cfg.tiny_alpha if layer in cfg.lazy_layers else 0.0
    else:
        alpha = float(torch.rand((), generator=g, dtype=torch.float64) * 6.0)
    beta = float(torch.rand((), generator=g, dtype=torch.float64) * 3.0) if cfg.recency else 0.0
    return alpha, u.float(), beta


def positions(cfg: Config, device="cpu") -> torch.Tensor:
    """Position of every packed token inside its own sequence (int64 [T])."""
    return torch.cat([torch.arange(n, device=device) for n in cfg.seqlens]) if cfg.seqlens else \
        torch.zeros(0, dtype=torch.int64, device=device)


def layer_inputs(cfg: Config, layer: int, device="cpu"):
    """Q [T, hq, d], K [T, hkv, d], V [T, hkv, d] bf16 tensors of one layer."""
    T, d = cfg.total_tokens, cfg.d
    Q = torch.randn((T, cfg.hq, d), generator=_gen(device, cfg.seed, layer, 1), device=device)
    K = torch.randn((T, cfg.hkv, d), generator=_gen(device, cfg.seed, layer, 2), device=device)
    V = torch.randn((T, cfg.hkv, d), generator=_gen(device, cfg.seed, layer, 3), device=device)
    alpha, u, beta = layer_params(cfg, layer)
    if alpha != 0.0:
        bias = (alpha * u).to(device)
        Q += bias
        cu = cfg.cu_seqlens()
        for b in range(cfg.batch):
            K[cu[b]: cu[b] + min(cfg.S, cfg.seqlens[b])] += bias
    if beta != 0.0:
        g = _gen("cpu", cfg.seed, layer, 9)
        w = torch.tan(math.pi * (torch.rand(d, generator=g, dtype=torch.float64) - 0.5)) / 64.0
        phi = torch.rand(d, generator=g, dtype=torch.float64) * (2.0 * math.pi)
        a = math.sqrt(beta * math.sqrt(d))
        pos = positions(cfg, device).to(torch.float64)
        r = torch.cos(pos[:, None] * w.to(device)[None, :] + phi.to(device)[None, :]) * math.sqrt(2.0 / d)
        r = (a * r).float()
        Q += r[:, None, :]
        K += r[:, None, :]
    return Q.to(torch.bfloat16), K.to(torch.bfloat16), V.to(torch.bfloat16)


def zero_queries(cfg: Config, layer: int, device="cpu"):
    """Layer inputs with every query row set to zero (uniform attention)."""
    Q, K, V = layer_inputs(cfg, layer, device)
    return torch.zeros_like(Q), K, V


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor's bits (copied to the host)."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
