"""Seeded synthetic inputs for the W4A8 routed-expert MoE layer.

This module is the one place shared by the CUDA path's tests/benchmark and the
CPU oracle.  It draws random numbers and nothing else: no quantisation, no
routing, no GEMM.  Every tensor it returns is a plain input of the layer:

* ``hidden``  bf16 ``[T, H]``  token activations, ~N(0, 1), optionally with a
  seeded 1% of channels multiplied by 20 before the bf16 cast (activation
  outliers);
* ``logits``  f32  ``[T, E]``  router logits, ~N(0, 1) plus an optional
  per-expert Zipf bias ``-s * ln(rank_e)`` (``rank_e`` a seeded permutation of
  1..E) and optionally a seeded set of experts forced to ``-inf``;
* per expert ``e``: ``w13`` bf16 ``[2I, H]`` (gate rows ``[0, I)``, up rows
  ``[I, 2I)``) and ``w2`` bf16 ``[H, I]``, ~N(0, 0.02).

The shapes follow the pages' model: 256 routed experts per MoE layer and
``moe_intermediate_size`` 2048 (GLM-5.3 W4AFP8 blog "From 755GB to 395GB",
section "what was quantised"; GLM-5.3-W4A8 model card, limitations).  Hidden
size 6144 and top-8 are the workload definitions used throughout this repo.

Generation runs on any torch device.  CPU and CUDA generators give different
streams for the same seed, so a caller that needs identical inputs on both
sides generates once and copies (small cases: generate on CPU; full-size
cases: generate on the GPU and copy the needed parts to the host).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch

__all__ = ["MoEConfig", "CONFIGS", "config_by_name", "gen_hidden", "gen_logits",
           "gen_expert_weights", "gen_routing_bias", "outlier_channels",
           "forced_empty_experts"]


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int            # tokens
    H: int            # hidden size (K of the gate/up GEMM, N of the down GEMM)
    I: int            # per-expert intermediate size
    E: int            # routed experts
    k: int            # experts per token
    seed: int
    zipf_s: float = 0.0          # 0 = uniform routing logits
    outlier_frac: float = 0.0    # fraction of hidden channels scaled by outlier_gain
    outlier_gain: float = 20.0
    forced_empty: int = 0        # experts whose logits are set to -inf
    weight_std: float = 0.02

    @property
    def A(self) -> int:
        """Number of (token, slot) assignments."""
        return self.T * self.k

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


# The five workloads.  Index 0 is small enough for the oracle to finish the
# whole layer in seconds; index 1 (decode, 64 tokens) is the benchmark's
# default workload.
CONFIGS = [
    MoEConfig("tiny_t16_h512_i256_e8_k2", T=16, H=512, I=256, E=8, k=2, seed=1000),
    MoEConfig("decode_t64_h6144_i2048_e256_k8", T=64, H=6144, I=2048, E=256, k=8, seed=1001),
    MoEConfig("decode_t256_zipf_h6144_i2048_e256_k8", T=256, H=6144, I=2048, E=256, k=8,
              seed=1002, zipf_s=1.1),
    MoEConfig("prefill_t16384_outlier_h6144_i2048_e256_k8", T=16384, H=6144, I=2048, E=256, k=8,
              seed=1003, outlier_frac=0.01),
    MoEConfig("prefill_t65536_zipf_empty16_h6144_i2048_e256_k8", T=65536, H=6144, I=2048, E=256,
              k=8, seed=1004, zipf_s=1.1, forced_empty=16),
]


def config_by_name(name: str) -> MoEConfig:
    for c in CONFIGS:
        if c.name == name:
            return c
    raise KeyError(name)


def _cpu_gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_channels(cfg: MoEConfig) -> torch.Tensor:
    """Seeded channel indices (int64, sorted) that carry activation outliers."""
    n = int(round(cfg.outlier_frac * cfg.H))
    if n == 0:
        return torch.zeros(0, dtype=torch.int64)
    perm = torch.randperm(cfg.H, generator=_cpu_gen(cfg.seed * 31 + 3))
    return perm[:n].sort().values


def forced_empty_experts(cfg: MoEConfig) -> torch.Tensor:
    """Seeded expert ids (int64, sorted) whose logits are -inf."""
    if cfg.forced_empty == 0:
        return torch.zeros(0, dtype=torch.int64)
    perm = torch.randperm(cfg.E, generator=_cpu_gen(cfg.seed * 31 + 5))
    return perm[:cfg.forced_empty].sort().values


def gen_routing_bias(cfg: MoEConfig) -> torch.Tensor:
    """Per-expert logit bias (f32 [E]) on the CPU: ``-s*ln(rank)`` or zeros."""
    if cfg.zipf_s == 0.0:
        return torch.zeros(cfg.E, dtype=torch.float32)
    rank = torch.randperm(cfg.E, generator=_cpu_gen(cfg.seed * 31 + 4)).to(torch.float64) + 1.0
    return (-cfg.zipf_s * torch.log(rank)).to(torch.float32)


def gen_hidden(cfg: MoEConfig, device="cpu", T: Optional[int] = None) -> torch.Tensor:
    """bf16 [T, H] hidden states."""
    T = cfg.T if T is None else T
    x = torch.randn(T, cfg.H, generator=_gen(cfg.seed * 31 + 1, device), device=device,
                    dtype=torch.float32)
    ch = outlier_channels(cfg)
    if ch.numel():
        x[:, ch.to(device)] *= cfg.outlier_gain
    return x.to(torch.bfloat16)


def gen_logits(cfg: MoEConfig, device="cpu", T: Optional[int] = None) -> torch.Tensor:
    """f32 [T, E] router logits."""
    T = cfg.T if T is None else T
    l = torch.randn(T, cfg.E, generator=_gen(cfg.seed * 31 + 2, device), device=device,
                    dtype=torch.float32)
    l += gen_routing_bias(cfg).to(device)[None, :]
    fe = forced_empty_experts(cfg)
    if fe.numel():
        l[:, fe.to(device)] = -math.inf
    return l


def gen_expert_weights(cfg: MoEConfig, e: int, device="cpu"):
    """(w13 bf16 [2I, H], w2 bf16 [H, I]) for expert ``e``."""
    g = _gen(cfg.seed * 1000003 + 2 * e + 11, device)
    w13 = (torch.randn(2 * cfg.I, cfg.H, generator=g, device=device, dtype=torch.float32)
           * cfg.weight_std).to(torch.bfloat16)
    w2 = (torch.randn(cfg.H, cfg.I, generator=g, device=device, dtype=torch.float32)
          * cfg.weight_std).to(torch.bfloat16)
    return w13, w2


def gen_shared_weights(cfg: MoEConfig, device="cpu"):
    """(w13 bf16 [2I, H], w2 bf16 [H, I]) of the shared expert, which has the
    routed experts' shape (its own seed stream)."""
    g = _gen(cfg.seed * 1000003 + 7, device)
    w13 = (torch.randn(2 * cfg.I, cfg.H, generator=g, device=device, dtype=torch.float32)
           * cfg.weight_std).to(torch.bfloat16)
    w2 = (torch.randn(cfg.H, cfg.I, generator=g, device=device, dtype=torch.float32)
          * cfg.weight_std).to(torch.bfloat16)
    return w13, w2
