"""Seeded synthetic inputs for the frozen-NF4 QLoRA linear layer.

This module holds workload shapes and random-number recipes only: it contains
none of the method's arithmetic (no quantisation, no dequantisation, no matmul).
Both the CPU oracle tests and the GPU path draw their inputs from here, so the
two sides always see the same bits.

Recipe (one torch CPU generator per tensor, seed = 1000*config_index + tensor_id):
  tensor_id 0  W   fp32 [N, K]  ~ N(0, w_std); optionally 0.1% of entries x10
  tensor_id 1  X   bf16 [M, K]  ~ N(0, 1)
  tensor_id 2  A   bf16 [r, K]  ~ N(0, 1) * sqrt(2 / r)
  tensor_id 3  B   bf16 [N, r]  ~ N(0, b_std)
  tensor_id 4  dY  bf16 [M, N]  ~ N(0, 1)
  tensor_id 5  outlier positions: randperm(N*K)[: N*K // 1000]
bf16 tensors are drawn in fp32 and cast with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math

import torch

W_ID, X_ID, A_ID, B_ID, DY_ID, OUTLIER_ID = 0, 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class Linear:
    """One QLoRA linear layer workload: W is [N, K] (out x in), M tokens."""
    name: str
    config_index: int
    N: int
    K: int
    M: int
    r: int
    alpha: float
    w_std: float = 0.02
    b_std: float = 0.01
    outliers: bool = False
    layer_id: int = 0   # distinguishes several linears inside one config

    @property
    def scale(self) -> float:
        return self.alpha / self.r

    def seed(self, tensor_id: int) -> int:
        return 1000 * self.config_index + 100 * self.layer_id + tensor_id

    def flops_fwd_bwd(self) -> int:
        """Algorithmic FLOPs of fwd + bwd: 4MNK (Y and dX) + 6Mr(N+K) (LoRA)."""
        M, N, K, r = self.M, self.N, self.K, self.r
        return 4 * M * N * K + 6 * M * r * (N + K)


# The five workloads (tiny, LLaMA-7B attention, LLaMA-7B MLP, 65B-scale shapes,
# small-batch sweep). Index = position in the workload list; it seeds the RNG.
TINY = Linear("tiny_512x512_m64_r8", 0, N=512, K=512, M=64, r=8, alpha=16.0)
ATTN7B = Linear("llama7b_attn_4096x4096_m4096_r16", 1, N=4096, K=4096, M=4096, r=16,
                alpha=32.0, outliers=True)
MLP7B = [
    Linear("llama7b_mlp_gate_11008x4096_m4096_r64", 2, N=11008, K=4096, M=4096, r=64,
           alpha=16.0, layer_id=0),
    Linear("llama7b_mlp_up_11008x4096_m4096_r64", 2, N=11008, K=4096, M=4096, r=64,
           alpha=16.0, layer_id=1),
    Linear("llama7b_mlp_down_4096x11008_m4096_r64", 2, N=4096, K=11008, M=4096, r=64,
           alpha=16.0, layer_id=2),
]
L65B = [
    Linear("65b_attn_8192x8192_m2048_r64", 3, N=8192, K=8192, M=2048, r=64, alpha=16.0,
           w_std=0.015, layer_id=0),
    Linear("65b_mlp_up_22016x8192_m2048_r64", 3, N=22016, K=8192, M=2048, r=64, alpha=16.0,
           w_std=0.015, layer_id=1),
    Linear("65b_mlp_down_8192x22016_m2048_r64", 3, N=8192, K=22016, M=2048, r=64,
           alpha=16.0, w_std=0.015, layer_id=2),
]
SWEEP = [
    Linear(f"sweep_{N}x{K}_m{M}_r16", 4, N=N, K=K, M=M, r=16, alpha=32.0,
           layer_id=li * 4 + mi)
    for li, (N, K) in enumerate([(8192, 8192), (22016, 8192)])
    for mi, M in enumerate([1, 4, 16, 64])
]

ALL = [TINY, ATTN7B, *MLP7B, *L65B, *SWEEP]


def by_name(name: str) -> Linear:
    for cfg in ALL:
        if cfg.name == name:
            return cfg
    raise KeyError(name)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def weight(cfg: Linear) -> torch.Tensor:
    """fp32 [N, K] weight ~ N(0, w_std), with 0.1% outliers scaled x10 if asked."""
    w = torch.randn(cfg.N, cfg.K, generator=_gen(cfg.seed(W_ID)), dtype=torch.float32)
    w.mul_(cfg.w_std)
    if cfg.outliers:
        numel = cfg.N * cfg.K
        idx = torch.randperm(numel, generator=_gen(cfg.seed(OUTLIER_ID)))[: numel // 1000]
        flat = w.view(-1)
        flat[idx] = flat[idx] * 10.0
    return w


def _bf16(shape, seed: int, std: float) -> torch.Tensor:
    t = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def activations(cfg: Linear, M: int | None = None) -> torch.Tensor:
    """bf16 [M, K] layer input ~ N(0, 1)."""
    return _bf16((cfg.M if M is None else M, cfg.K), cfg.seed(X_ID), 1.0)


def lora_a(cfg: Linear) -> torch.Tensor:
    """bf16 [r, K] down-projection ~ N(0, 1) * sqrt(2 / r)."""
    return _bf16((cfg.r, cfg.K), cfg.seed(A_ID), math.sqrt(2.0 / cfg.r))


def lora_b(cfg: Linear) -> torch.Tensor:
    """bf16 [N, r] up-projection ~ N(0, b_std)."""
    return _bf16((cfg.N, cfg.r), cfg.seed(B_ID), cfg.b_std)


def grad_output(cfg: Linear, M: int | None = None) -> torch.Tensor:
    """bf16 [M, N] upstream gradient ~ N(0, 1)."""
    return _bf16((cfg.M if M is None else M, cfg.N), cfg.seed(DY_ID), 1.0)


def custom(N: int, K: int, M: int, r: int, alpha: float = 16.0, seed_base: int = 90,
           w_std: float = 0.02, b_std: float = 0.01, outliers: bool = False) -> Linear:
    """A workload of arbitrary shape (ragged tails, edge cases) with its own seeds."""
    return Linear(f"custom_{N}x{K}_m{M}_r{r}", seed_base, N=N, K=K, M=M, r=r, alpha=alpha,
                  w_std=w_std, b_std=b_std, outliers=outliers)
