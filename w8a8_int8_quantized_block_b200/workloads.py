"""Seeded synthetic inputs for the ConvRot W8A8 linear.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic (no rotation, quantisation or GEMM), so both the CUDA
path and the CPU oracle can take their inputs from it.

The pages' workloads are real diffusion-transformer activations and trained
weights, which are not available; these distributions stand in for them.
Shapes follow the pages: hidden size K = 5376 and T = 38656 tokens at 768p
("mmh3turbo" METADATA, "Why it is fast, and where it is not"), head_dim 128.

Draw order for a linear: X ~ N(0,1) f32 [M, K] -> outlier channel indices
(randperm(K)[:n_out]) -> per-token factors exp(U[ln lo, ln hi]) [M] (when
enabled) -> W ~ N(0, w_std) f32 [N, K] -> bias ~ N(0, bias_std) f32 [N].
Outlier channels are multiplied by ``out_scale`` and rows by their factor in
f32, then X is rounded to bf16 (nearest-even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LinearSpec:
    name: str
    M: int
    K: int
    N: int
    block: int = 128
    seed: int = 0
    n_out: int = 0           # outlier channels
    out_scale: float = 1.0   # factor applied to the outlier channels
    token_scale: bool = False  # per-token factor log-uniform on [0.1, 10]
    w_std: float = 0.02
    bias_std: float = 0.01   # 0 -> zero bias

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K


@dataclass(frozen=True)
class MlpSpec:
    name: str
    M: int
    K: int      # model width
    H: int      # hidden width (4x)
    block: int = 128
    seed: int = 3
    n_out: int = 54
    out_scale: float = 10.0
    token_scale: bool = True
    w_std: float = 0.02

    @property
    def ops(self) -> int:
        return 2 * self.M * self.H * self.K * 2


@dataclass(frozen=True)
class BmmSpec:
    name: str
    batch: int
    M: int
    N: int
    K: int
    seed: int = 4

    @property
    def ops(self) -> int:
        return 2 * self.batch * self.M * self.N * self.K


def _one_percent(K: int) -> int:
    return int(round(0.01 * K))


# The five workloads: a tiny parity case, one projection at 4096 tokens, the
# full 768p projection (the throughput workload), a 4x MLP pair and a batched
# skinny-K GEMM shaped like attention's Q K^T.
TINY = LinearSpec("tiny_m256_k512_n512", 256, 512, 512, seed=0, n_out=4, out_scale=20.0)
PROJ_4K = LinearSpec("proj_m4096_k5376_n5376", 4096, 5376, 5376, seed=1,
                     n_out=_one_percent(5376), out_scale=10.0)
PROJ_768P = LinearSpec("proj_m38656_k5376_n5376", 38656, 5376, 5376, seed=2,
                       n_out=_one_percent(5376), out_scale=10.0, token_scale=True)
MLP_768P = MlpSpec("mlp_m38656_k5376_h21504", 38656, 5376, 21504, seed=3,
                   n_out=_one_percent(5376), out_scale=10.0, token_scale=True)
QK_BMM = BmmSpec("qk_b42_m8192_n8192_k128", 42, 8192, 8192, 128, seed=4)

ALL = {s.name: s for s in (TINY, PROJ_4K, PROJ_768P, MLP_768P, QK_BMM)}


def _activations(g: torch.Generator, M: int, K: int, n_out: int, out_scale: float,
                 token_scale: bool) -> torch.Tensor:
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if n_out > 0:
        idx = torch.randperm(K, generator=g)[:n_out]
        x[:, idx] *= out_scale
    if token_scale:
        lo, hi = math.log(0.1), math.log(10.0)
        f = torch.exp(torch.rand(M, generator=g, dtype=torch.float32) * (hi - lo) + lo)
        x *= f[:, None]
    return x.to(torch.bfloat16)


def linear_inputs(spec: LinearSpec, M: int | None = None):
    """(x bf16 [M, K], w f32 [N, K], bias f32 [N] or None) on the CPU.

    ``M`` overrides the token count (rows are drawn from the same stream, so a
    smaller M is a prefix only when no per-token factor is drawn)."""
    g = torch.Generator().manual_seed(spec.seed)
    m = spec.M if M is None else M
    x = _activations(g, m, spec.K, spec.n_out, spec.out_scale, spec.token_scale)
    w = torch.randn(spec.N, spec.K, generator=g, dtype=torch.float32) * spec.w_std
    bias = None
    if spec.bias_std > 0:
        bias = torch.randn(spec.N, generator=g, dtype=torch.float32) * spec.bias_std
    return x, w, bias


def mlp_inputs(spec: MlpSpec, M: int | None = None):
    """(x bf16 [M, K], w_up f32 [H, K], w_down f32 [K, H]) on the CPU; biases are zero."""
    g = torch.Generator().manual_seed(spec.seed)
    m = spec.M if M is None else M
    x = _activations(g, m, spec.K, spec.n_out, spec.out_scale, spec.token_scale)
    w_up = torch.randn(spec.H, spec.K, generator=g, dtype=torch.float32) * spec.w_std
    w_down = torch.randn(spec.K, spec.H, generator=g, dtype=torch.float32) * spec.w_std
    return x, w_up, w_down


def bmm_inputs(spec: BmmSpec, M: int | None = None, N: int | None = None):
    """(q bf16 [B, M, K], k bf16 [B, N, K]) ~ N(0, 1) on the CPU."""
    g = torch.Generator().manual_seed(spec.seed)
    m = spec.M if M is None else M
    n = spec.N if N is None else N
    q = torch.randn(spec.batch, m, spec.K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(spec.batch, n, spec.K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k


def custom_linear(M: int, K: int, N: int, seed: int, block: int = 128, n_out: int = 0,
                  out_scale: float = 10.0, token_scale: bool = False, bias_std: float = 0.01):
    """Arbitrary-shape linear inputs for edge-case tests."""
    spec = LinearSpec(f"custom_m{M}_k{K}_n{N}", M, K, N, block=block, seed=seed, n_out=n_out,
                      out_scale=out_scale, token_scale=token_scale, bias_std=bias_std)
    return spec, linear_inputs(spec)
