"""Seeded synthetic inputs shared by the tests and the benchmark.

This module holds no arithmetic of the quantized linear layer: it only draws
random tensors. Every draw comes from one CPU ``torch.Generator`` seeded with
``seed``, in a fixed order: X, outlier channels, W, bias.

Workload recipe (diffusion-transformer linear layers; the pages describe the
layers of a DiT pipeline but publish no data, so these stand in for it):
  * X: randn(M, K) fp32; the outlier channels (2 of 256 for K=256, else 1% of K,
    rounded half-to-even) are multiplied by 20; then cast to bf16 (RN).
  * W: randn(N, K) * 0.02, cast to bf16 (RN).
  * bias: randn(N) * 0.01 in fp32 (only when requested).
"""
from dataclasses import dataclass
from typing import Optional

import torch


def outlier_count(K: int) -> int:
    if K == 256:
        return 2
    return int(round(0.01 * K))  # Python round: half to even


@dataclass
class LinearInputs:
    x: torch.Tensor            # bf16 [M, K]
    w: torch.Tensor            # bf16 [N, K]
    bias: Optional[torch.Tensor]  # fp32 [N] or None
    outlier_idx: torch.Tensor  # int64 [n_out]


def make_linear_inputs(M: int, K: int, N: int, seed: int = 0, with_bias: bool = False,
                       n_outliers: Optional[int] = None, outlier_gain: float = 20.0,
                       w_std: float = 0.02) -> LinearInputs:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    n_out = outlier_count(K) if n_outliers is None else n_outliers
    idx = torch.randperm(K, generator=g)[:n_out]
    if n_out > 0:
        x[:, idx] *= outlier_gain
    x = x.to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g, dtype=torch.float32) * w_std).to(torch.bfloat16)
    bias = None
    if with_bias:
        bias = torch.randn(N, generator=g, dtype=torch.float32) * 0.01
    return LinearInputs(x=x, w=w, bias=bias, outlier_idx=idx)


def make_activations(M: int, K: int, seed: int = 0) -> torch.Tensor:
    """Only the activation draw of ``make_linear_inputs`` (same seed, same X)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    idx = torch.randperm(K, generator=g)[:outlier_count(K)]
    if len(idx) > 0:
        x[:, idx] *= 20.0
    return x.to(torch.bfloat16)


# Named workloads (sizes of the diffusion-transformer layers this path serves).
WORKLOADS = {
    "nvfp4_tiny": dict(M=128, K=256, N=256, bias=False),
    "fp8r_4096x3072x3072": dict(M=4096, K=3072, N=3072, bias=False),
    "nvfp4_attn_proj": dict(M=4096, K=3072, N=3072, bias=True),
    "nvfp4_attn_qkv": dict(M=4096, K=3072, N=9216, bias=True),
    "nvfp4_mlp_up": dict(M=4096, K=3072, N=12288, bias=False),
    "nvfp4_mlp_down": dict(M=4096, K=12288, N=3072, bias=False),
}
