"""GPU parity of the SVDQuant-style NVFP4 linear (svdq_w4a4, NVFP4 variant, of the
Nunchaku pages): the 4-bit residual GEMM plus a 16-bit low-rank branch.

Tolerance: the usual per-element bound of the NVFP4 linear (1e-3 * T + one bf16 ulp)
plus 2^-8 * T_lr, T_lr = sum_j |D[m,j] up[n,j]|: the branch is 16-bit (its
activations are rounded to bf16 once, after division by alpha, so each term carries
at most about 2^-9 relative error; the factor 2 is margin).
"""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import Nvfp4Case, check_linear, scalar_dev, to_dev

pytestmark = pytest.mark.gpu

LR_TOL = 2.0 ** -8


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def lowrank_operands(K, N, r, seed):
    g = torch.Generator().manual_seed(seed)
    down = (torch.randn(r, K, generator=g) * 0.02).to(torch.bfloat16)
    up = (torch.randn(N, r, generator=g) * 0.05).to(torch.bfloat16)
    return down, up


@pytest.mark.parametrize("M,K,N,r", [
    (600, 512, 520, 32),    # CTA pairs, ragged M and N
    (130, 1024, 1536, 32),  # single-CTA tiles
    (512, 768, 1000, 64),   # the largest rank: all 4 bf16 MMAs
    (256, 256, 384, 8),     # the smallest rank
])
def test_gemm_lowrank_with_host_branch_activations(M, K, N, r):
    c = Nvfp4Case(M, K, N, seed=M + r, bias=True)
    d = c.device_args()
    down, up = lowrank_operands(K, N, r, seed=r)
    D = oracle.lowrank_down(c.x, down)                     # exact, fp64
    alpha = float(np.float32(c.gx) * np.float32(c.gw))     # as the kernel forms it (fp32)
    lr_act = to_dev(_bf16(D / alpha))
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws)
    y = q.nvfp4_linear_gemm_lowrank(M, d["w"], d["weight_scale_2"], d["input_scale"], ws,
                                    lr_act, to_dev(up), bias=d["bias"])
    torch.cuda.synchronize()
    xq, xs = c.oracle_act()
    _, y64, T, Tlr = oracle.svdq_nvfp4_linear(xq, xs, c.wq, c.ws, c.gx, c.gw, D, up, c.bias)
    check_linear(y, y64, T, f"svdq gemm {M}x{K}x{N} r{r}", extra=LR_TOL * Tlr)
    # the branch matters: without it the output is off by far more than the tolerance
    _, y64_main, _ = oracle.nvfp4_linear(xq, xs, c.wq, c.ws, c.gx, c.gw, c.bias)
    assert np.abs(y64 - y64_main).max() > 10 * (LR_TOL * Tlr).max()


def test_gemm_lowrank_rejects_bad_rank():
    c = Nvfp4Case(128, 256, 256, seed=1)
    d = c.device_args()
    ws = torch.empty(q.nvfp4_linear_workspace_size(128, 256, 256), dtype=torch.uint8,
                     device="cuda")
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws)
    for r in (4, 12, 72):
        act = torch.zeros(128, r, dtype=torch.bfloat16, device="cuda")
        up = torch.zeros(256, r, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(q.QLinearError):
            q.nvfp4_linear_gemm_lowrank(128, d["w"], d["weight_scale_2"], d["input_scale"], ws,
                                        act, up)
