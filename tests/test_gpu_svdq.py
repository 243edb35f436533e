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
    (40, 768, 1000, 32),    # skinny kernel (64 rows of A per stage)
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


class SvdqCase:
    """Seeded svdq layer: outlier activations, per-column smoothing multipliers
    (1 / sqrt of the column's amax, so outlier columns are scaled down), a rank-r
    bf16 branch and an oracle-quantized 4-bit residual weight."""

    def __init__(self, M, K, N, r, seed, bias=True):
        c = Nvfp4Case(M, K, N, seed=seed, bias=bias)
        self.M, self.K, self.N, self.r = M, K, N, r
        self.x, self.wq, self.ws, self.gw, self.bias = c.x, c.wq, c.ws, c.gw, c.bias
        amax = c.x.float().abs().amax(dim=0).clamp(min=1e-3)
        self.smooth = (1.0 / amax.sqrt()).numpy().astype(np.float32)
        self.down, self.up = lowrank_operands(K, N, r, seed=seed + 1)
        self.xs = oracle.smooth_bf16(self.x, self.smooth)
        self.gx = np.float32(oracle.nvfp4_global_scale(self.xs))

    def device_args(self):
        return dict(x=to_dev(self.x), w=to_dev(self.wq), w_scale=to_dev(self.ws),
                    weight_scale_2=scalar_dev(self.gw), input_scale=scalar_dev(float(self.gx)),
                    lora_down=to_dev(self.down), lora_up=to_dev(self.up),
                    smooth=to_dev(torch.from_numpy(self.smooth)),
                    bias=None if self.bias is None else to_dev(self.bias))

    def reference(self):
        xq, xsc = oracle.nvfp4_quantize(self.xs, self.gx)
        D = oracle.lowrank_down(self.xs, self.down)
        return (xq, xsc, D) + oracle.svdq_nvfp4_linear(xq, xsc, self.wq, self.ws, self.gx,
                                                       self.gw, D, self.up, self.bias)


@pytest.mark.parametrize("M,K,N,r", [
    (600, 512, 520, 32),
    (130, 1024, 1536, 16),
    (1024, 3072, 3072, 32),
    (24, 512, 640, 32),     # skinny kernel (32 rows of A per stage)
])
def test_svdq_linear_end_to_end(M, K, N, r):
    from gpu_helpers import unpack_act_scale_atoms
    c = SvdqCase(M, K, N, r, seed=M + r)
    d = c.device_args()
    ws = torch.full((q.svdq_nvfp4_linear_workspace_size(M, K, N, r),), 0xCD, dtype=torch.uint8,
                    device="cuda")
    y = q.svdq_nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                            d["lora_down"], d["lora_up"], smooth=d["smooth"], bias=d["bias"],
                            workspace=ws)
    torch.cuda.synchronize()
    xq, xsc, D, _, y64, T, Tlr = c.reference()
    # the smoothed activations' codes and scales: bit-exact
    codes_off, sf_off, _ = q.nvfp4_linear_workspace_layout(M, K, N)
    buf = ws.cpu().numpy()
    assert np.array_equal(buf[codes_off:codes_off + M * K // 2].reshape(M, K // 2), xq)
    atoms = buf[sf_off:sf_off + -(-M // 128) * (-(-K // 256) * 4) * 512]
    assert np.array_equal(unpack_act_scale_atoms(atoms, M, K), xsc)
    # the branch activations bf16(D / alpha), from fp32 tensor-core sums: within one ulp
    alpha = float(np.float32(c.gx) * np.float32(c.gw))
    base = q.nvfp4_linear_workspace_size(M, K, N)
    lr = oracle.bf16_bits_to_f64(buf[base:base + M * r * 2].view(np.uint16).reshape(M, r))
    want = D / alpha
    assert np.all(np.abs(lr - want) <= 2.0 * oracle.bf16_ulp(want) + 1e-30)
    check_linear(y, y64, T, f"svdq {M}x{K}x{N} r{r}", extra=LR_TOL * Tlr)


def test_svdq_without_smoothing_equals_gemm_lowrank_path():
    M, K, N, r = 512, 768, 1000, 32
    c = SvdqCase(M, K, N, r, seed=9)
    d = c.device_args()
    gx = scalar_dev(float(np.float32(oracle.nvfp4_global_scale(c.x))))
    y1 = q.svdq_nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], gx,
                             d["lora_down"], d["lora_up"], bias=d["bias"])
    torch.cuda.synchronize()
    # the same branch activations through the split calls
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], gx, ws)
    wsv = torch.empty(q.svdq_nvfp4_linear_workspace_size(M, K, N, r), dtype=torch.uint8,
                      device="cuda")
    q.svdq_nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], gx, d["lora_down"],
                        d["lora_up"], bias=d["bias"], workspace=wsv)
    base = q.nvfp4_linear_workspace_size(M, K, N)
    lr_act = wsv[base:base + M * r * 2].view(torch.bfloat16).reshape(M, r)
    y2 = q.nvfp4_linear_gemm_lowrank(M, d["w"], d["weight_scale_2"], gx, ws, lr_act.clone(),
                                     d["lora_up"], bias=d["bias"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
