"""Whole-output parity at the full layer sizes, and out-of-bounds write checks.

1. The NVFP4 MLP up projection (4096 x 3072 x 12288, the layer the benchmark times,
   through the same entry point and tile choice) and the fp8r layer (4096 x 3072 x
   3072) are compared with the fp64 oracle on every output element, not a sample.
2. Canaries (compute-sanitizer is not available on this machine): the output Y, the
   workspace and, for the fused MLP epilogue, the next layer's workspace are placed
   inside larger buffers whose bytes on both sides hold a known pattern; after each
   call those bytes must be unchanged and the inside must be correct. Covered:
   nvfp4_linear, nvfp4_linear_single_launch, fp8r_linear, nvfp4_linear_gelu_quantize
   (its next_workspace), svdq_nvfp4_linear, nvfp4_linear_noalloc, w4a16_linear and
   int4_linear, with N % 8 != 0 (the element-wise tail stores) where the entry point
   takes it.
"""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import Fp8rCase, Nvfp4Case, check_linear, scalar_dev, to_dev

pytestmark = pytest.mark.gpu

PAD = 4096            # canary bytes on each side (keeps 16-byte alignment)
CANARY = 0xA5


class Guarded:
    """A tensor view inside a larger uint8 buffer with canary bytes around it."""

    def __init__(self, nbytes: int, dtype=torch.uint8, shape=None, fill=None):
        self.nbytes = nbytes
        self.buf = torch.full((PAD + nbytes + PAD,), CANARY, dtype=torch.uint8, device="cuda")
        inner = self.buf[PAD:PAD + nbytes]
        if fill is not None:
            inner.fill_(fill)
        t = inner.view(dtype)
        self.t = t if shape is None else t.view(shape)

    def check(self, what: str):
        torch.cuda.synchronize()
        head = self.buf[:PAD].cpu().numpy()
        tail = self.buf[PAD + self.nbytes:].cpu().numpy()
        bad_h = np.flatnonzero(head != CANARY)
        bad_t = np.flatnonzero(tail != CANARY)
        assert bad_h.size == 0 and bad_t.size == 0, (
            f"{what}: {bad_h.size} bytes written before and {bad_t.size} after the buffer "
            f"(first offsets {bad_h[-3:] - PAD if bad_h.size else []}, {bad_t[:3]})")


def guarded_y(M, N):
    # NaN inside: every element must be written
    g = Guarded(M * N * 2, torch.bfloat16, (M, N))
    g.t.fill_(float("nan"))
    return g


# ----------------------------------------------------------------------------- full outputs

def test_nvfp4_mlp_up_whole_output():
    c = Nvfp4Case(4096, 3072, 12288, seed=0)
    d = c.device_args()
    y = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"])
    torch.cuda.synchronize()
    _, y64, T = c.reference()
    check_linear(y, y64, T, "nvfp4 4096x3072x12288, every element")
    assert q.read_device_status() == 0


def test_fp8r_4096x3072x3072_whole_output():
    c = Fp8rCase(4096, 3072, 3072, seed=0)
    d = c.device_args()
    y = q.fp8r_linear(d["x"], d["w"], d["w_scale"])
    torch.cuda.synchronize()
    _, y64, T = c.reference()
    check_linear(y, y64, T, "fp8r 4096x3072x3072, every element")
    assert q.read_device_status() == 0


# ----------------------------------------------------------------------------- canaries

@pytest.mark.parametrize("M,K,N,bias", [
    (600, 512, 520, True),     # CTA pairs, ragged tiles
    (130, 1024, 1000, False),  # single-CTA tiles
    (64, 3072, 200, True),     # N % 8 != 0: element-wise tail stores
    (17, 96, 136, False),      # lone CTA with fewer than 128 rows of A
])
def test_nvfp4_linear_writes_nothing_outside(M, K, N, bias):
    c = Nvfp4Case(M, K, N, seed=M + 3, bias=bias)
    d = c.device_args()
    yg = guarded_y(M, N)
    wg = Guarded(q.nvfp4_linear_workspace_size(M, K, N), fill=0x5A)
    q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                   bias=d["bias"], y=yg.t, workspace=wg.t)
    yg.check("nvfp4_linear y")
    wg.check("nvfp4_linear workspace")
    _, y64, T = c.reference()
    check_linear(yg.t, y64, T, "nvfp4_linear inside the canaries")


@pytest.mark.parametrize("M,K,N", [(600, 512, 520), (64, 3072, 200)])
def test_single_launch_writes_nothing_outside(M, K, N):
    c = Nvfp4Case(M, K, N, seed=M + 4, bias=True)
    d = c.device_args()
    yg = guarded_y(M, N)
    wg = Guarded(q.nvfp4_linear_workspace_size(M, K, N), fill=0xFF)
    q.nvfp4_linear_single_launch(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                                 d["input_scale"], bias=d["bias"], y=yg.t, workspace=wg.t)
    yg.check("nvfp4_linear_single_launch y")
    wg.check("nvfp4_linear_single_launch workspace (sync words included)")
    _, y64, T = c.reference()
    check_linear(yg.t, y64, T, "nvfp4_linear_single_launch inside the canaries")


@pytest.mark.parametrize("M,K,N", [(600, 512, 520), (64, 1024, 200), (300, 256, 3000)])
def test_fp8r_linear_writes_nothing_outside(M, K, N):
    c = Fp8rCase(M, K, N, seed=M + 5, bias=True)
    d = c.device_args()
    yg = guarded_y(M, N)
    wg = Guarded(q.fp8r_linear_workspace_size(M, K, N), fill=0x5A)
    q.fp8r_linear(d["x"], d["w"], d["w_scale"], bias=d["bias"], y=yg.t, workspace=wg.t)
    yg.check("fp8r_linear y")
    wg.check("fp8r_linear workspace")
    _, y64, T = c.reference()
    check_linear(yg.t, y64, T, "fp8r_linear inside the canaries")


def test_gelu_quantize_writes_nothing_outside_next_workspace():
    M, K, N, N2 = 600, 512, 1024, 256
    c = Nvfp4Case(M, K, N, seed=11, bias=True)
    d = c.device_args()
    y = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                       bias=d["bias"])
    torch.cuda.synchronize()
    h_ref, _ = oracle.gelu_bf16(y)
    g2 = float(np.float32(oracle.nvfp4_global_scale(h_ref)))
    nxt = Guarded(q.nvfp4_linear_workspace_size(M, N, N2), fill=0xAB)
    wg = Guarded(q.nvfp4_linear_workspace_size(M, K, N), fill=0x5A)
    q.nvfp4_linear_gelu_quantize(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                                 d["input_scale"], scalar_dev(g2), nxt.t, bias=d["bias"],
                                 workspace=wg.t)
    nxt.check("nvfp4_linear_gelu_quantize next_workspace")
    wg.check("nvfp4_linear_gelu_quantize workspace")
    # the down projection on it stays inside its own buffers too
    down = Nvfp4Case(M, N, N2, seed=12)
    dd = down.device_args()
    yg = guarded_y(M, N2)
    q.nvfp4_linear_quantized_input(M, dd["w"], dd["w_scale"], dd["weight_scale_2"],
                                   scalar_dev(g2), nxt.t, y=yg.t)
    yg.check("nvfp4_linear_quantized_input y")
    nxt.check("nvfp4_linear_quantized_input workspace")
    assert bool(torch.isfinite(yg.t).all())


def test_svdq_writes_nothing_outside():
    from test_gpu_svdq import SvdqCase
    c = SvdqCase(600, 512, 520, 32, seed=13)
    d = c.device_args()
    yg = guarded_y(c.M, c.N)
    wg = Guarded(q.svdq_nvfp4_linear_workspace_size(c.M, c.K, c.N, c.r), fill=0x5A)
    q.svdq_nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                        d["lora_down"], d["lora_up"], smooth=d["smooth"], bias=d["bias"],
                        y=yg.t, workspace=wg.t)
    yg.check("svdq_nvfp4_linear y")
    wg.check("svdq_nvfp4_linear workspace")
    assert bool(torch.isfinite(yg.t).all())


def test_noalloc_w4a16_int4_write_nothing_outside():
    c = Nvfp4Case(64, 3072, 200, seed=14, bias=True)
    d = c.device_args()
    yg = guarded_y(c.M, c.N)
    q.nvfp4_linear_noalloc(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                           bias=d["bias"], y=yg.t)
    yg.check("nvfp4_linear_noalloc y")
    _, y64, T = c.reference()
    check_linear(yg.t, y64, T, "nvfp4_linear_noalloc inside the canaries")
    # W4A16 on the same weight, three rows of activations
    yw = guarded_y(3, c.N)
    q.w4a16_linear(d["x"][:3].contiguous(), d["w"], d["w_scale"], d["weight_scale_2"],
                   bias=d["bias"], y=yw.t)
    yw.check("w4a16_linear y")
    assert bool(torch.isfinite(yw.t).all())
    # INT4 W4A4 with a ragged N
    x = d["x"][:, :2048].contiguous()
    w = (torch.randn(200, 2048, generator=torch.Generator().manual_seed(15)) * 0.02)
    wq, ws = q.prepare_int4_weight(to_dev(w.to(torch.bfloat16)))
    yi = guarded_y(64, 200)
    wg = Guarded(q.int4_linear_workspace_size(64, 2048, 200), fill=0x5A)
    q.int4_linear(x, wq, ws, y=yi.t, workspace=wg.t)
    yi.check("int4_linear y")
    wg.check("int4_linear workspace")
    assert bool(torch.isfinite(yi.t).all())
    assert q.read_device_status() == 0


@pytest.mark.parametrize("M,K,N,bn", [(600, 512, 520, 224), (64, 3072, 200, 128), (17, 96, 136, 192)])
def test_laid_out_weight_scales_write_nothing_outside(M, K, N, bn):
    # the atoms exactly fill their reported size; the laid-out linear writes only Y and
    # the workspace (ragged N, a lone CTA, N % 8 != 0)
    c = Nvfp4Case(M, K, N, seed=M + bn, bias=True)
    d = c.device_args()
    n_atoms = q.nvfp4_weight_scale_atoms_size(N, K, bn)
    ag = Guarded(n_atoms, fill=0x5A)
    q.nvfp4_layout_weight_scales(d["w_scale"], bn, atoms=ag.t)
    ag.check("nvfp4_layout_weight_scales atoms")
    yg = guarded_y(M, N)
    wg = Guarded(q.nvfp4_linear_workspace_size(M, K, N), fill=0x5A)
    q.nvfp4_linear_laid_out(d["x"], d["w"], ag.t, bn, d["weight_scale_2"], d["input_scale"],
                            bias=d["bias"], y=yg.t, workspace=wg.t)
    yg.check("nvfp4_linear_laid_out y")
    wg.check("nvfp4_linear_laid_out workspace")
    ag.check("nvfp4_linear_laid_out atoms (read only)")
    _, y64, T = c.reference()
    check_linear(yg.t, y64, T, "nvfp4_linear_laid_out inside the canaries")
    assert q.read_device_status() == 0


def test_int4_gemm_workspace_write_nothing_outside():
    # the f16 operands and row factors stay inside int4_linear_gemm's workspace
    M, K, N = 130, 576, 200
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(31)).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=torch.Generator().manual_seed(32)) * 0.02).to(torch.bfloat16)
    xq, xs = q.int4_quantize_rows(to_dev(x))
    wq, ws = q.prepare_int4_weight(to_dev(w))
    wg = Guarded(q.int4_linear_gemm_workspace_size(M, K, N), fill=0x5A)
    yg = guarded_y(M, N)
    q.int4_linear_gemm(xq, xs, wq, ws, y=yg.t, workspace=wg.t)
    wg.check("int4_linear_gemm workspace")
    yg.check("int4_linear_gemm y")
    assert bool(torch.isfinite(yg.t).all())
    assert q.read_device_status() == 0
