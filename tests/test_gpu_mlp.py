"""GPU parity of the MLP path with the fused GELU + NVFP4 requantization epilogue:
nvfp4_linear_gelu_quantize (up projection -> quantized GELU into the down
projection's workspace) and nvfp4_linear_quantized_input (the down projection).

The up projection's pre-GELU value v = bf16(alpha * acc + bias) is the value
nvfp4_linear stores as Y (same kernels, same arithmetic), so the oracle starts from
that Y: h = bf16(GELU(v)) in fp64, then the NVFP4 quantization of h (the oracle's
rule) under the given global scale. Codes and block scales must match bit for bit
on every 16-element block that holds no element whose exact GELU lies within the
GPU's fp32 error of a bf16 rounding midpoint (oracle.gelu_bf16 flags those; they
are at most a few per thousand). The down projection is checked against the
oracle linear on the codes the GPU wrote, within the usual tolerance.
"""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import (Nvfp4Case, check_linear, sample_rows, scalar_dev, to_dev,
                         unpack_act_scale_atoms)

pytestmark = pytest.mark.gpu


def _act_part(ws, M, K):
    codes_off, sf_off, _ = q.nvfp4_linear_workspace_layout(M, K, 256)
    buf = ws.cpu().numpy()
    KG = K // 64
    codes = buf[codes_off:codes_off + M * K // 2].reshape(M, K // 2)
    atoms = buf[sf_off:sf_off + -(-M // 128) * KG * 512]
    return codes, unpack_act_scale_atoms(atoms, M, K), atoms


def run_up(M, K, N, seed, bias=True, n_next=256):
    c = Nvfp4Case(M, K, N, seed=seed, bias=bias)
    d = c.device_args()
    y = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                       bias=d["bias"])
    torch.cuda.synchronize()
    h_ref, amb = oracle.gelu_bf16(y)
    g2 = np.float32(oracle.nvfp4_global_scale(h_ref))
    next_ws = torch.full((q.nvfp4_linear_workspace_size(M, N, n_next),), 0xAB, dtype=torch.uint8,
                         device="cuda")
    q.nvfp4_linear_gelu_quantize(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                                 d["input_scale"], scalar_dev(float(g2)), next_ws, bias=d["bias"])
    torch.cuda.synchronize()
    return c, d, y, h_ref, amb, g2, next_ws


def check_codes(M, N, h_ref, amb, g2, next_ws):
    codes, scales, atoms = _act_part(next_ws, M, N)
    xq_ref, xs_ref = oracle.nvfp4_quantize(h_ref, g2)
    block_amb = amb.reshape(M, N // 16, 16).any(axis=2)           # [M, N/16]
    assert block_amb.mean() < 0.02, block_amb.mean()
    ok_s = scales == xs_ref
    assert np.all(ok_s | block_amb), np.argwhere(~(ok_s | block_amb))[:5]
    byte_amb = np.repeat(block_amb, 8, axis=1)                      # 8 code bytes per block
    ok_q = codes == xq_ref
    assert np.all(ok_q | byte_amb), np.argwhere(~(ok_q | byte_amb))[:5]
    # padding rows of the last 128-row atom group carry zero scales
    m_pad = -(-M // 128) * 128
    if m_pad > M:
        pad = unpack_act_scale_atoms(atoms, m_pad, N)[M:]
        assert not pad.any()
    return codes, scales


@pytest.mark.parametrize("M,K,N", [
    (600, 512, 1024),   # CTA pairs, ragged M, 2 rows of padding atoms
    (130, 256, 768),    # single-CTA tiles, tile widths that do not divide N
    (1024, 3072, 3072),
])
def test_gelu_quantize_codes_bit_exact(M, K, N):
    _, _, _, h_ref, amb, g2, next_ws = run_up(M, K, N, seed=M + K)
    check_codes(M, N, h_ref, amb, g2, next_ws)


def test_mlp_up_to_down_matches_oracle():
    M, K, N, N2 = 512, 768, 1536, 512
    c, d, y, h_ref, amb, g2, next_ws = run_up(M, K, N, seed=77, n_next=N2)
    codes, scales = check_codes(M, N, h_ref, amb, g2, next_ws)
    down = Nvfp4Case(M, N, N2, seed=78, bias=True)   # its weight, scales and bias
    dd = down.device_args()
    y2 = q.nvfp4_linear_quantized_input(M, dd["w"], dd["w_scale"], dd["weight_scale_2"],
                                        scalar_dev(float(g2)), next_ws, bias=dd["bias"])
    torch.cuda.synchronize()
    _, y64, T = oracle.nvfp4_linear(codes, scales, down.wq, down.ws, g2, down.gw, down.bias)
    check_linear(y2, y64, T, "down projection on fused-epilogue codes")


def test_quantized_input_equals_nvfp4_linear():
    # a workspace whose activations come from the ordinary prologue gives nvfp4_linear
    M, K, N = 700, 1280, 1000
    c = Nvfp4Case(M, K, N, seed=5, bias=True)
    d = c.device_args()
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws)
    y1 = q.nvfp4_linear_quantized_input(M, d["w"], d["w_scale"], d["weight_scale_2"],
                                        d["input_scale"], ws, bias=d["bias"])
    y2 = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                        bias=d["bias"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_dit_mlp_up_sampled_rows():
    M, K, N = 4096, 3072, 12288
    _, _, y, h_ref, amb, g2, next_ws = run_up(M, K, N, seed=0, bias=False)
    rows = sample_rows(M, 12, seed=3)
    codes, scales, _ = _act_part(next_ws, M, N)
    xq_ref, xs_ref = oracle.nvfp4_quantize(h_ref[rows], g2)
    block_amb = amb[rows].reshape(len(rows), N // 16, 16).any(axis=2)
    assert np.all((scales[rows] == xs_ref) | block_amb)
    assert np.all((codes[rows] == xq_ref) | np.repeat(block_amb, 8, axis=1))
    assert q.read_device_status() == 0


def test_rejects_n_not_multiple_of_256():
    c = Nvfp4Case(128, 256, 384, seed=1)
    d = c.device_args()
    next_ws = torch.empty(q.nvfp4_linear_workspace_size(128, 384, 256), dtype=torch.uint8,
                          device="cuda")
    with pytest.raises(q.QLinearError):
        q.nvfp4_linear_gelu_quantize(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                                     d["input_scale"], d["input_scale"], next_ws)
