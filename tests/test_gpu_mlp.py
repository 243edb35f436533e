"""GPU parity of the MLP path with the fused GELU + NVFP4 requantization epilogue:
nvfp4_linear_gelu_quantize (up projection -> quantized GELU into the down
projection's workspace) and nvfp4_linear_quantized_input (the down projection).

The up projection's pre-GELU value v = bf16(alpha * acc + bias) is the value
nvfp4_linear stores as Y (same kernels, same arithmetic), so the oracle starts from
that Y: h = bf16(GELU(v)) in fp64, then the NVFP4 quantization of h (the oracle's
rule) under the given global scale. Codes and block scales must match bit for bit
on every 16-element block that holds no element whose exact GELU lies within the
GPU's fp32 error of a bf16 rounding midpoint (oracle.gelu_bf16 flags those; they
are at most a few per thousand). Those blocks are checked too: their codes and
scale must equal the oracle's quantization of the block with each flagged element
taken at one of its two bf16 roundings (the oracle's, or the neighbour on the
side of the exact fp64 GELU), so no block goes unchecked. The down projection is
checked against the oracle linear on the codes the GPU wrote, within the usual
tolerance.
"""
import itertools

import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import (Nvfp4Case, bf16_bits, check_linear, sample_rows, scalar_dev, to_dev,
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


def _other_rounding(v_bits: int, h_bits: int) -> int:
    """The bf16 neighbour of h (bits) on the side of the exact fp64 GELU of v."""
    v = float(oracle.bf16_bits_to_f64(np.array([v_bits], dtype=np.uint16))[0])
    h = float(oracle.bf16_bits_to_f64(np.array([h_bits], dtype=np.uint16))[0])
    exact = oracle.gelu(v)
    if exact == h:
        return h_bits
    if h == 0.0:
        return 0x0001 if exact > 0 else 0x8001
    up = (exact > h) == (h > 0)                  # away from zero in magnitude
    return (h_bits + 1) if up else (h_bits - 1)


def check_ambiguous_blocks(v_bits, h_ref, amb, g2, codes, scales):
    """Every block with a flagged element: the GPU's 8 code bytes and scale equal the
    oracle's NVFP4 of the block for some choice of rounding of its flagged elements.
    v_bits, h_ref, amb: [R, N]; codes [R, N/2]; scales [R, N/16]."""
    R, N = h_ref.shape
    blk = amb.reshape(R, N // 16, 16).any(axis=2)
    cands, owner = [], []
    for r, b in np.argwhere(blk):
        hb = h_ref[r, 16 * b:16 * b + 16]
        opts = []
        for i in range(16):
            if amb[r, 16 * b + i]:
                opts.append(sorted({int(hb[i]), _other_rounding(int(v_bits[r, 16 * b + i]),
                                                                 int(hb[i]))}))
            else:
                opts.append([int(hb[i])])
        combos = list(itertools.product(*opts))
        assert len(combos) <= 256, "too many flagged elements in one block"
        cands.extend(combos)
        owner.extend([(r, b)] * len(combos))
    if not cands:
        return 0
    cq, cs = oracle.nvfp4_quantize(np.array(cands, dtype=np.uint16), g2)   # [C, 8], [C, 1]
    matched = {}
    for (r, b), q8, s1 in zip(owner, cq, cs):
        if np.array_equal(codes[r, 8 * b:8 * b + 8], q8) and scales[r, b] == s1[0]:
            matched[(r, b)] = True
    missing = [rb for rb in map(tuple, np.argwhere(blk)) if rb not in matched]
    assert not missing, f"{len(missing)} ambiguous blocks match no valid rounding, e.g. {missing[:5]}"
    return int(blk.sum())


def check_codes(M, N, h_ref, amb, g2, next_ws, v_bits):
    codes, scales, atoms = _act_part(next_ws, M, N)
    xq_ref, xs_ref = oracle.nvfp4_quantize(h_ref, g2)
    block_amb = amb.reshape(M, N // 16, 16).any(axis=2)           # [M, N/16]
    assert block_amb.mean() < 0.02, block_amb.mean()
    ok_s = scales == xs_ref
    assert np.all(ok_s | block_amb), np.argwhere(~(ok_s | block_amb))[:5]
    byte_amb = np.repeat(block_amb, 8, axis=1)                      # 8 code bytes per block
    ok_q = codes == xq_ref
    assert np.all(ok_q | byte_amb), np.argwhere(~(ok_q | byte_amb))[:5]
    check_ambiguous_blocks(v_bits, h_ref, amb, g2, codes, scales)
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
    _, _, y, h_ref, amb, g2, next_ws = run_up(M, K, N, seed=M + K)
    check_codes(M, N, h_ref, amb, g2, next_ws, bf16_bits(y))


def test_mlp_up_to_down_matches_oracle():
    M, K, N, N2 = 512, 768, 1536, 512
    c, d, y, h_ref, amb, g2, next_ws = run_up(M, K, N, seed=77, n_next=N2)
    codes, scales = check_codes(M, N, h_ref, amb, g2, next_ws, bf16_bits(y))
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
    check_ambiguous_blocks(bf16_bits(y)[rows], h_ref[rows], amb[rows], g2, codes[rows],
                           scales[rows])
    assert q.read_device_status() == 0


def test_rejects_n_not_multiple_of_256():
    c = Nvfp4Case(128, 256, 384, seed=1)
    d = c.device_args()
    next_ws = torch.empty(q.nvfp4_linear_workspace_size(128, 384, 256), dtype=torch.uint8,
                          device="cuda")
    with pytest.raises(q.QLinearError):
        q.nvfp4_linear_gelu_quantize(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                                     d["input_scale"], d["input_scale"], next_ws)
