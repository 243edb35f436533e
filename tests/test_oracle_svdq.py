"""Pins of the oracle's SVDQuant-style pieces (smoothing, 16-bit low-rank branch,
and the NVFP4 linear with the branch added), independent of the oracle's own code:
  * smoothing by a power of two is an exact exponent shift; hand-worked cases of the
    fp32 product rounded to bf16;
  * the low-rank down projection of small integers equals the exact integer product;
  * with a zero up projection the linear reduces to the pinned nvfp4_linear; with
    all-zero residual codes it is the closed form bf16(D up^T + bias) on integers;
  * the low-rank term is linear in `up`, and T_lr is the sum of absolute terms.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import make_linear_inputs


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_smoothing_by_powers_of_two_is_exact():
    x = (torch.randn(8, 64) * 3).to(torch.bfloat16)
    s = np.array([2.0 ** (k % 7 - 3) for k in range(64)], dtype=np.float32)
    got = oracle.smooth_bf16(x, s)
    want = _bits((x.float() * torch.from_numpy(s)).to(torch.bfloat16))  # exact: no rounding
    assert np.array_equal(got, want)


def test_smoothing_rounds_in_fp32_then_bf16():
    # 1.5 * fp32(1/3): the fp32 product 0.50000001... rounds to bf16 0.5
    x = torch.tensor([[1.5, -1.5]], dtype=torch.bfloat16)
    s = np.array([1.0 / 3.0, 1.0 / 3.0], dtype=np.float32)
    got = oracle.bf16_bits_to_f64(oracle.smooth_bf16(x, s))
    assert got.tolist() == [[0.5, -0.5]]
    # 1.0078125 * 1.0078125 = 1.01568603515625 (exact in fp32); its bf16 neighbours
    # are 1.015625 and 1.0234375, so the result is 1.015625
    x = torch.tensor([[1.0078125]], dtype=torch.bfloat16)
    s = np.array([1.0078125], dtype=np.float32)
    assert oracle.bf16_bits_to_f64(oracle.smooth_bf16(x, s))[0, 0] == 1.015625


def test_lowrank_down_integer_brute_force():
    rng = np.random.default_rng(0)
    xi = rng.integers(-8, 9, size=(5, 48))
    di = rng.integers(-8, 9, size=(4, 48))
    xs = _bits(torch.from_numpy(xi).to(torch.bfloat16))
    down = _bits(torch.from_numpy(di).to(torch.bfloat16))
    D = oracle.lowrank_down(xs, down)
    assert np.array_equal(D, (xi @ di.T).astype(np.float64))


def test_zero_up_projection_reduces_to_nvfp4_linear():
    inp = make_linear_inputs(64, 256, 96, seed=3, with_bias=True)
    gw = oracle.nvfp4_global_scale(inp.w)
    wq, ws = oracle.nvfp4_quantize(inp.w, gw)
    gx = oracle.nvfp4_global_scale(inp.x)
    xq, xs = oracle.nvfp4_quantize(inp.x, gx)
    D = np.random.default_rng(1).standard_normal((64, 32))
    up = np.zeros((96, 32), dtype=np.uint16)
    y, y64, T, Tlr = oracle.svdq_nvfp4_linear(xq, xs, wq, ws, gx, gw, D, up, inp.bias.numpy())
    y_ref, y64_ref, T_ref = oracle.nvfp4_linear(xq, xs, wq, ws, gx, gw, inp.bias.numpy())
    assert np.array_equal(y, y_ref) and np.array_equal(y64, y64_ref) and np.array_equal(T, T_ref)
    assert not Tlr.any()


def test_zero_residual_closed_form_and_linearity():
    M, K, N, r = 6, 64, 10, 3
    rng = np.random.default_rng(2)
    xq = np.zeros((M, K // 2), dtype=np.uint8)
    xs = np.zeros((M, K // 16), dtype=np.uint8)
    wq = np.zeros((N, K // 2), dtype=np.uint8)
    ws = np.full((N, K // 16), 0x38, dtype=np.uint8)  # scale 1.0, codes 0
    Di = rng.integers(-5, 6, size=(M, r))
    ui = rng.integers(-5, 6, size=(N, r))
    up = _bits(torch.from_numpy(ui).to(torch.bfloat16))
    bias = np.arange(N, dtype=np.float32) * 0.5
    y, y64, T, Tlr = oracle.svdq_nvfp4_linear(xq, xs, wq, ws, 1.0, 1.0, Di.astype(float), up, bias)
    want = (Di @ ui.T).astype(np.float64) + bias
    assert np.array_equal(y64, want)
    assert np.array_equal(oracle.bf16_bits_to_f64(y), want)        # small integers: exact bf16
    assert np.array_equal(Tlr, (np.abs(Di)[:, None, :] * np.abs(ui)[None, :, :]).sum(-1))
    up2 = _bits(torch.from_numpy(2 * ui).to(torch.bfloat16))
    _, y64b, _, _ = oracle.svdq_nvfp4_linear(xq, xs, wq, ws, 1.0, 1.0, Di.astype(float), up2, bias)
    assert np.array_equal(y64b - bias, 2 * (y64 - bias))


def test_smoothing_rounds_to_fp32_first_golden():
    """tests/golden/svdq_smoothing_rounding.txt: the fp32 product lands exactly on a
    bf16 midpoint (a tie to even), where one rounding of the exact product would go the
    other way."""
    import os
    rows = {}
    path = os.path.join(os.path.dirname(__file__), "golden", "svdq_smoothing_rounding.txt")
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows[key] = [int(v, 16) for v in vals]
    x = torch.from_numpy(np.array(rows["x_bits"], np.uint16).view(np.int16)).view(
        torch.bfloat16).reshape(1, 1)
    smooth = np.array(rows["smooth_bits"], np.uint32).view(np.float32)
    out = oracle.smooth_bf16(x, smooth)
    assert int(out[0, 0]) == rows["xs_bits"][0]


def test_low_rank_term_is_not_scaled_by_the_global_scales():
    # with a zero 4-bit residual, Y = D up^T + bias whatever input_scale and
    # weight_scale_2 are: only the 4-bit product carries them
    M, K, N, r = 4, 64, 6, 3
    rng = np.random.default_rng(5)
    xq = np.zeros((M, K // 2), dtype=np.uint8)
    xs = np.full((M, K // 16), 0x38, dtype=np.uint8)
    wq = np.zeros((N, K // 2), dtype=np.uint8)
    ws = np.full((N, K // 16), 0x38, dtype=np.uint8)
    Di = rng.integers(-5, 6, size=(M, r))
    ui = rng.integers(-5, 6, size=(N, r))
    up = _bits(torch.from_numpy(ui).to(torch.bfloat16))
    bias = np.arange(N, dtype=np.float32)
    _, y64, _, _ = oracle.svdq_nvfp4_linear(xq, xs, wq, ws, 0.5, 0.25, Di.astype(float), up, bias)
    assert np.array_equal(y64, (Di @ ui.T).astype(np.float64) + bias)


def test_lowrank_down_is_exact_under_cancellation():
    # 2^24 + 1 - 2^24: an fp32 accumulation loses the 1, the exact contraction keeps it
    K = 16
    xi = np.zeros((2, K))
    xi[0, :3] = [2.0 ** 24, 1.0, -(2.0 ** 24)]
    xi[1, :4] = [2.0 ** 30, 3.0, -(2.0 ** 30), 0.5]
    xs = _bits(torch.from_numpy(xi).to(torch.bfloat16))
    down = _bits(torch.ones(1, K, dtype=torch.bfloat16))
    D = oracle.lowrank_down(xs, down)
    assert D[0, 0] == 1.0 and D[1, 0] == 3.5
