"""Pins of the oracle's W4A16 pieces (NVFP4 weights dequantized to bf16, bf16
activations, a plain linear), independent of the oracle's own code:
  * with weight_scale_2 = 1 every dequantized weight is the exact product of the
    golden E2M1 grid and PyTorch's E4M3 decode (the product has at most 6
    significant bits, so bf16 holds it);
  * for arbitrary fp32 weight_scale_2 the dequantized weight equals numpy's fp32
    cast of the exact rational product followed by PyTorch's bf16 cast;
  * a hand-derived case where rounding to fp32 first and then to bf16 differs from
    rounding the exact product to bf16 once;
  * the linear on small integers equals the exact integer matmul, and for a
    power-of-two weight_scale_2 it equals the (separately pinned) fallback oracle
    that scales after the sum.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from synthetic import make_linear_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_grid():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_grid.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                code, v = line.split()
                vals[int(code, 16)] = float(v)
    return vals


def _e4m3_value(code):
    return torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()


def _bf16_bits(values_f32):
    t = torch.from_numpy(np.asarray(values_f32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _pack(codes):
    codes = np.asarray(codes, np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def test_dequant_unit_global_scale_is_the_exact_grid_product():
    grid = _e2m1_grid()
    scale_codes = [0x00, 0x01, 0x07, 0x08, 0x30, 0x38, 0x3C, 0x40, 0x55, 0x7E]
    codes = np.array([c for c in range(16)], np.uint8)
    q = _pack(np.tile(codes, (len(scale_codes), 1)))
    s = np.array(scale_codes, np.uint8)[:, None]
    got = oracle.bf16_bits_to_f64(oracle.w4a16_dequantize_bf16(q, s, 1.0))
    for i, sc in enumerate(scale_codes):
        want = [grid[c] * _e4m3_value(sc) for c in range(16)]
        assert got[i].tolist() == want, hex(sc)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dequant_is_fp32_then_bf16_rounding_of_the_exact_product(seed):
    rng = np.random.default_rng(seed)
    grid = _e2m1_grid()
    R, K = 6, 64
    codes = rng.integers(0, 16, size=(R, K)).astype(np.uint8)
    sc = rng.integers(0, 0x7F, size=(R, K // 16)).astype(np.uint8)  # no NaN codes
    ws2 = np.float32(rng.uniform(1e-4, 3.0))
    got = oracle.w4a16_dequantize_bf16(_pack(codes), sc, ws2)
    exact = np.array([[float(Fraction(grid[int(codes[r, k])]) *
                             Fraction(_e4m3_value(int(sc[r, k // 16]))) * Fraction(float(ws2)))
                       for k in range(K)] for r in range(R)])  # exact in fp64 (<= 30 bits)
    # zeros keep the sign of the IEEE product (code 0x8 is -0)
    signs = np.array([[np.copysign(1.0, grid[int(codes[r, k])]) for k in range(K)]
                      for r in range(R)])
    exact = np.where(exact == 0.0, np.copysign(0.0, signs), exact)
    want = _bf16_bits(exact.astype(np.float32))  # numpy RN to fp32, then torch RN to bf16
    assert np.array_equal(got, want)


def _find_double_rounding_case():
    """An fp32 weight_scale_2 f and a product v * bs in {3, 1.5} such that the exact
    weight P = v * bs * f is not a bf16 midpoint, its fp32 rounding is one, and the
    tie then goes the other way than a single rounding of P to bf16 would."""
    for c in (3, Fraction(3, 2)):
        for e in range(0, 64):  # bf16 values b = 1 + e/128 in [1, 1.5)
            b = Fraction(1) + Fraction(e, 128)
            mid = b + Fraction(1, 256)
            f0 = np.float32(float(mid / c))
            for d in range(-3, 4):
                f = f0
                for _ in range(abs(d)):
                    f = np.nextafter(f, np.float32(2.0) if d > 0 else np.float32(0.0))
                P = c * Fraction(float(f))
                if P == mid or Fraction(float(np.float32(float(P)))) != mid:
                    continue
                even_is_b = e % 2 == 0
                double = b if even_is_b else b + Fraction(1, 128)
                single = b + Fraction(1, 128) if P > mid else b
                if double != single:
                    return c, f, float(double), float(single)
    return None


def test_double_rounding_hand_case():
    # The exact product rounds to fp32 exactly onto a bf16 midpoint, which then
    # rounds to the even neighbour; rounding the exact product to bf16 in one step
    # would give the other neighbour.
    case = _find_double_rounding_case()
    assert case is not None
    c, f, double, single = case
    code, scale = (5, 0x38) if c == 3 else (3, 0x38)  # 3.0 x 1.0 or 1.5 x 1.0
    q = _pack(np.array([[code] + [0] * 15], np.uint8))
    s = np.array([[scale]], np.uint8)
    got = oracle.bf16_bits_to_f64(oracle.w4a16_dequantize_bf16(q, s, f))[0, 0]
    assert got == double and got != single


def test_linear_small_integers_is_the_integer_matmul():
    rng = np.random.default_rng(3)
    M, K, N = 5, 64, 7
    xi = rng.integers(-8, 9, size=(M, K))
    # codes 2 (1.0), 4 (2.0), 6 (4.0) and their negatives, unit scales: integer weights
    pick = np.array([0x2, 0x4, 0x6, 0xA, 0xC, 0xE, 0x0], np.uint8)
    codes = pick[rng.integers(0, len(pick), size=(N, K))]
    grid = _e2m1_grid()
    wi = np.vectorize(lambda c: int(grid[int(c)]))(codes)
    s = np.full((N, K // 16), 0x38, np.uint8)
    x = torch.from_numpy(xi).to(torch.bfloat16)
    bias = np.arange(N, dtype=np.float32) - 3.0
    y, y64, T = oracle.w4a16_linear(x, _pack(codes), s, 1.0, bias)
    want = (torch.from_numpy(xi) @ torch.from_numpy(wi).T).numpy().astype(np.float64) + bias
    assert np.array_equal(y64, want)
    assert np.array_equal(oracle.bf16_bits_to_f64(y), want)   # |values| < 256: exact in bf16
    assert np.array_equal(T, (np.abs(xi)[:, None, :] * np.abs(wi)[None, :, :]).sum(-1))


@pytest.mark.parametrize("j", [-3, 0, 2])
def test_power_of_two_global_scale_matches_the_scaled_fallback(j):
    inp = make_linear_inputs(16, 128, 24, seed=7 + j, with_bias=True)
    gw = oracle.nvfp4_global_scale(inp.w)
    wq, ws = oracle.nvfp4_quantize(inp.w, gw)
    ws2 = np.float32(2.0 ** j)
    _, y64, _ = oracle.w4a16_linear(inp.x, wq, ws, ws2, inp.bias.numpy())
    y64_fb = oracle.nvfp4_linear_unquantized_act(inp.x, wq, ws, ws2, inp.bias.numpy())
    assert np.array_equal(y64, y64_fb)
