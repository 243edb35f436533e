"""Pins of the oracle's contractions.

* Brute force in exact rational arithmetic on tiny shapes: every dequantized
  NVFP4 value is a multiple of 2^-10 (E2M1 values are multiples of 1/2, E4M3
  values multiples of 2^-9), every E4M3 value a multiple of 2^-9, so the sums
  are computed exactly with Python integers and compared with the fp64 oracle.
* Closed forms: all-ones codes with unit scales give K * alpha; fp8r with unit
  scales and small-integer codes is the plain integer matmul.
* The device-fallback remark of the BFL page ("Kernels", last paragraph: without
  activation quantization the outputs differ slightly from the fused kernels):
  the oracle with quantized activations differs from the one without by a small
  but clearly nonzero amount.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from synthetic import make_linear_inputs

E2M1_VAL = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
            Fraction(3), Fraction(4), Fraction(6)]


def e2m1_exact(n):
    v = E2M1_VAL[n & 7]
    return -v if n & 8 else v


def e4m3_exact(c):
    s, e, m = (c >> 7) & 1, (c >> 3) & 15, c & 7
    assert not (e == 15 and m == 7)
    v = Fraction(m, 512) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if s else v


def nvfp4_row_exact(q, s):
    K = q.size * 2
    out = []
    for k in range(K):
        byte = int(q[k // 2])
        nib = byte & 0xF if k % 2 == 0 else byte >> 4
        out.append(e2m1_exact(nib) * e4m3_exact(int(s[k // 16])))
    return out


def bf16_exact_round(v: Fraction) -> int:
    """Nearest-even bf16 of an exact rational (normal range only, as used here)."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    m = a * 128                          # in [128, 256)
    fl = int(m)
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    if fl == 256:
        fl = 128
        e += 1
    return sign | ((e + 127) << 7) | (fl - 128)


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (3, 2, 32), (4, 4, 64), (2, 3, 48)])
def test_nvfp4_linear_bruteforce_exact(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    xq = rng.integers(0, 256, size=(M, K // 2)).astype(np.uint8)
    wq = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
    xs = rng.integers(0, 0x7F, size=(M, K // 16)).astype(np.uint8)
    ws = rng.integers(0, 0x7F, size=(N, K // 16)).astype(np.uint8)
    gi, gw = 2.0 ** -7, 2.0 ** -4                 # powers of two: y64 is exact
    y, y64, T = oracle.nvfp4_linear(xq, xs, wq, ws, gi, gw)
    for m in range(M):
        a = nvfp4_row_exact(xq[m], xs[m])
        for n in range(N):
            b = nvfp4_row_exact(wq[n], ws[n])
            acc = sum(p * q for p, q in zip(a, b))
            absacc = sum(abs(p * q) for p, q in zip(a, b))
            want = acc * Fraction(gi) * Fraction(gw)
            assert Fraction(y64[m, n]) == want, (m, n)
            assert Fraction(T[m, n]) == absacc * Fraction(gi) * Fraction(gw)
            assert int(y[m, n]) == bf16_exact_round(want), (m, n)


def test_nvfp4_linear_bias_added_after_scale():
    K = 32
    ones = np.full((1, K // 2), 0x22, np.uint8)     # every element 1.0
    unit = np.full((1, K // 16), 0x38, np.uint8)    # E4M3 1.0
    bias = np.array([0.25], np.float32)
    y, y64, T = oracle.nvfp4_linear(ones, unit, ones, unit, 0.5, 0.125, bias)
    assert y64[0, 0] == K * 0.5 * 0.125 + 0.25     # closed form: K * alpha + bias
    assert T[0, 0] == K * 0.5 * 0.125


def test_nvfp4_linear_transposed_operands_differ():
    # A swap of X and W roles must change y for a non-symmetric case (guards
    # against a transposed operand in the contraction).
    rng = np.random.default_rng(9)
    xq = rng.integers(0, 256, size=(2, 16)).astype(np.uint8)
    wq = rng.integers(0, 256, size=(3, 16)).astype(np.uint8)
    xs = rng.integers(0x30, 0x40, size=(2, 2)).astype(np.uint8)
    ws = rng.integers(0x30, 0x40, size=(3, 2)).astype(np.uint8)
    _, y1, _ = oracle.nvfp4_linear(xq, xs, wq, ws, 1.0, 1.0)
    _, y2, _ = oracle.nvfp4_linear(wq, ws, xq, xs, 1.0, 1.0)
    assert np.array_equal(y1, y2.T)
    assert y1.shape == (2, 3)


def test_fp8r_linear_is_integer_matmul_with_unit_scales():
    rng = np.random.default_rng(10)
    M, N, K = 5, 7, 40
    a = rng.integers(-16, 17, size=(M, K))
    b = rng.integers(-16, 17, size=(N, K))
    enc = lambda v: oracle.e4m3_encode(v.astype(np.float32))   # small ints are exact in E4M3
    xq, wq = enc(a), enc(b)
    y, y64, T = oracle.fp8r_linear(xq, np.ones(M, np.float32), wq, np.ones(N, np.float32))
    ref = a @ b.T
    assert np.array_equal(y64, ref.astype(np.float64))
    assert np.array_equal(T, (np.abs(a) @ np.abs(b).T).astype(np.float64))


def test_fp8r_linear_row_scales_bruteforce():
    rng = np.random.default_rng(11)
    M, N, K = 3, 4, 24
    xq = rng.integers(0, 0x7F, size=(M, K)).astype(np.uint8) | (rng.integers(0, 2, (M, K)) << 7).astype(np.uint8)
    wq = rng.integers(0, 0x7F, size=(N, K)).astype(np.uint8)
    xs = (2.0 ** rng.integers(-8, 0, size=M)).astype(np.float32)
    ws = (2.0 ** rng.integers(-8, 0, size=N)).astype(np.float32)
    bias = np.array([0.5, -0.25, 0.0, 1.0], np.float32)
    y, y64, _ = oracle.fp8r_linear(xq, xs, wq, ws, bias)
    for m in range(M):
        for n in range(N):
            acc = sum(e4m3_exact(int(xq[m, k])) * e4m3_exact(int(wq[n, k])) for k in range(K))
            want = acc * Fraction(float(xs[m])) * Fraction(float(ws[n])) + Fraction(float(bias[n]))
            assert Fraction(y64[m, n]) == want
            assert int(y[m, n]) == bf16_exact_round(want)


def test_activation_quantization_changes_output_slightly():
    inp = make_linear_inputs(64, 256, 64, seed=12)
    gw = oracle.nvfp4_global_scale(inp.w)
    wq, ws = oracle.nvfp4_quantize(inp.w, gw)
    gx = oracle.nvfp4_global_scale(inp.x)
    xq, xs = oracle.nvfp4_quantize(inp.x, gx)
    _, yq, _ = oracle.nvfp4_linear(xq, xs, wq, ws, gx, gw)
    yu = oracle.nvfp4_linear_unquantized_act(inp.x, wq, ws, gw)
    rel = np.linalg.norm(yq - yu) / np.linalg.norm(yu)
    # 4-bit activations with 16-element blocks: a few percent to tens of percent
    # of relative error, far above the 5e-3 GPU-vs-oracle tolerance, well below 1.
    assert 0.02 < rel < 0.5, rel
