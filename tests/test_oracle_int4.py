"""Pins of the oracle's INT4 W4A4 pieces (the INT4 variant of the Nunchaku page's
svdq_w4a4 family; format reading: signed 4-bit codes in [-8, 7], one fp32 scale =
amax / 7 per 64-element group, codes = clamp(round-half-even(x / scale)) with the
reciprocal multiply), independent of the oracle's own code:
  * inputs that are exactly code * 2^e with a +-7 in every group come back as those
    codes and scales (the largest magnitude maps to 7);
  * hand-worked ties round to even; zero groups give zero codes and scale 0;
  * sign symmetry; the clamp to [-8, 7] (only reachable through rounding up);
  * the linear equals exact rational arithmetic on tiny shapes (Fractions), a closed
    form, and numpy's matmul of the dequantized operands;
  * a row of three groups worked by hand (tests/golden/int4_worked_groups.txt): its
    packed bytes, scales and the bf16 result of its linear with itself (a tie).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def unpack(q):
    """uint8 [R, K/2] -> int [R, K] (element 2j in the low nibble, two's complement)."""
    lo = (q & 0xF).astype(np.int64)
    hi = (q >> 4).astype(np.int64)
    out = np.empty((q.shape[0], q.shape[1] * 2), np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return np.where(out >= 8, out - 16, out)


def pack(c):
    c = np.asarray(c, np.int64) & 0xF
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_pack_unpack_round_trip_over_all_codes():
    codes = np.arange(-8, 8).repeat(8).reshape(2, 64)
    assert np.array_equal(unpack(pack(codes)), codes)


def test_representable_inputs_come_back_exactly():
    rng = np.random.default_rng(0)
    R, K = 6, 256
    codes = rng.integers(-7, 8, size=(R, K))
    exps = rng.integers(-12, 6, size=(R, K // 64))
    for r in range(R):
        for g in range(K // 64):
            codes[r, g * 64 + int(rng.integers(0, 64))] = 7 if rng.random() < 0.5 else -7
    scale = np.ldexp(1.0, exps).astype(np.float32)
    x = codes * np.repeat(scale, 64, axis=1)          # exact: 3 significant bits
    q, s = oracle.int4_quantize(bf16(x))
    assert np.array_equal(s, scale)
    assert np.array_equal(unpack(q), codes)


def test_ties_round_to_even_and_zero_groups():
    x = np.zeros((2, 64), np.float32)
    x[0, :8] = [7.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 0.49]    # scale 1
    q, s = oracle.int4_quantize(bf16(x))
    assert s[0, 0] == 1.0 and s[1, 0] == 0.0
    assert unpack(q)[0, :8].tolist() == [7, 2, 4, -2, 0, 0, 2, 0]
    assert not unpack(q)[1].any()


def test_sign_symmetry():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 192)).astype(np.float32)
    q1, s1 = oracle.int4_quantize(bf16(x))
    q2, s2 = oracle.int4_quantize(bf16(-x))
    assert np.array_equal(s1, s2)
    assert np.array_equal(unpack(q2), -unpack(q1))


def test_codes_stay_in_range():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 640)) * np.exp(rng.standard_normal((64, 1)))).astype(np.float32)
    q, s = oracle.int4_quantize(bf16(x))
    c = unpack(q)
    assert c.min() >= -8 and c.max() <= 7
    # the group maximum maps to +-7 (up to the rounding of amax / 7 and its reciprocal)
    xb = bf16(x).float().numpy()
    for r in range(0, 64, 7):
        g = 3
        i = np.argmax(np.abs(xb[r, g * 64:(g + 1) * 64]))
        assert abs(c[r, g * 64 + i]) == 7


def _exact_linear(cx, sx, cw, sw, bias):
    M, K = cx.shape
    N = cw.shape[0]
    y = np.empty((M, N), object)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for g in range(K // 64):
                isum = int(np.dot(cx[m, g * 64:(g + 1) * 64], cw[n, g * 64:(g + 1) * 64]))
                acc += Fraction(float(sx[m, g])) * Fraction(float(sw[n, g])) * isum
            y[m, n] = acc + (Fraction(float(bias[n])) if bias is not None else 0)
    return y


@pytest.mark.parametrize("M,K,N", [(1, 64, 1), (3, 128, 2), (2, 192, 4)])
def test_linear_equals_exact_rational_arithmetic(M, K, N):
    rng = np.random.default_rng(M * 100 + N)
    cx = rng.integers(-8, 8, size=(M, K))
    cw = rng.integers(-8, 8, size=(N, K))
    sx = rng.random((M, K // 64)).astype(np.float32) + 0.01
    sw = rng.random((N, K // 64)).astype(np.float32) * 1e-3
    bias = rng.standard_normal(N).astype(np.float32)
    _, y64, T = oracle.int4_linear(pack(cx), sx, pack(cw), sw, bias)
    exact = _exact_linear(cx, sx, cw, sw, bias)
    for m in range(M):
        for n in range(N):
            assert abs(Fraction(y64[m, n]) - exact[m, n]) <= Fraction(1e-14) * Fraction(T[m, n] + 1)


def test_linear_closed_form_all_ones():
    M, K, N = 2, 256, 3
    ones = np.ones((M, K), np.int64)
    y, y64, _ = oracle.int4_linear(pack(ones), np.ones((M, K // 64), np.float32),
                                   pack(np.ones((N, K), np.int64)),
                                   np.ones((N, K // 64), np.float32))
    assert np.all(y64 == K)
    assert np.all(oracle.bf16_bits_to_f64(y) == K)


def test_linear_equals_numpy_matmul_of_dequantized_operands():
    rng = np.random.default_rng(7)
    M, K, N = 9, 320, 11
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq, xs = oracle.int4_quantize(bf16(x))
    wq, ws = oracle.int4_quantize(bf16(w))
    _, y64, T = oracle.int4_linear(xq, xs, wq, ws)
    xd = unpack(xq) * np.repeat(xs.astype(np.float64), 64, axis=1)
    wd = unpack(wq) * np.repeat(ws.astype(np.float64), 64, axis=1)
    ref = xd @ wd.T
    assert np.all(np.abs(y64 - ref) <= 1e-12 * T + 1e-300)
    # and the 4-bit result is a plausible approximation of the unquantized product
    full = bf16(x).double().numpy() @ bf16(w).double().numpy().T
    assert np.linalg.norm(y64 - full) / np.linalg.norm(full) < 0.3


def _expand(tokens, conv):
    out = []
    for t in tokens:
        if "*" in t:
            v, n = t.split("*")
            out += [conv(v)] * int(n)
        else:
            out.append(conv(t))
    return out


def test_hand_worked_groups_from_golden_file():
    """tests/golden/int4_worked_groups.txt: codes, scales and one output worked by hand."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "int4_worked_groups.txt")
    xs, fields = [], {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        key, *rest = line.split()
        if key == "x":
            xs += _expand(rest, float)
        else:
            fields[key] = rest
    assert len(xs) == 192
    x = torch.tensor([xs], dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(x.float(), torch.tensor([xs]))  # every value is exact in bf16
    q, s = oracle.int4_quantize(x)
    want_bytes = np.array(_expand(fields["bytes"], lambda v: int(v, 16)), np.uint8)
    np.testing.assert_array_equal(q[0], want_bytes)
    np.testing.assert_array_equal(s[0], np.array([float(v) for v in fields["scales"]], np.float32))
    y, y64, _ = oracle.int4_linear(q, s, q, s)
    assert y64[0, 0] == 251.5
    want_y = float(fields["y"][0])
    got = torch.tensor([int(y[0, 0])], dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    assert float(got.float()[0]) == want_y


def test_reciprocal_group_golden():
    """tests/golden/int4_reciprocal_group.txt: a group whose codes differ between
    x * RN32(1/scale) (the reading) and x / scale (a tie there), worked by exact
    arithmetic."""
    import os
    rows = {}
    path = os.path.join(os.path.dirname(__file__), "golden", "int4_reciprocal_group.txt")
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows[key] = [int(v, 16) for v in vals]
    b = np.array(rows["x_bits"], np.uint16)
    x = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).reshape(1, -1)
    q, s = oracle.int4_quantize(x)
    assert int(s.view(np.uint32)[0, 0]) == rows["scale_bits"][0]
    assert list(q[0]) == rows["bytes"]
