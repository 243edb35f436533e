"""Pins of the oracle's quantizers: a worked example derived by hand, and
invariants that any correct implementation of the stated rule must satisfy.

NVFP4 scheme: "BFL (fp8r / nvfp4)", scheme list, nvfp4 entry (packed E2M1, one
E4M3 scale per 16 elements, global fp32 scale). fp8r: same page, fp8r entry
(per-row E4M3 quantization of activations at run time).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from synthetic import make_linear_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def load_worked_block():
    xs, scales, rows = [], None, []
    g = y64 = ybits = None
    with open(os.path.join(GOLDEN, "nvfp4_worked_block.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "g":
                g = float(vals[0])
            elif key == "x":
                xs.extend(float(v) for v in vals)
            elif key == "scales":
                scales = [int(v, 16) for v in vals]
            elif key == "bytes":
                rows.extend(int(v, 16) for v in vals)
            elif key == "y64":
                y64 = float(vals[0])
            elif key == "ybits":
                ybits = int(vals[0], 16)
    return g, xs, scales, rows, y64, ybits


def test_nvfp4_worked_block_golden():
    g, xs, scales, codes, _, _ = load_worked_block()
    x = _bf16([xs])
    assert x.float().tolist()[0] == xs  # every input is exact in bf16
    q, s = oracle.nvfp4_quantize(x, g)
    assert list(s[0]) == scales
    assert list(q[0]) == codes


def test_nvfp4_worked_linear_golden():
    g, xs, scales, codes, y64_want, ybits = load_worked_block()
    q = np.array([codes], np.uint8)
    s = np.array([scales], np.uint8)
    y, y64, T = oracle.nvfp4_linear(q, s, q, s, g, g)
    assert abs(y64[0, 0] - y64_want) <= 1e-12 * y64_want
    assert int(y[0, 0]) == ybits
    assert T[0, 0] == pytest.approx(y64_want, rel=1e-12)  # all products are squares


def _representable_blocks(rng, R, K, g):
    """bf16 rows whose blocks are code * scale * g exactly, with a +-6 per block and
    normal, unsaturated scales, so that quantization must return those codes."""
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    nb = K // 16
    codes = rng.integers(0, 16, size=(R, K)).astype(np.uint8)
    pos6 = rng.integers(0, 16, size=(R, nb))
    for r in range(R):
        for b in range(nb):
            codes[r, b * 16 + pos6[r, b]] = 0x7 | (rng.integers(0, 2) << 3)
    # normal E4M3 scales, exponent field 1..14 (avoid 448-saturation at the top)
    sc = (rng.integers(1, 15, size=(R, nb)) << 3) | rng.integers(0, 8, size=(R, nb))
    sval = np.array([[oracle.e4m3_decode(int(c)) for c in row] for row in sc])
    val = mags[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    x = val * np.repeat(sval, 16, axis=1) * g
    return x, codes, sc.astype(np.uint8)


def _pack(codes):
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


@pytest.mark.parametrize("g", [2.0 ** -6, 2.0 ** -3, 1.0])
def test_nvfp4_representable_input_is_exact(g):
    rng = np.random.default_rng(3)
    x, codes, sc = _representable_blocks(rng, 8, 128, g)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(xb.double().numpy(), x)  # exact in bf16
    q, s = oracle.nvfp4_quantize(xb, g)
    assert np.array_equal(s, sc)
    # -0 codes (0x8) come back as +0 only if the value is zero; the generator can
    # produce code 0x8 (value -0.0), which bf16 keeps, so compare packed bytes.
    assert np.array_equal(q, _pack(codes))


def test_nvfp4_idempotent_on_normal_unsaturated_blocks():
    g = 2.0 ** -5
    inp = make_linear_inputs(16, 256, 1, seed=4)
    x = inp.x
    q1, s1 = oracle.nvfp4_quantize(x, g)
    ok = (s1 >= 0x08) & (s1 <= 0x7D)           # normal, below the saturating scale
    sf = np.abs(x.float().numpy()).reshape(16, 16, 16).max(-1) / np.float32(6 * g)
    ok &= sf < 440                              # the block scale did not saturate
    deq = oracle.nvfp4_dequantize(q1, s1) * g   # code * scale * g, exact in bf16 (g = 2^-5)
    xb2 = torch.from_numpy(deq).to(torch.bfloat16)
    assert np.array_equal(xb2.double().numpy(), deq)
    q2, s2 = oracle.nvfp4_quantize(xb2, g)
    assert ok.sum() > 200
    assert np.array_equal(s2[ok], s1[ok])
    okq = np.repeat(ok, 8, axis=1)
    assert np.array_equal(q2[okq], q1[okq])


def test_nvfp4_sign_symmetry_and_zero_block():
    inp = make_linear_inputs(8, 256, 1, seed=5)
    g = oracle.nvfp4_global_scale(inp.x)
    q, s = oracle.nvfp4_quantize(inp.x, g)
    qn, sn = oracle.nvfp4_quantize(-inp.x, g)
    assert np.array_equal(s, sn)
    assert np.array_equal(qn, q ^ 0x88)        # every nibble's sign bit flips
    z = torch.zeros(2, 32, dtype=torch.bfloat16)
    z[1, 3] = -0.0
    qz, sz = oracle.nvfp4_quantize(z, g)
    assert not qz.any() and not sz.any()


def test_nvfp4_block_whose_scale_rounds_to_zero_encodes_zeros():
    # tiny values of either sign: the block scale rounds to E4M3 zero, so d = 0 and the
    # whole block is encoded as +0 codes (no -0 nibbles)
    x = torch.full((1, 32), -(2.0 ** -30), dtype=torch.bfloat16)
    x[0, 1::2] = 2.0 ** -31
    x[0, 16:] = 1.0                             # the second block is ordinary
    q, s = oracle.nvfp4_quantize(x, 1.0)
    assert s[0, 0] == 0 and s[0, 1] != 0
    assert not q[0, :8].any()
    assert q[0, 8:].all()


def test_nvfp4_saturation_when_input_scale_too_small():
    inp = make_linear_inputs(4, 256, 1, seed=6)
    g = oracle.nvfp4_global_scale(inp.x) / 4   # activations exceed the calibration
    q, s = oracle.nvfp4_quantize(inp.x, g)
    assert (s == 0x7E).any()
    nib = np.stack([q & 0xF, q >> 4], -1).reshape(4, 256)
    assert ((nib & 7) == 7).sum() > 0


def test_nvfp4_global_scale_rule():
    x = _bf16([[1.0, -2688.0, 3.0, 0.5] * 4])
    assert oracle.nvfp4_global_scale(x) == 1.0
    x = _bf16([[0.0] * 16])
    assert oracle.nvfp4_global_scale(x) == 0.0


def test_fp8r_quantize_invariants():
    inp = make_linear_inputs(32, 512, 1, seed=7)
    q, s = oracle.fp8r_quantize_rows(inp.x)
    xf = inp.x.float().numpy()
    amax = np.abs(xf).max(1)
    assert np.array_equal(s, (amax / np.float32(448)).astype(np.float32))
    # the row maximum maps to +-448 (within one E4M3 step) and nothing exceeds it
    vals = np.vectorize(oracle.e4m3_decode)(q)
    assert np.all(np.abs(vals).max(1) >= 416) and np.all(np.abs(vals) <= 448)
    qn, sn = oracle.fp8r_quantize_rows(-inp.x)
    assert np.array_equal(sn, s) and np.array_equal(qn, q ^ 0x80)
    # zero row -> zero scale and zero codes
    z = torch.zeros(2, 64, dtype=torch.bfloat16)
    qz, sz = oracle.fp8r_quantize_rows(z)
    assert not qz.any() and not sz.any()


def test_fp8r_representable_rows_are_exact():
    # rows x = code * (amax/448) where the row max is code 0x7E (448) and the scale
    # amax/448 is a power of two: quantization returns the codes.
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 0x7F, size=(6, 64)).astype(np.uint8)
    codes = np.where(codes == 0x7F, 0x7E, codes)
    codes[:, 5] = 0x7E
    codes |= (rng.integers(0, 2, size=codes.shape) << 7).astype(np.uint8)
    scale = 2.0 ** -rng.integers(2, 10, size=(6, 1))
    vals = np.vectorize(oracle.e4m3_decode)(codes) * scale
    xb = torch.from_numpy(vals).to(torch.bfloat16)
    assert np.array_equal(xb.double().numpy(), vals)
    q, s = oracle.fp8r_quantize_rows(xb)
    assert np.array_equal(s, scale[:, 0].astype(np.float32))
    # codes 0x80 (-0) and 0x00 decode to the same zero: compare values
    assert np.array_equal(np.vectorize(oracle.e4m3_decode)(q), vals / scale)


def test_fp8r_worked_row_golden():
    # one row worked by exact rational arithmetic (the fixture's header): the scale bits,
    # the reciprocal-multiply reading (it differs from a division on four elements), a
    # subnormal code, zero and a negative value
    rows = {}
    with open(os.path.join(GOLDEN, "fp8r_worked_row.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows[key] = [int(v, 16) for v in vals]
    bits = np.array(rows["x_bits"], np.uint16)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).reshape(1, -1)
    q, s = oracle.fp8r_quantize_rows(x)
    assert int(s.view(np.uint32)[0]) == rows["scale_bits"][0]
    assert list(q[0]) == rows["codes"]


def _golden_hex(name):
    rows = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows[key] = [int(v, 16) for v in vals]
    return rows


def _bf16_row(bits):
    b = np.array(bits, np.uint16)
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).reshape(1, -1)


def test_nvfp4_reciprocal_block_golden():
    # a block worked by exact arithmetic whose codes differ on five elements between
    # x * RN32(1/d) (the reading) and x / d (ties there)
    rows = _golden_hex("nvfp4_reciprocal_block.txt")
    g = float(np.array(rows["g_bits"], np.uint32).view(np.float32)[0])
    q, s = oracle.nvfp4_quantize(_bf16_row(rows["x_bits"]), g)
    assert list(s[0]) == rows["scales"]
    assert list(q[0]) == rows["bytes"]


def test_nvfp4_scale_constant_rounding_order_golden():
    rows = {}
    with open(os.path.join(GOLDEN, "nvfp4_rounding_order.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows[key] = vals
    g = float(np.array([int(rows["g_bits"][0], 16)], np.uint32).view(np.float32)[0])
    x = _bf16([[float(v) for v in rows["x"]]])
    q, s = oracle.nvfp4_quantize(x, g)
    assert list(s[0]) == [int(v, 16) for v in rows["scales"]]
    assert list(q[0]) == [int(v, 16) for v in rows["bytes"]]
