"""Pins of the oracle's element formats against sources other than itself.

* E2M1 / E4M3 grids: golden tables from the OCP format definitions
  (tests/golden/*.txt) and, for E4M3, PyTorch's float8_e4m3fn decode.
* Encoders: exact-midpoint ties and saturation (golden), round trips, sign
  symmetry, monotonicity, PyTorch's RN cast (E4M3, in range) and an exhaustive
  nearest-value brute force in numpy (E2M1).
* bf16 rounding: PyTorch's fp32 -> bf16 cast on fp32-exact inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def test_e2m1_grid_golden():
    rows = list(_rows("e2m1_grid.txt"))
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1_decode(int(code, 16))
        want = float(val)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got, want)


def test_e4m3_special_golden():
    for code, val in _rows("e4m3_special.txt"):
        got = oracle.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got), code
        else:
            want = float(val)
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got)


def test_e4m3_all_256_vs_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if c in (0x7F, 0xFF):
            assert math.isnan(got) and math.isnan(ref[c])
        else:
            assert got == ref[c], (hex(c), got, ref[c])


def test_e4m3_ascending_and_extremes():
    vals = [oracle.e4m3_decode(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    assert vals[-1] == 448.0 and vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6


def test_rounding_ties_and_saturation_golden():
    for fmt, v, code in _rows("rounding_ties.txt"):
        enc = oracle.e2m1_encode if fmt == "e2m1" else oracle.e4m3_encode
        got = int(enc(np.array([float(v)], np.float32))[0])
        assert got == int(code, 16), (fmt, v, hex(got), code)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_round_trip_every_code(fmt):
    if fmt == "e2m1":
        codes = range(16)
        dec, enc = oracle.e2m1_decode, oracle.e2m1_encode
    else:
        codes = [c for c in range(256) if c not in (0x7F, 0xFF)]
        dec, enc = oracle.e4m3_decode, oracle.e4m3_encode
    vals = np.array([dec(c) for c in codes], np.float32)
    got = enc(vals)
    assert list(got) == list(codes)


def test_e4m3_encoder_vs_torch_cast_in_range():
    # torch's float -> float8_e4m3fn cast rounds to nearest-even; it does not
    # saturate, so only |v| <= 448 is compared. Every fp32 bit pattern from
    # 2^-12 to 448 with a stride co-prime to the mantissa width, plus all exact
    # midpoints between neighbouring codes and their fp32 neighbours.
    lo = np.float32(2.0 ** -12).view(np.uint32)
    hi = np.float32(448.0).view(np.uint32)
    bits = np.arange(lo, hi + 1, 97, dtype=np.uint32)
    grid = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    v = np.concatenate([bits.view(np.float32), extra]).astype(np.float32)
    v = np.concatenate([v, -v])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


def _e2m1_bruteforce(v):
    """Nearest of the 8 magnitudes by full distance table; ties to the even code;
    saturating at 6; sign kept."""
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[:, None] - mags[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among tied candidates prefer the even code
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    pick = np.where(a >= 6, 7, pick)
    return (pick | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def test_e2m1_encoder_vs_bruteforce_sweep():
    lo = np.float32(2.0 ** -8).view(np.uint32)
    hi = np.float32(16.0).view(np.uint32)
    bits = np.arange(lo, hi, 31, dtype=np.uint32)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = (mags[:-1] + mags[1:]) / 2
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(9))])
    v = np.concatenate([bits.view(np.float32), extra, np.float32([0.0, 1e-30, 1e30])])
    v = np.concatenate([v, -v]).astype(np.float32)
    got = oracle.e2m1_encode(v)
    ref = _e2m1_bruteforce(v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_encoder_monotone_and_sign_symmetric(fmt):
    rng = np.random.default_rng(1)
    v = np.sort(np.concatenate([rng.uniform(0, 8 if fmt == "e2m1" else 500, 200000),
                                rng.lognormal(-4, 3, 50000)])).astype(np.float32)
    enc = oracle.e2m1_encode if fmt == "e2m1" else oracle.e4m3_encode
    dec = oracle.e2m1_decode if fmt == "e2m1" else oracle.e4m3_decode
    pos = enc(v)
    neg = enc(-v)
    signbit = 0x8 if fmt == "e2m1" else 0x80
    assert np.all(neg == (pos | signbit))
    vals = np.array([dec(int(c)) for c in np.unique(pos)])
    decoded = np.interp(pos, np.unique(pos), vals)  # value of each code
    assert np.all(np.diff(decoded) >= 0)


def test_bf16_from_double_vs_torch_on_fp32_inputs():
    # For inputs exactly representable in fp32 one rounding from fp64 equals
    # torch's fp32 -> bf16 RN cast.
    rng = np.random.default_rng(2)
    f = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(1000),
        rng.lognormal(0, 20, 100000).astype(np.float32),
        np.float32([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3e38, -3e38, 1e-39, -1e-40]),
    ])
    f = f[np.isfinite(f)]
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_from_double(f.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(f[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


def test_bf16_from_double_single_rounding():
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7 -> ties to even (1.0);
    # 1 + 2^-8 + 2^-40 is above it -> 1 + 2^-7. A double-rounding path through
    # fp32 would give 1.0 for the second one.
    got = oracle.bf16_from_double(np.array([1 + 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40,
                                            -(1 + 3 * 2.0 ** -8)]))
    assert list(got) == [0x3F80, 0x3F81, 0xBF82]


def test_bf16_from_double_subnormals_vs_torch():
    # the fp32 subnormal range, where bf16 keeps a quantum of 2^-133: one rounding from
    # fp64 equals torch's fp32 -> bf16 round-to-nearest-even cast
    pos = np.arange(1, 0x800000, 13, dtype=np.uint32)
    f = np.concatenate([pos, pos | np.uint32(0x80000000)]).view(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_from_double(f.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(f[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


def test_e4m3_encode_nan_is_a_nan_code():
    # E4M3 (OCP) has no infinity; its NaN is S.1111.111
    codes = oracle.e4m3_encode(np.float32([np.nan, -np.nan]))
    assert all(c & 0x7F == 0x7F for c in codes)
    assert all(np.isnan(oracle.e4m3_decode(int(c))) for c in codes)
