"""Checks that the oracle's pins catch plausible mistakes (test infrastructure; it is
not collected by pytest).

For each planted mistake the script copies oracle/, synthetic/, the oracle's pin tests
and their fixtures into a temporary directory, replaces one fragment of the copy's
oracle.cpp, builds the copy and runs the pins there. The repository is not modified.

    python tests/plant_mistakes.py              # every mistake
    python tests/plant_mistakes.py INT4 fp8r    # those whose name contains a word

A mistake is caught when at least one pin fails. Three are marked equivalent: they give
the same result on every input the path produces, so every pin passes. They are:
  - INT4 clamp at -7: the rule never yields -8, since |x * RN32(1/scale)| <= 7 (1 + 2^-23);
  - INT4 tolerance without |scale|: the group scales are never negative;
  - bf16 overflow tested with > instead of >=: the fp32 conversion of 2^128 is already
    infinite.
The exit status is 1 if a mistake that should be caught passes, if an equivalent one is
caught, or if a fragment is no longer found in oracle.cpp.
"""
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_TESTS = ["test_oracle_formats.py", "test_oracle_quant.py", "test_oracle_linear.py",
             "test_oracle_gelu.py", "test_oracle_svdq.py", "test_oracle_w4a16.py",
             "test_oracle_int4.py"]

# (name, fragment of oracle/oracle.cpp, the mistaken fragment, equivalent)
MISTAKES = [
    ('NVFP4 codes from x / d',
     'codes[i] = oracle_e2m1_encode(v[i] * inv);',
     'codes[i] = oracle_e2m1_encode(v[i] / d); (void)inv;',
     False),
    ('NVFP4 c = RN32(RN32(1/6) / g)',
     'const float c = 1.0f / (6.0f * g);',
     'const float c = (1.0f / 6.0f) / g;',
     False),
    ('NVFP4 d without g',
     'float d = (float)oracle_e4m3_decode(sc) * g;',
     'float d = (float)oracle_e4m3_decode(sc);',
     False),
    ('NVFP4 nibbles swapped',
     'qb[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));',
     'qb[j] = (uint8_t)((codes[2 * j + 1] & 0xF) | ((codes[2 * j] & 0xF) << 4));',
     False),
    ('global scale amax / 448',
     'return amax / 2688.0f;',
     'return amax / 448.0f;',
     False),
    ('dequantization scale index k / 32',
     'oracle_e4m3_decode(s[r * (K / 16) + k / 16]);\n    }',
     'oracle_e4m3_decode(s[r * (K / 16) + k / 32]);\n    }',
     False),
    ('alpha without the weight scale',
     'double alpha = alpha_m[m] * alpha_n[n];',
     'double alpha = alpha_m[m];',
     False),
    ('tolerance sum without absolute values',
     'absacc += std::fabs(p);',
     'absacc += p;',
     False),
    ('bias added before the scale',
     'double v = alpha * acc + (bias ? (double)bias[n] : 0.0);',
     'double v = alpha * (acc + (bias ? (double)bias[n] : 0.0));',
     False),
    ('fp8r scale amax / 240',
     'float sc = amax / 448.0f;',
     'float sc = amax / 240.0f;',
     False),
    ('W4A16 without the fp32 rounding',
     'const float w32 = (float)exact;  // one RN to fp32\n      out[r * K + k] = oracle_bf16_from_double((double)w32);',
     'out[r * K + k] = oracle_bf16_from_double(exact);',
     False),
    ('W4A16 without weight_scale_2',
     '*\n                           (double)weight_scale_2;',
     '*\n                           1.0;',
     False),
    ('INT4 scale amax / 8',
     'const float sc = amax / 7.0f;',
     'const float sc = amax / 8.0f;',
     False),
    ('INT4 truncation',
     'double rq = std::nearbyint(static_cast<double>(t));',
     'double rq = std::trunc(static_cast<double>(t));',
     False),
    ('INT4 round half away from zero',
     'double rq = std::nearbyint(static_cast<double>(t));',
     'double rq = std::round(static_cast<double>(t));',
     False),
    ('INT4 clamp at -7',
     'if (rq < -8.0) rq = -8.0;',
     'if (rq < -7.0) rq = -7.0;',
     True),
    ('INT4 codes from x / scale',
     'const float t = bf16_to_float(xg[i + e]) * inv;',
     'const float t = bf16_to_float(xg[i + e]) / sc;',
     False),
    ('INT4 nibble sign extension by 8',
     'return nib >= 8 ? nib - 16 : nib;',
     'return nib >= 8 ? nib - 8 : nib;',
     False),
    ('INT4 tolerance without |scale|',
     'absacc += std::fabs(sc) * static_cast<double>(iabs);',
     'absacc += sc * static_cast<double>(iabs);',
     True),
    ('element ties to odd',
     'return (lo % 2 == 0) ? lo : hi;',
     'return (lo % 2 == 0) ? hi : lo;',
     False),
    ('bf16 truncation',
     'double r = std::nearbyint(a / q) * q;',
     'double r = std::floor(a / q) * q;',
     False),
    ('GELU with erfc(+v/sqrt2)',
     'return 0.5 * v * std::erfc(-v / std::sqrt(2.0));',
     'return 0.5 * v * std::erfc(v / std::sqrt(2.0));',
     False),
    ('smoothing rounded once',
     'out[m * K + k] = oracle_bf16_from_double(static_cast<double>(p));',
     'out[m * K + k] = oracle_bf16_from_double(static_cast<double>(bf16_to_float(x[m * K + k])) * smooth[k]);',
     False),
    ('low-rank down transposed',
     'static_cast<double>(bf16_to_float(down[j * K + k]));',
     'static_cast<double>(bf16_to_float(down[k * r + j]));',
     False),
    ('E4M3 subnormal exponent',
     'if (e == 0) mag = std::ldexp((double)m, -9);',
     'if (e == 0) mag = std::ldexp((double)m, -10);',
     False),
    ('E2M1 subnormal value',
     'double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + m / 2.0, e - 1);',
     'double mag = (e == 0) ? 1.0 * m : std::ldexp(1.0 + m / 2.0, e - 1);',
     False),
    ('low-rank term scaled by alpha',
     'const double v = main64[m * N + n] + lr + (bias ? static_cast<double>(bias[n]) : 0.0);',
     'const double v = main64[m * N + n] + (double)input_scale * weight_scale_2 * lr + (bias ? static_cast<double>(bias[n]) : 0.0);',
     False),
    ('low-rank up transposed',
     'D[m * r + j] * static_cast<double>(bf16_to_float(up[n * r + j]));',
     'D[m * r + j] * static_cast<double>(bf16_to_float(up[j * N + n]));',
     False),
    ('SVDQuant bias dropped',
     'const double v = main64[m * N + n] + lr + (bias ? static_cast<double>(bias[n]) : 0.0);',
     'const double v = main64[m * N + n] + lr;',
     False),
    ('low-rank D accumulated in fp32',
     '      double acc = 0.0;\n      for (int64_t k = 0; k < K; ++k)\n        acc += static_cast<double>(bf16_to_float(xs[m * K + k])) *',
     '      float acc = 0.0f;\n      for (int64_t k = 0; k < K; ++k)\n        acc += static_cast<float>(bf16_to_float(xs[m * K + k])) *',
     False),
    ('NVFP4 block amax over 8 elements',
     '      for (int i = 0; i < 16; ++i) {\n        v[i] = bf16_to_float(xb[i]);\n        float a = std::fabs(v[i]);\n        if (a > amax) amax = a;',
     '      for (int i = 0; i < 16; ++i) {\n        v[i] = bf16_to_float(xb[i]);\n        float a = std::fabs(v[i]);\n        if (i < 8 && a > amax) amax = a;',
     False),
    ('global scale from the signed max',
     'float a = std::fabs(bf16_to_float(x[i]));\n    if (a > amax) amax = a;\n  }\n  return amax / 2688.0f;',
     'float a = bf16_to_float(x[i]);\n    if (a > amax) amax = a;\n  }\n  return amax / 2688.0f;',
     False),
    ('GELU factor',
     'return 0.5 * v * std::erfc(-v / std::sqrt(2.0));',
     'return v * std::erfc(-v / std::sqrt(2.0)) / 2.0000001;',
     False),
    ('GELU band without v^2',
     'const double rel_tol = tol_const + tol_sq * v * v;',
     'const double rel_tol = tol_const;',
     False),
    ('GELU band neighbour on the wrong side',
     'if (g > vb) other = (b & 0x8000) ? (b == 0x8000 ? 0x0001 : b - 1) : b + 1;',
     'if (g < vb) other = (b & 0x8000) ? (b == 0x8000 ? 0x0001 : b - 1) : b + 1;',
     False),
    ('bf16 subnormal quantum 2^-134',
     'q = std::ldexp(1.0, -133);',
     'q = std::ldexp(1.0, -134);',
     False),
    ('bf16 overflow test > instead of >=',
     'if (r >= std::ldexp(1.0, 128)) return sign | 0x7F80;',
     'if (r > std::ldexp(1.0, 128)) return sign | 0x7F80;',
     True),
    ('NaN encoded as 448',
     'if (std::isnan(v)) return 0x7F;',
     'if (std::isnan(v)) return 0x7E;',
     False),
    ('E2M1 sign from v < 0',
     'uint8_t sign = std::signbit(v) ? 0x8 : 0x0;',
     'uint8_t sign = (v < 0) ? 0x8 : 0x0;',
     False),
    ('fp8r scales on the wrong operand',
     'for (int64_t m = 0; m < M; ++m) am[m] = (double)xs[m];\n  for (int64_t n = 0; n < N; ++n) an[n] = (double)ws[n];',
     'for (int64_t m = 0; m < M; ++m) am[m] = (double)ws[m % N];\n  for (int64_t n = 0; n < N; ++n) an[n] = (double)xs[n % M];',
     False),
    ('W4A16 bias dropped',
     'std::vector<double> am((size_t)M, 1.0), an((size_t)N, 1.0);\n  contract(A.data(), B.data(), M, K, N, am.data(), an.data(), bias, y, y64, T);',
     'std::vector<double> am((size_t)M, 1.0), an((size_t)N, 1.0);\n  contract(A.data(), B.data(), M, K, N, am.data(), an.data(), nullptr, y, y64, T);',
     False),
    ('INT4 group scale index',
     'const double sc = static_cast<double>(xs[m * G + g]) * static_cast<double>(ws[n * G + g]);',
     'const double sc = static_cast<double>(xs[m * G + g]) * static_cast<double>(ws[n * G + (G - 1 - g)]);',
     False),
    ('INT4 bias dropped',
     'const double v = acc + (bias ? static_cast<double>(bias[n]) : 0.0);',
     'const double v = acc;',
     False),
    ('fp8r zero row as -0 codes',
     'for (int64_t k = 0; k < K; ++k) q[r * K + k] = 0;',
     'for (int64_t k = 0; k < K; ++k) q[r * K + k] = 0x80;',
     False),
    ('NVFP4 zero-scale block keeps -0',
     'for (int i = 0; i < 16; ++i) codes[i] = 0;',
     'for (int i = 0; i < 16; ++i) codes[i] = (v[i] < 0) ? 8 : 0;',
     False),
    ('INT4 code 8 read as +8',
     'return nib >= 8 ? nib - 16 : nib;',
     'return nib > 8 ? nib - 16 : nib;',
     False),
    ('fp8r codes from x / scale',
     'for (int64_t k = 0; k < K; ++k) q[r * K + k] = oracle_e4m3_encode(bf16_to_float(xr[k]) * inv);',
     'for (int64_t k = 0; k < K; ++k) q[r * K + k] = oracle_e4m3_encode(bf16_to_float(xr[k]) / sc); (void)inv;',
     False),
]


def copy_tree(dst):
    for pkg in ("oracle", "synthetic"):
        shutil.copytree(os.path.join(ROOT, pkg), os.path.join(dst, pkg),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    for f in PIN_TESTS + ["conftest.py"]:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))


def plant(name, old, new):
    """Returns 'caught', 'passed', 'missing' (fragment not found) or 'build failed'."""
    src = open(os.path.join(ROOT, "oracle", "oracle.cpp")).read()
    if src.count(old) != 1:
        return "missing", ""
    with tempfile.TemporaryDirectory() as tmp:
        copy_tree(tmp)
        with open(os.path.join(tmp, "oracle", "oracle.cpp"), "w") as f:
            f.write(src.replace(old, new))
        b = subprocess.run([sys.executable, "-c", "from oracle import build; build.build(True)"],
                           cwd=tmp, capture_output=True, text=True)
        if b.returncode != 0:
            return "build failed", b.stderr[-300:]
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider"]
                           + [os.path.join("tests", f) for f in PIN_TESTS],
                           cwd=tmp, capture_output=True, text=True, timeout=1800)
        failed = [l for l in r.stdout.splitlines() if l.startswith("FAILED")]
        return ("caught" if r.returncode != 0 else "passed"), (failed[0] if failed else "")


def main(words):
    bad = 0
    for name, old, new, equivalent in MISTAKES:
        if words and not any(w in name for w in words):
            continue
        outcome, detail = plant(name, old, new)
        ok = outcome == ("passed" if equivalent else "caught")
        bad += not ok
        tag = "ok " if ok else "BAD"
        print(f"{tag} {name}: {outcome}{' (equivalent)' if equivalent else ''}  {detail}",
              flush=True)
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
