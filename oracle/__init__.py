"""Python face of the plain CPU oracle (numpy in, numpy out).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the benchmark's CPU-baseline / reference leg, never by the product
package. It shares no code with the CUDA path. Arithmetic lives in
``oracle.cpp``; this module only marshals arguments.

bf16 tensors are passed as their raw uint16 bit patterns.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        u8p, u16p, f32p, f64p = (C.POINTER(C.c_uint8), C.POINTER(C.c_uint16),
                                  C.POINTER(C.c_float), C.POINTER(C.c_double))
        i64 = C.c_int64
        L.oracle_set_threads.argtypes = [C.c_int]
        L.oracle_get_threads.restype = C.c_int
        L.oracle_e4m3_decode.argtypes = [C.c_uint8]
        L.oracle_e4m3_decode.restype = C.c_double
        L.oracle_e2m1_decode.argtypes = [C.c_uint8]
        L.oracle_e2m1_decode.restype = C.c_double
        L.oracle_e4m3_encode.argtypes = [C.c_float]
        L.oracle_e4m3_encode.restype = C.c_uint8
        L.oracle_e2m1_encode.argtypes = [C.c_float]
        L.oracle_e2m1_encode.restype = C.c_uint8
        L.oracle_e4m3_encode_array.argtypes = [f32p, i64, u8p]
        L.oracle_e2m1_encode_array.argtypes = [f32p, i64, u8p]
        L.oracle_e4m3_encode_bits_range.argtypes = [C.c_uint32, i64, u8p]
        L.oracle_e2m1_encode_bits_range.argtypes = [C.c_uint32, i64, u8p]
        L.oracle_bf16_from_double.argtypes = [C.c_double]
        L.oracle_bf16_from_double.restype = C.c_uint16
        L.oracle_bf16_from_double_array.argtypes = [f64p, i64, u16p]
        L.oracle_gelu.argtypes = [C.c_double]
        L.oracle_gelu.restype = C.c_double
        L.oracle_gelu_bf16.argtypes = [u16p, i64, C.c_double, C.c_double, u16p, u8p]
        L.oracle_smooth_bf16.argtypes = [u16p, i64, i64, f32p, u16p]
        L.oracle_lowrank_down.argtypes = [u16p, i64, i64, u16p, i64, f64p]
        L.oracle_svdq_nvfp4_linear.argtypes = [u8p, u8p, i64, i64, u8p, u8p, i64, C.c_float,
                                               C.c_float, f64p, u16p, i64, f32p, u16p, f64p,
                                               f64p, f64p]
        L.oracle_svdq_nvfp4_linear.restype = C.c_int
        L.oracle_nvfp4_global_scale.argtypes = [u16p, i64]
        L.oracle_nvfp4_global_scale.restype = C.c_float
        L.oracle_nvfp4_quantize.argtypes = [u16p, i64, i64, C.c_float, u8p, u8p]
        L.oracle_nvfp4_quantize.restype = C.c_int
        L.oracle_nvfp4_dequantize.argtypes = [u8p, u8p, i64, i64, f64p]
        L.oracle_nvfp4_dequantize.restype = C.c_int
        L.oracle_nvfp4_linear.argtypes = [u8p, u8p, i64, i64, u8p, u8p, i64, C.c_float,
                                          C.c_float, f32p, u16p, f64p, f64p]
        L.oracle_nvfp4_linear.restype = C.c_int
        L.oracle_nvfp4_linear_unquantized_act.argtypes = [u16p, i64, i64, u8p, u8p, i64,
                                                          C.c_float, f32p, f64p]
        L.oracle_nvfp4_linear_unquantized_act.restype = C.c_int
        L.oracle_fp8r_quantize_rows.argtypes = [u16p, i64, i64, u8p, f32p]
        L.oracle_fp8r_quantize_rows.restype = C.c_int
        L.oracle_fp8r_linear.argtypes = [u8p, f32p, i64, i64, u8p, f32p, i64, f32p,
                                         u16p, f64p, f64p]
        L.oracle_fp8r_linear.restype = C.c_int
        L.oracle_w4a16_dequantize_bf16.argtypes = [u8p, u8p, i64, i64, C.c_float, u16p]
        L.oracle_w4a16_dequantize_bf16.restype = C.c_int
        L.oracle_w4a16_linear.argtypes = [u16p, i64, i64, u8p, u8p, i64, C.c_float, f32p, u16p,
                                          f64p, f64p]
        L.oracle_w4a16_linear.restype = C.c_int
        L.oracle_int4_quantize.argtypes = [u16p, i64, i64, u8p, f32p]
        L.oracle_int4_quantize.restype = C.c_int
        L.oracle_int4_linear.argtypes = [u8p, f32p, i64, i64, u8p, f32p, i64, f32p, u16p, f64p,
                                         f64p]
        L.oracle_int4_linear.restype = C.c_int
        _lib = L
    return _lib


def _p(a, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(C.POINTER(ctype))


def _bits16(x):
    """bf16 data as a contiguous uint16 numpy array (accepts torch bf16 or uint16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.uint16)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


def e4m3_decode(code: int) -> float:
    return float(lib().oracle_e4m3_decode(code & 0xFF))


def e2m1_decode(nibble: int) -> float:
    return float(lib().oracle_e2m1_decode(nibble & 0xF))


def e4m3_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_p(v, C.c_float), v.size, _p(out, C.c_uint8))
    return out


def e2m1_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_p(v, C.c_float), v.size, _p(out, C.c_uint8))
    return out


def e4m3_encode_bits_range(first: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint8)
    lib().oracle_e4m3_encode_bits_range(first, count, _p(out, C.c_uint8))
    return out


def e2m1_encode_bits_range(first: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint8)
    lib().oracle_e2m1_encode_bits_range(first, count, _p(out, C.c_uint8))
    return out


def bf16_from_double(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().oracle_bf16_from_double_array(_p(v, C.c_double), v.size, _p(out, C.c_uint16))
    return out


def gelu(v: float) -> float:
    """Exact GELU v * Phi(v) in fp64 (oracle_gelu)."""
    return lib().oracle_gelu(float(v))


def gelu_bf16(y, rel_tol: float = 2.0 ** -20, rel_tol_sq: float = 2.0 ** -22):
    """bf16(GELU(y)) of a bf16 tensor (torch bf16 or uint16 bits), in fp64, plus the
    mask of elements whose exact GELU lies within (rel_tol + rel_tol_sq * y^2) * |value|
    of a bf16 rounding midpoint (where an fp32 evaluation may round the other way).
    The defaults bound an fp32 evaluation 0.5 v * erfcf(-v * RN(1/sqrt 2)) with erfcf
    within 4 ulp: (v^2 + |v| + 6) fp32 ulps, doubled."""
    bits = _bits16(y)
    h = np.empty(bits.shape, dtype=np.uint16)
    amb = np.empty(bits.shape, dtype=np.uint8)
    lib().oracle_gelu_bf16(_p(bits, C.c_uint16), bits.size, float(rel_tol), float(rel_tol_sq),
                           _p(h, C.c_uint16), _p(amb, C.c_uint8))
    return h, amb.astype(bool)


def smooth_bf16(x, smooth) -> np.ndarray:
    """bf16(RN32(x * smooth)) per element, smooth fp32 [K] over the last axis (uint16 bits)."""
    bits = _bits16(x)
    M, K = bits.shape
    sm = np.ascontiguousarray(smooth, dtype=np.float32)
    assert sm.shape == (K,)
    out = np.empty_like(bits)
    lib().oracle_smooth_bf16(_p(bits, C.c_uint16), M, K, _p(sm, C.c_float), _p(out, C.c_uint16))
    return out


def lowrank_down(xs, down) -> np.ndarray:
    """D = xs @ down^T exactly (fp64); xs bf16 [M, K], down bf16 [r, K]."""
    a, b = _bits16(xs), _bits16(down)
    M, K = a.shape
    r = b.shape[0]
    assert b.shape == (r, K)
    D = np.empty((M, r), dtype=np.float64)
    lib().oracle_lowrank_down(_p(a, C.c_uint16), M, K, _p(b, C.c_uint16), r, _p(D, C.c_double))
    return D


def svdq_nvfp4_linear(xq, xs, wq, ws, input_scale, weight_scale_2, D, up, bias=None):
    """SVDQuant-style NVFP4 linear: (y bf16 bits, y64, T, T_lr), see oracle.cpp."""
    M, K = xq.shape[0], xq.shape[1] * 2
    N = wq.shape[0]
    D = np.ascontiguousarray(D, dtype=np.float64)
    upb = _bits16(up)
    r = D.shape[1]
    assert upb.shape == (N, r)
    y = np.empty((M, N), dtype=np.uint16)
    y64, T, Tlr = (np.empty((M, N)) for _ in range(3))
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    rc = lib().oracle_svdq_nvfp4_linear(
        _p(np.ascontiguousarray(xq), C.c_uint8), _p(np.ascontiguousarray(xs), C.c_uint8), M, K,
        _p(np.ascontiguousarray(wq), C.c_uint8), _p(np.ascontiguousarray(ws), C.c_uint8), N,
        float(input_scale), float(weight_scale_2), _p(D, C.c_double), _p(upb, C.c_uint16), r,
        _p(b, C.c_float), _p(y, C.c_uint16), _p(y64, C.c_double), _p(T, C.c_double),
        _p(Tlr, C.c_double))
    assert rc == 0
    return y, y64, T, Tlr


def nvfp4_global_scale(x) -> float:
    """Calibration rule of the workloads: amax / (6 * 448), fp32."""
    xb = _bits16(x)
    return float(lib().oracle_nvfp4_global_scale(_p(xb, C.c_uint16), xb.size))


def nvfp4_quantize(x, g: float):
    """bf16 [R, K] -> (codes uint8 [R, K/2], block scales uint8 [R, K/16])."""
    xb = _bits16(x)
    R, K = xb.shape
    q = np.empty((R, K // 2), np.uint8)
    s = np.empty((R, K // 16), np.uint8)
    rc = lib().oracle_nvfp4_quantize(_p(xb, C.c_uint16), R, K, np.float32(g),
                                     _p(q, C.c_uint8), _p(s, C.c_uint8))
    if rc != 0:
        raise ValueError(f"oracle_nvfp4_quantize: bad shape {xb.shape}")
    return q, s


def nvfp4_dequantize(q, s) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    R, K = q.shape[0], q.shape[1] * 2
    out = np.empty((R, K), np.float64)
    lib().oracle_nvfp4_dequantize(_p(q, C.c_uint8), _p(s, C.c_uint8), R, K, _p(out, C.c_double))
    return out


def nvfp4_linear(xq, xs, wq, ws, input_scale, weight_scale_2, bias=None):
    """Returns (y bf16 bits uint16 [M,N], y fp64 [M,N], tolerance scale T fp64 [M,N])."""
    xq = np.ascontiguousarray(xq, np.uint8)
    xs = np.ascontiguousarray(xs, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    ws = np.ascontiguousarray(ws, np.uint8)
    M, K = xq.shape[0], xq.shape[1] * 2
    N = wq.shape[0]
    assert wq.shape[1] * 2 == K and xs.shape == (M, K // 16) and ws.shape == (N, K // 16)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    y = np.empty((M, N), np.uint16)
    y64 = np.empty((M, N), np.float64)
    T = np.empty((M, N), np.float64)
    rc = lib().oracle_nvfp4_linear(_p(xq, C.c_uint8), _p(xs, C.c_uint8), M, K,
                                   _p(wq, C.c_uint8), _p(ws, C.c_uint8), N,
                                   np.float32(input_scale), np.float32(weight_scale_2),
                                   _p(b, C.c_float), _p(y, C.c_uint16), _p(y64, C.c_double),
                                   _p(T, C.c_double))
    if rc != 0:
        raise ValueError("oracle_nvfp4_linear: bad shape")
    return y, y64, T


def nvfp4_linear_unquantized_act(x, wq, ws, weight_scale_2, bias=None):
    xb = _bits16(x)
    wq = np.ascontiguousarray(wq, np.uint8)
    ws = np.ascontiguousarray(ws, np.uint8)
    M, K = xb.shape
    N = wq.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    y64 = np.empty((M, N), np.float64)
    rc = lib().oracle_nvfp4_linear_unquantized_act(_p(xb, C.c_uint16), M, K, _p(wq, C.c_uint8),
                                                   _p(ws, C.c_uint8), N,
                                                   np.float32(weight_scale_2), _p(b, C.c_float),
                                                   _p(y64, C.c_double))
    if rc != 0:
        raise ValueError("bad shape")
    return y64


def w4a16_dequantize_bf16(q, s, weight_scale_2) -> np.ndarray:
    """bf16 bits [R, K] of bf16(fp32(E2M1(q) * E4M3(s) * weight_scale_2))."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    R, K = q.shape[0], q.shape[1] * 2
    out = np.empty((R, K), np.uint16)
    rc = lib().oracle_w4a16_dequantize_bf16(_p(q, C.c_uint8), _p(s, C.c_uint8), R, K,
                                            np.float32(weight_scale_2), _p(out, C.c_uint16))
    if rc != 0:
        raise ValueError("oracle_w4a16_dequantize_bf16: bad shape")
    return out


def w4a16_linear(x, wq, ws, weight_scale_2, bias=None):
    """W4A16 linear on bf16 activations x [M, K] and NVFP4 weights: returns (y bf16
    bits [M, N], y fp64 [M, N], tolerance scale T fp64 [M, N])."""
    xb = _bits16(x)
    wq = np.ascontiguousarray(wq, np.uint8)
    ws = np.ascontiguousarray(ws, np.uint8)
    M, K = xb.shape
    N = wq.shape[0]
    assert wq.shape[1] * 2 == K and ws.shape == (N, K // 16)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    y = np.empty((M, N), np.uint16)
    y64 = np.empty((M, N), np.float64)
    T = np.empty((M, N), np.float64)
    rc = lib().oracle_w4a16_linear(_p(xb, C.c_uint16), M, K, _p(wq, C.c_uint8),
                                   _p(ws, C.c_uint8), N, np.float32(weight_scale_2),
                                   _p(b, C.c_float), _p(y, C.c_uint16), _p(y64, C.c_double),
                                   _p(T, C.c_double))
    if rc != 0:
        raise ValueError("oracle_w4a16_linear: bad shape")
    return y, y64, T


def fp8r_quantize_rows(x):
    """bf16 [R, K] -> (E4M3 codes uint8 [R, K], fp32 row scales [R])."""
    xb = _bits16(x)
    R, K = xb.shape
    q = np.empty((R, K), np.uint8)
    s = np.empty((R,), np.float32)
    rc = lib().oracle_fp8r_quantize_rows(_p(xb, C.c_uint16), R, K, _p(q, C.c_uint8),
                                         _p(s, C.c_float))
    if rc != 0:
        raise ValueError("bad shape")
    return q, s


def fp8r_linear(xq, xs, wq, ws, bias=None):
    """Returns (y bf16 bits uint16 [M,N], y fp64, tolerance scale T)."""
    xq = np.ascontiguousarray(xq, np.uint8)
    xs = np.ascontiguousarray(xs, np.float32)
    wq = np.ascontiguousarray(wq, np.uint8)
    ws = np.ascontiguousarray(ws, np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    y = np.empty((M, N), np.uint16)
    y64 = np.empty((M, N), np.float64)
    T = np.empty((M, N), np.float64)
    rc = lib().oracle_fp8r_linear(_p(xq, C.c_uint8), _p(xs, C.c_float), M, K, _p(wq, C.c_uint8),
                                  _p(ws, C.c_float), N, _p(b, C.c_float), _p(y, C.c_uint16),
                                  _p(y64, C.c_double), _p(T, C.c_double))
    if rc != 0:
        raise ValueError("bad shape")
    return y, y64, T


def bf16_ulp(v) -> np.ndarray:
    """Spacing of bf16 values at |v|: 2^(floor(log2|v|) - 7) for normal |v|,
    2^-133 for zero and subnormals."""
    a = np.abs(np.asarray(v, np.float64))
    out = np.full(a.shape, 2.0 ** -133)
    normal = a >= 2.0 ** -126
    e = np.floor(np.log2(a[normal]))
    out[normal] = np.ldexp(1.0, (e - 7).astype(np.int64))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def int4_quantize(x):
    """bf16 [R, K] -> (INT4 codes uint8 [R, K/2], element 2j in the low nibble, two's
    complement; fp32 group scales [R, K/64]). K % 64 == 0."""
    xb = _bits16(x)
    R, K = xb.shape
    q = np.empty((R, K // 2), np.uint8)
    s = np.empty((R, K // 64), np.float32)
    rc = lib().oracle_int4_quantize(_p(xb, C.c_uint16), R, K, _p(q, C.c_uint8), _p(s, C.c_float))
    if rc != 0:
        raise ValueError("oracle_int4_quantize: bad shape")
    return q, s


def int4_linear(xq, xs, wq, ws, bias=None):
    """INT4 W4A4 linear: returns (y bf16 bits [M, N], y fp64, tolerance scale T)."""
    xq = np.ascontiguousarray(xq, np.uint8)
    xs = np.ascontiguousarray(xs, np.float32)
    wq = np.ascontiguousarray(wq, np.uint8)
    ws = np.ascontiguousarray(ws, np.float32)
    M, K = xq.shape[0], xq.shape[1] * 2
    N = wq.shape[0]
    assert wq.shape[1] * 2 == K and xs.shape == (M, K // 64) and ws.shape == (N, K // 64)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    y = np.empty((M, N), np.uint16)
    y64 = np.empty((M, N), np.float64)
    T = np.empty((M, N), np.float64)
    rc = lib().oracle_int4_linear(_p(xq, C.c_uint8), _p(xs, C.c_float), M, K, _p(wq, C.c_uint8),
                                  _p(ws, C.c_float), N, _p(b, C.c_float), _p(y, C.c_uint16),
                                  _p(y64, C.c_double), _p(T, C.c_double))
    if rc != 0:
        raise ValueError("oracle_int4_linear: bad shape")
    return y, y64, T
