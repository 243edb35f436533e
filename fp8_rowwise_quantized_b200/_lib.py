"""ctypes binding of libqlinear.so (the C ABI in include/qlinear.h).

Argument marshalling only: tensors are passed as device pointers with the
current torch stream; every step of the computation runs in the library's
kernels. There is no fallback: if the library is missing or fails to load,
``load()`` raises.
"""
import ctypes as C
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlinear.so")

QL_OK = 0
QL_ERR_INVALID_ARG = 1
QL_ERR_SHAPE = 2
QL_ERR_ALIGN = 3
QL_ERR_DEVICE = 4
QL_ERR_WORKSPACE = 5
QL_ERR_LAUNCH = 6
QL_ERR_TIMEOUT = 7

# Every symbol the header declares, with (restype, argtypes).
_vp, _i64, _sz, _u8p, _f32p, _ip = C.c_void_p, C.c_int64, C.c_size_t, C.c_void_p, C.c_void_p, C.c_void_p
SIGNATURES = {
    "nvfp4_quantize_act": (C.c_int, [_vp, _i64, _i64, _f32p, _u8p, _u8p, _vp]),
    "nvfp4_linear_workspace_size": (C.c_size_t, [_i64, _i64, _i64]),
    "nvfp4_weight_scale_atoms_size": (C.c_size_t, [_i64, _i64, C.c_int]),
    "nvfp4_layout_weight_scales": (C.c_int, [_u8p, _i64, _i64, C.c_int, _u8p, _sz, _vp]),
    "nvfp4_linear_laid_out": (C.c_int, [_vp, _i64, _i64, _u8p, _u8p, C.c_int, _i64, _f32p, _f32p,
                                        _f32p, _vp, _vp, _sz, _vp]),
    "nvfp4_linear": (C.c_int, [_vp, _i64, _i64, _u8p, _u8p, _i64, _f32p, _f32p, _f32p, _vp, _vp,
                               _sz, _vp]),
    "nvfp4_linear_single_launch": (C.c_int, [_vp, _i64, _i64, _u8p, _u8p, _i64, _f32p, _f32p,
                                             _f32p, _vp, _vp, _sz, _vp]),
    "nvfp4_linear_gelu_quantize": (C.c_int, [_vp, _i64, _i64, _u8p, _u8p, _i64, _f32p, _f32p,
                                             _f32p, _f32p, _vp, _sz, _vp, _sz, _vp]),
    "nvfp4_linear_quantized_input": (C.c_int, [_i64, _i64, _u8p, _u8p, _i64, _f32p, _f32p,
                                               _f32p, _vp, _vp, _sz, _vp]),
    "nvfp4_linear_gemm_lowrank": (C.c_int, [_i64, _i64, _u8p, _i64, _f32p, _f32p, _f32p, _vp,
                                            _vp, _i64, _vp, _vp, _sz, _vp]),
    "svdq_nvfp4_linear_workspace_size": (C.c_size_t, [_i64, _i64, _i64, _i64]),
    "svdq_nvfp4_linear": (C.c_int, [_vp, _i64, _i64, _f32p, _vp, _vp, _i64, _u8p, _u8p, _i64,
                                    _f32p, _f32p, _f32p, _vp, _vp, _sz, _vp]),
    "w4a16_linear": (C.c_int, [_vp, _i64, _i64, _u8p, _u8p, _i64, _f32p, _f32p, _vp, _vp]),
    "nvfp4_linear_prologue": (C.c_int, [_vp, _i64, _i64, _u8p, _i64, _f32p, _vp, _sz, _vp]),
    "nvfp4_linear_gemm": (C.c_int, [_i64, _i64, _u8p, _i64, _f32p, _f32p, _f32p, _vp, _vp, _sz,
                                    _vp]),
    "nvfp4_linear_workspace_layout": (C.c_int, [_i64, _i64, _i64, C.POINTER(C.c_size_t),
                                                C.POINTER(C.c_size_t), C.POINTER(C.c_size_t)]),
    "nvfp4_global_scale": (C.c_int, [_vp, _i64, _f32p, _vp]),
    "nvfp4_linear_noalloc": (C.c_int, [_vp, _i64, _i64, _u8p, _u8p, _i64, _f32p, _f32p, _f32p,
                                       _vp, _vp]),
    "int4_quantize_rows": (C.c_int, [_vp, _i64, _i64, _u8p, _f32p, _vp]),
    "int4_linear_workspace_size": (C.c_size_t, [_i64, _i64, _i64]),
    "int4_linear": (C.c_int, [_vp, _i64, _i64, _u8p, _f32p, _i64, _f32p, _vp, _vp, _sz, _vp]),
    "int4_linear_gemm_workspace_size": (C.c_size_t, [_i64, _i64, _i64]),
    "int4_linear_gemm": (C.c_int, [_u8p, _f32p, _i64, _i64, _u8p, _f32p, _i64, _f32p, _vp,
                                   _vp, _sz, _vp]),
    "fp8r_quantize_rows": (C.c_int, [_vp, _i64, _i64, _u8p, _f32p, _vp]),
    "fp8r_linear_workspace_size": (C.c_size_t, [_i64, _i64, _i64]),
    "fp8r_linear": (C.c_int, [_vp, _i64, _i64, _u8p, _f32p, _i64, _f32p, _vp, _vp, _sz, _vp]),
    "fp8r_linear_gemm": (C.c_int, [_u8p, _f32p, _i64, _i64, _u8p, _f32p, _i64, _f32p, _vp, _vp]),
    "ql_encode_e4m3": (C.c_int, [_f32p, _u8p, _i64, _vp]),
    "ql_encode_e2m1": (C.c_int, [_f32p, _u8p, _i64, _vp]),
    "ql_read_device_status": (C.c_int, [C.POINTER(C.c_int)]),
    "ql_read_gemm_clock": (C.c_int, [C.POINTER(C.c_int64), C.POINTER(C.c_int64)]),
    "ql_set_fault_injection": (None, [C.c_int, C.c_int]),
    "ql_set_tile_override": (C.c_int, [C.c_int, C.c_int]),
    "ql_tile_config": (C.c_int, [C.c_int, _i64, _i64, _i64, C.POINTER(C.c_int),
                                 C.POINTER(C.c_int)]),
    "ql_status_string": (C.c_char_p, [C.c_int]),
    "ql_last_error_message": (C.c_char_p, []),
}

_lib = None
_lock = threading.Lock()


class QLinearError(RuntimeError):
    def __init__(self, fn, status, detail=""):
        self.status = status
        lib = load()
        text = lib.ql_status_string(status).decode()
        msg = f"{fn}: {text} (status {status})"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)


def load():
    """Load libqlinear.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m fp8_rowwise_quantized_b200.build` "
                "(there is no fallback path)")
        lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(fn_name, status):
    if status != QL_OK:
        detail = ""
        if status in (QL_ERR_LAUNCH, QL_ERR_DEVICE, QL_ERR_SHAPE, QL_ERR_WORKSPACE):
            detail = load().ql_last_error_message().decode()
        raise QLinearError(fn_name, status, detail)
