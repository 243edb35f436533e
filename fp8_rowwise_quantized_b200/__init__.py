"""B200 (sm_100a) NVFP4 / FP8-rowwise quantized linear layer.

Python face of the C ABI in ``include/qlinear.h``: the same entry points, taking
torch CUDA tensors. PyTorch only provides device memory and the current stream;
the computation runs in the library's CUDA kernels (there is no CPU or library
fallback, and a missing ``libqlinear.so`` raises on first use).

The scheme (Diffusers page "BFL (fp8r / nvfp4)", scheme list):
  * nvfp4: packed E2M1 weight (two values per byte), one E4M3 scale per 16
    elements, global fp32 ``weight_scale_2`` and calibrated fp32 ``input_scale``;
    activations are quantized to NVFP4 at run time;
  * fp8r: E4M3 weight with one fp32 scale per row; activations are quantized per
    row to E4M3 at run time.
"""
from typing import Optional, Tuple

import torch

from . import _lib

__all__ = [
    "nvfp4_quantize_act", "nvfp4_linear", "nvfp4_linear_single_launch", "nvfp4_linear_noalloc",
    "nvfp4_linear_prologue", "nvfp4_linear_gelu_quantize", "nvfp4_linear_quantized_input",
    "nvfp4_linear_gemm_lowrank", "svdq_nvfp4_linear", "svdq_nvfp4_linear_workspace_size",
    "w4a16_linear", "int4_quantize_rows", "int4_linear", "int4_linear_gemm",
    "int4_linear_workspace_size", "prepare_int4_weight",
    "nvfp4_linear_gemm",
    "nvfp4_linear_workspace_size", "nvfp4_linear_workspace_layout", "nvfp4_global_scale",
    "fp8r_quantize_rows", "fp8r_linear", "fp8r_linear_gemm", "fp8r_linear_workspace_size",
    "ql_encode_e4m3", "ql_encode_e2m1", "read_device_status", "set_fault_injection",
    "set_tile_override", "tile_config",
    "prepare_nvfp4_weight", "prepare_fp8r_weight", "QLinearError", "library_path",
]

QLinearError = _lib.QLinearError
library_path = _lib.LIB_PATH


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _need(t: torch.Tensor, name: str, dtype, ndim: Optional[int] = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _scalar(t: torch.Tensor, name: str):
    _need(t, name, torch.float32)
    if t.numel() != 1:
        raise ValueError(f"{name} must hold one fp32 value")


# ----------------------------------------------------------------------------- NVFP4

def nvfp4_quantize_act(x: torch.Tensor, input_scale: torch.Tensor,
                       xq: Optional[torch.Tensor] = None,
                       xs: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 [M, K] -> (packed E2M1 codes uint8 [M, K/2], E4M3 block scales uint8 [M, K/16])."""
    _need(x, "x", torch.bfloat16, 2)
    _scalar(input_scale, "input_scale")
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if xs is None:
        xs = torch.empty((M, K // 16), dtype=torch.uint8, device=x.device)
    _lib.check("nvfp4_quantize_act", _lib.load().nvfp4_quantize_act(
        _ptr(x), M, K, _ptr(input_scale), _ptr(xq), _ptr(xs), _stream()))
    return xq, xs


def nvfp4_linear_workspace_size(M: int, K: int, N: int) -> int:
    return int(_lib.load().nvfp4_linear_workspace_size(M, K, N))


def nvfp4_linear_workspace_layout(M: int, K: int, N: int) -> Tuple[int, int, int]:
    a, b, c = (_lib.C.c_size_t(), _lib.C.c_size_t(), _lib.C.c_size_t())
    _lib.check("nvfp4_linear_workspace_layout", _lib.load().nvfp4_linear_workspace_layout(
        M, K, N, _lib.C.byref(a), _lib.C.byref(b), _lib.C.byref(c)))
    return a.value, b.value, c.value


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is None:
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", torch.uint8)
    return workspace


def nvfp4_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                 weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                 bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = bf16(input_scale * weight_scale_2 * (NVFP4(x) @ NVFP4(w)^T) + bias).

    x bf16 [M, K]; w uint8 [N, K/2]; w_scale uint8 [N, K/16] (E4M3 codes);
    weight_scale_2 / input_scale fp32 scalars; bias fp32 [N] or None."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _scalar(weight_scale_2, "weight_scale_2")
    _scalar(input_scale, "input_scale")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] * 2 != K or tuple(w_scale.shape) != (N, K // 16):
        raise ValueError("weight shapes do not match x")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), x.device, workspace)
    _lib.check("nvfp4_linear", _lib.load().nvfp4_linear(
        _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2), _ptr(input_scale),
        _ptr(bias), _ptr(y), _ptr(ws), ws.numel(), _stream()))
    return y


def nvfp4_linear_single_launch(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                               weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                               bias: Optional[torch.Tensor] = None,
                               y: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear as one kernel launch (quantization inside the GEMM launch, then a
    grid-wide barrier, then the GEMM); same bits as nvfp4_linear. Needs K % 256 == 0."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _scalar(weight_scale_2, "weight_scale_2")
    _scalar(input_scale, "input_scale")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] * 2 != K or tuple(w_scale.shape) != (N, K // 16):
        raise ValueError("weight shapes do not match x")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), x.device, workspace)
    _lib.check("nvfp4_linear_single_launch", _lib.load().nvfp4_linear_single_launch(
        _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2), _ptr(input_scale),
        _ptr(bias), _ptr(y), _ptr(ws), ws.numel(), _stream()))
    return y


def nvfp4_linear_gelu_quantize(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                               weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                               next_input_scale: torch.Tensor, next_workspace: torch.Tensor,
                               bias: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None) -> None:
    """MLP up projection + GELU + NVFP4 quantization for the down projection: writes
    NVFP4(GELU(linear)) (global scale next_input_scale) into the activation part of
    next_workspace, a uint8 buffer of nvfp4_linear_workspace_size(M, N, N_down)
    bytes, for nvfp4_linear_quantized_input. Needs N % 256 == 0."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _need(next_workspace, "next_workspace", torch.uint8, 1)
    _scalar(weight_scale_2, "weight_scale_2")
    _scalar(input_scale, "input_scale")
    _scalar(next_input_scale, "next_input_scale")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] * 2 != K or tuple(w_scale.shape) != (N, K // 16):
        raise ValueError("weight shapes do not match x")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), x.device, workspace)
    _lib.check("nvfp4_linear_gelu_quantize", _lib.load().nvfp4_linear_gelu_quantize(
        _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2), _ptr(input_scale),
        _ptr(bias), _ptr(next_input_scale), _ptr(next_workspace), next_workspace.numel(),
        _ptr(ws), ws.numel(), _stream()))


def nvfp4_linear_quantized_input(M: int, w: torch.Tensor, w_scale: torch.Tensor,
                                 weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                                 workspace: torch.Tensor, bias: Optional[torch.Tensor] = None,
                                 y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear on activations already quantized into `workspace` (by
    nvfp4_linear_gelu_quantize): weight-scale layout, then the GEMM."""
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _need(workspace, "workspace", torch.uint8, 1)
    _scalar(weight_scale_2, "weight_scale_2")
    _scalar(input_scale, "input_scale")
    N, K = w.shape[0], w.shape[1] * 2
    if tuple(w_scale.shape) != (N, K // 16):
        raise ValueError("weight scale shape does not match w")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=w.device)
    _lib.check("nvfp4_linear_quantized_input", _lib.load().nvfp4_linear_quantized_input(
        M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias),
        _ptr(y), _ptr(workspace), workspace.numel(), _stream()))
    return y


def nvfp4_linear_gemm_lowrank(M: int, w: torch.Tensor, weight_scale_2: torch.Tensor,
                              input_scale: torch.Tensor, workspace: torch.Tensor,
                              lr_act: torch.Tensor, lr_up: torch.Tensor,
                              bias: Optional[torch.Tensor] = None,
                              y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear_gemm plus the low-rank branch alpha * lr_act @ lr_up^T: lr_act bf16
    [M, r] (the branch's activations divided by alpha), lr_up bf16 [N, r]."""
    _need(w, "w", torch.uint8, 2)
    _need(workspace, "workspace", torch.uint8, 1)
    _need(lr_act, "lr_act", torch.bfloat16, 2)
    _need(lr_up, "lr_up", torch.bfloat16, 2)
    _scalar(weight_scale_2, "weight_scale_2")
    _scalar(input_scale, "input_scale")
    N, K = w.shape[0], w.shape[1] * 2
    r = lr_act.shape[1]
    if lr_act.shape[0] != M or tuple(lr_up.shape) != (N, r):
        raise ValueError("low-rank operand shapes do not match")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=w.device)
    _lib.check("nvfp4_linear_gemm_lowrank", _lib.load().nvfp4_linear_gemm_lowrank(
        M, K, _ptr(w), N, _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(lr_act),
        _ptr(lr_up), r, _ptr(y), _ptr(workspace), workspace.numel(), _stream()))
    return y


def svdq_nvfp4_linear_workspace_size(M: int, K: int, N: int, rank: int) -> int:
    return int(_lib.load().svdq_nvfp4_linear_workspace_size(M, K, N, rank))


def svdq_nvfp4_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                      weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                      lora_down: torch.Tensor, lora_up: torch.Tensor,
                      smooth: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                      y: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """SVDQuant-style NVFP4 linear: Y = bf16(alpha * NVFP4(xs) NVFP4(w)^T
    + (xs lora_down^T) lora_up^T + bias), xs = bf16(x * smooth). lora_down bf16 [r, K],
    lora_up bf16 [N, r], smooth fp32 [K] or None; input_scale calibrated on xs."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _need(lora_down, "lora_down", torch.bfloat16, 2)
    _need(lora_up, "lora_up", torch.bfloat16, 2)
    _scalar(weight_scale_2, "weight_scale_2")
    _scalar(input_scale, "input_scale")
    M, K = x.shape
    N = w.shape[0]
    r = lora_down.shape[0]
    if w.shape[1] * 2 != K or tuple(w_scale.shape) != (N, K // 16):
        raise ValueError("weight shapes do not match x")
    if tuple(lora_down.shape) != (r, K) or tuple(lora_up.shape) != (N, r):
        raise ValueError("low-rank shapes do not match")
    if smooth is not None:
        _need(smooth, "smooth", torch.float32, 1)
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(svdq_nvfp4_linear_workspace_size(M, K, N, r), x.device, workspace)
    _lib.check("svdq_nvfp4_linear", _lib.load().svdq_nvfp4_linear(
        _ptr(x), M, K, _ptr(smooth), _ptr(lora_down), _ptr(lora_up), r, _ptr(w), _ptr(w_scale),
        N, _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(y), _ptr(ws), ws.numel(),
        _stream()))
    return y


def w4a16_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                 weight_scale_2: torch.Tensor, bias: Optional[torch.Tensor] = None,
                 y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = bf16(x @ what^T + bias) with what = bf16(fp32(E2M1(w) * E4M3(w_scale) *
    weight_scale_2)): 4-bit weights, bf16 activations (modulation layers).

    x bf16 [M, K]; w uint8 [N, K/2]; w_scale uint8 [N, K/16]; weight_scale_2 fp32
    scalar; bias fp32 [N] or None."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _scalar(weight_scale_2, "weight_scale_2")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] * 2 != K or tuple(w_scale.shape) != (N, K // 16):
        raise ValueError("weight shapes do not match x")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _lib.check("w4a16_linear", _lib.load().w4a16_linear(
        _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2), _ptr(bias), _ptr(y),
        _stream()))
    return y


def nvfp4_linear_noalloc(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                         weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                         bias: Optional[torch.Tensor] = None,
                         y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear without a workspace argument, for callers that cannot allocate
    device memory: the library's fixed 32 MiB scratch array is used instead (see
    include/qlinear.h). Pass ``y`` to avoid the output allocation here as well."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _scalar(weight_scale_2, "weight_scale_2")
    _scalar(input_scale, "input_scale")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] * 2 != K or tuple(w_scale.shape) != (N, K // 16):
        raise ValueError("weight shapes do not match x")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _lib.check("nvfp4_linear_noalloc", _lib.load().nvfp4_linear_noalloc(
        _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2), _ptr(input_scale),
        _ptr(bias), _ptr(y), _stream()))
    return y


def nvfp4_linear_prologue(x: torch.Tensor, w_scale: torch.Tensor, input_scale: torch.Tensor,
                          workspace: torch.Tensor) -> None:
    _need(x, "x", torch.bfloat16, 2)
    _need(w_scale, "w_scale", torch.uint8, 2)
    _scalar(input_scale, "input_scale")
    M, K = x.shape
    N = w_scale.shape[0]
    _lib.check("nvfp4_linear_prologue", _lib.load().nvfp4_linear_prologue(
        _ptr(x), M, K, _ptr(w_scale), N, _ptr(input_scale), _ptr(workspace), workspace.numel(),
        _stream()))


def nvfp4_linear_gemm(M: int, w: torch.Tensor, weight_scale_2: torch.Tensor,
                      input_scale: torch.Tensor, workspace: torch.Tensor,
                      bias: Optional[torch.Tensor] = None,
                      y: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(w, "w", torch.uint8, 2)
    N, K = w.shape[0], w.shape[1] * 2
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=w.device)
    _lib.check("nvfp4_linear_gemm", _lib.load().nvfp4_linear_gemm(
        M, K, _ptr(w), N, _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(y),
        _ptr(workspace), workspace.numel(), _stream()))
    return y


def nvfp4_global_scale(x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Device fp32 scalar amax(|x|) / (6 * 448) (the calibration rule of the workloads)."""
    _need(x, "x", torch.bfloat16)
    if out is None:
        out = torch.empty((1,), dtype=torch.float32, device=x.device)
    _lib.check("nvfp4_global_scale", _lib.load().nvfp4_global_scale(
        _ptr(x), x.numel(), _ptr(out), _stream()))
    return out


def prepare_nvfp4_weight(w: torch.Tensor):
    """bf16 [N, K] weight -> (codes [N, K/2], scales [N, K/16], weight_scale_2 [1]),
    quantized on the GPU by the same kernel as the activations."""
    g = nvfp4_global_scale(w)
    wq, ws = nvfp4_quantize_act(w, g)
    return wq, ws, g


# ----------------------------------------------------------------------------- fp8r

# ----------------------------------------------------------------------------- INT4

def int4_quantize_rows(x: torch.Tensor, q: Optional[torch.Tensor] = None,
                       scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 [M, K] -> (INT4 codes uint8 [M, K/2], fp32 group scales [M, K/64])."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((M, K // 64), dtype=torch.float32, device=x.device)
    _lib.check("int4_quantize_rows", _lib.load().int4_quantize_rows(
        _ptr(x), M, K, _ptr(q), _ptr(scale), _stream()))
    return q, scale


def prepare_int4_weight(w: torch.Tensor):
    """bf16 weight [N, K] -> (INT4 codes [N, K/2], group scales [N, K/64])."""
    return int4_quantize_rows(w.contiguous())


def int4_linear_workspace_size(M: int, K: int, N: int) -> int:
    return int(_lib.load().int4_linear_workspace_size(M, K, N))


def int4_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """INT4 W4A4 linear: Y = bf16(sum_g xs ws sum_k qx qw + bias), x quantized at run time."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.float32, 2)
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] * 2 != K or tuple(w_scale.shape) != (N, K // 64):
        raise ValueError("weight shapes do not match x")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(int4_linear_workspace_size(M, K, N), x.device, workspace)
    _lib.check("int4_linear", _lib.load().int4_linear(
        _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(bias), _ptr(y), _ptr(ws), ws.numel(),
        _stream()))
    return y


def int4_linear_gemm(xq: torch.Tensor, x_scale: torch.Tensor, w: torch.Tensor,
                     w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     y: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(xq, "xq", torch.uint8, 2)
    _need(x_scale, "x_scale", torch.float32, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.float32, 2)
    M, K = xq.shape[0], xq.shape[1] * 2
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _lib.check("int4_linear_gemm", _lib.load().int4_linear_gemm(
        _ptr(xq), _ptr(x_scale), M, K, _ptr(w), _ptr(w_scale), N, _ptr(bias), _ptr(y),
        _stream()))
    return y


def fp8r_quantize_rows(x: torch.Tensor, xq: Optional[torch.Tensor] = None,
                       x_scale: Optional[torch.Tensor] = None):
    """bf16 [M, K] -> (E4M3 codes uint8 [M, K], fp32 row scales [M])."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    _lib.check("fp8r_quantize_rows", _lib.load().fp8r_quantize_rows(
        _ptr(x), M, K, _ptr(xq), _ptr(x_scale), _stream()))
    return xq, x_scale


def prepare_fp8r_weight(w: torch.Tensor):
    """bf16 [N, K] weight -> (E4M3 codes [N, K], fp32 per-row scales [N])."""
    return fp8r_quantize_rows(w)


def fp8r_linear_workspace_size(M: int, K: int, N: int) -> int:
    return int(_lib.load().fp8r_linear_workspace_size(M, K, N))


def fp8r_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = bf16(x_scale[m] * w_scale[n] * (E4M3(x) @ E4M3(w)^T) + bias)."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.uint8, 2)
    _need(w_scale, "w_scale", torch.float32, 1)
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K or w_scale.shape[0] != N:
        raise ValueError("weight shapes do not match x")
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(fp8r_linear_workspace_size(M, K, N), x.device, workspace)
    _lib.check("fp8r_linear", _lib.load().fp8r_linear(
        _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(bias), _ptr(y), _ptr(ws), ws.numel(),
        _stream()))
    return y


def fp8r_linear_gemm(xq: torch.Tensor, x_scale: torch.Tensor, w: torch.Tensor,
                     w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     y: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(xq, "xq", torch.uint8, 2)
    _need(w, "w", torch.uint8, 2)
    M, K = xq.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _lib.check("fp8r_linear_gemm", _lib.load().fp8r_linear_gemm(
        _ptr(xq), _ptr(x_scale), M, K, _ptr(w), _ptr(w_scale), N, _ptr(bias), _ptr(y),
        _stream()))
    return y


# ----------------------------------------------------------------------------- diagnostics

def ql_encode_e4m3(v: torch.Tensor) -> torch.Tensor:
    _need(v, "v", torch.float32)
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _lib.check("ql_encode_e4m3", _lib.load().ql_encode_e4m3(_ptr(v), _ptr(out), v.numel(), _stream()))
    return out


def ql_encode_e2m1(v: torch.Tensor) -> torch.Tensor:
    _need(v, "v", torch.float32)
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _lib.check("ql_encode_e2m1", _lib.load().ql_encode_e2m1(_ptr(v), _ptr(out), v.numel(), _stream()))
    return out


def read_device_status() -> int:
    st = _lib.C.c_int(0)
    _lib.check("ql_read_device_status", _lib.load().ql_read_device_status(_lib.C.byref(st)))
    return st.value


def set_fault_injection(enable: bool, timeout_ms: int = 0) -> None:
    _lib.load().ql_set_fault_injection(1 if enable else 0, int(timeout_ms))


def tile_config(M: int, N: int, K: int, fp4: bool = True) -> Tuple[int, int]:
    """(bn, cg) of the GEMM tiles a call of this size uses: (128 * cg) x bn."""
    bn, cg = _lib.C.c_int(), _lib.C.c_int()
    _lib.check("ql_tile_config", _lib.load().ql_tile_config(
        1 if fp4 else 0, M, N, K, _lib.C.byref(bn), _lib.C.byref(cg)))
    return bn.value, cg.value


def set_tile_override(bn: int = 0, cg: int = 0) -> None:
    """Force the GEMM tile ((128 * cg) x bn) for later calls; bn = 0 restores the
    automatic choice."""
    _lib.check("ql_set_tile_override", _lib.load().ql_set_tile_override(int(bn), int(cg)))
