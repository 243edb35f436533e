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

Every tensor argument is checked (dtype, shape, contiguity) and must live on the
device of the call (the device of its first tensor argument); the library call
runs with that device current, on its current stream.
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
    "set_tile_override", "tile_config", "read_gemm_clock",
    "prepare_nvfp4_weight", "prepare_fp8r_weight", "QLinearError", "library_path",
]

QLinearError = _lib.QLinearError
library_path = _lib.LIB_PATH


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype, ndim: Optional[int] = None,
          shape: Optional[tuple] = None, device: Optional[torch.device] = None):
    """Checks a tensor argument: dtype, rank, shape, contiguity, and that it is a
    CUDA tensor, on `device` (the device of the call) when one is given."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, but the call runs on {device}")


def _scalar(t: torch.Tensor, name: str, device: Optional[torch.device] = None):
    _need(t, name, torch.float32, device=device)
    if t.numel() != 1:
        raise ValueError(f"{name} must hold one fp32 value")


def _out(y: Optional[torch.Tensor], M: int, N: int, device: torch.device) -> torch.Tensor:
    """The bf16 [M, N] output: allocated when None, else checked."""
    if y is None:
        return torch.empty((M, N), dtype=torch.bfloat16, device=device)
    _need(y, "y", torch.bfloat16, 2, (M, N), device)
    return y


def _bias(bias: Optional[torch.Tensor], N: int, device: torch.device) -> None:
    if bias is not None:
        _need(bias, "bias", torch.float32, 1, (N,), device)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is None:
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", torch.uint8, device=device)
    if workspace.numel() < nbytes:
        raise ValueError(f"workspace holds {workspace.numel()} bytes, the call needs {nbytes}")
    return workspace


def _call(name: str, device: torch.device, *args) -> None:
    """Runs the C entry point `name` with `device` current, on that device's current
    stream (appended as the last argument); raises on a non-zero status."""
    with torch.cuda.device(device):
        stream = torch.cuda.current_stream(device).cuda_stream
        _lib.check(name, getattr(_lib.load(), name)(*args, stream))


def _nvfp4_weight(w: torch.Tensor, w_scale: torch.Tensor, K: int, dev) -> int:
    """Checks an NVFP4 weight (codes uint8 [N, K/2], scales uint8 [N, K/16]); returns N."""
    _need(w, "w", torch.uint8, 2, device=dev)
    N = w.shape[0]
    if w.shape[1] * 2 != K:
        raise ValueError(f"w must have K/2 = {K // 2} bytes per row, got {w.shape[1]}")
    _need(w_scale, "w_scale", torch.uint8, 2, (N, K // 16), dev)
    return N


# ----------------------------------------------------------------------------- NVFP4

def nvfp4_quantize_act(x: torch.Tensor, input_scale: torch.Tensor,
                       xq: Optional[torch.Tensor] = None,
                       xs: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 [M, K] -> (packed E2M1 codes uint8 [M, K/2], E4M3 block scales uint8 [M, K/16])."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    _scalar(input_scale, "input_scale", dev)
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    _need(xq, "xq", torch.uint8, 2, (M, K // 2), dev)
    if xs is None:
        xs = torch.empty((M, K // 16), dtype=torch.uint8, device=dev)
    _need(xs, "xs", torch.uint8, 2, (M, K // 16), dev)
    _call("nvfp4_quantize_act", dev, _ptr(x), M, K, _ptr(input_scale), _ptr(xq), _ptr(xs))
    return xq, xs


def nvfp4_linear_workspace_size(M: int, K: int, N: int) -> int:
    return int(_lib.load().nvfp4_linear_workspace_size(M, K, N))


def nvfp4_linear_workspace_layout(M: int, K: int, N: int) -> Tuple[int, int, int]:
    a, b, c = (_lib.C.c_size_t(), _lib.C.c_size_t(), _lib.C.c_size_t())
    _lib.check("nvfp4_linear_workspace_layout", _lib.load().nvfp4_linear_workspace_layout(
        M, K, N, _lib.C.byref(a), _lib.C.byref(b), _lib.C.byref(c)))
    return a.value, b.value, c.value


def nvfp4_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                 weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                 bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = bf16(input_scale * weight_scale_2 * (NVFP4(x) @ NVFP4(w)^T) + bias).

    x bf16 [M, K]; w uint8 [N, K/2]; w_scale uint8 [N, K/16] (E4M3 codes);
    weight_scale_2 / input_scale fp32 scalars; bias fp32 [N] or None."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    N = _nvfp4_weight(w, w_scale, K, dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), dev, workspace)
    _call("nvfp4_linear", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2),
          _ptr(input_scale), _ptr(bias), _ptr(y), _ptr(ws), ws.numel())
    return y


def nvfp4_weight_scale_atoms_size(N: int, K: int, bn: int) -> int:
    return int(_lib.load().nvfp4_weight_scale_atoms_size(N, K, bn))


def nvfp4_layout_weight_scales(w_scale: torch.Tensor, bn: int,
                               atoms: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The row-major E4M3 weight scales [N, K/16] laid out once for GEMM tiles of bn
    rows (128, 192, 224 or 256): the atoms nvfp4_linear_laid_out reads."""
    _need(w_scale, "w_scale", torch.uint8, 2)
    dev = w_scale.device
    N, K = w_scale.shape[0], w_scale.shape[1] * 16
    size = nvfp4_weight_scale_atoms_size(N, K, bn)
    if size == 0:
        raise ValueError(f"no weight-scale layout for N={N}, K={K}, bn={bn}")
    atoms = _workspace(size, dev, atoms)
    _call("nvfp4_layout_weight_scales", dev, _ptr(w_scale), N, K, int(bn), _ptr(atoms),
          atoms.numel())
    return atoms


def nvfp4_linear_laid_out(x: torch.Tensor, w: torch.Tensor, w_scale_atoms: torch.Tensor, bn: int,
                          weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                          bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear on weight scales laid out once by nvfp4_layout_weight_scales for
    tiles of bn rows (the call runs its GEMM at that tile width)."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    _need(w, "w", torch.uint8, 2, device=dev)
    N = w.shape[0]
    if w.shape[1] * 2 != K:
        raise ValueError(f"w must have K/2 = {K // 2} bytes per row, got {w.shape[1]}")
    size = nvfp4_weight_scale_atoms_size(N, K, bn)
    if size == 0:
        raise ValueError(f"no weight-scale layout for N={N}, K={K}, bn={bn}")
    _need(w_scale_atoms, "w_scale_atoms", torch.uint8, 1, device=dev)
    if w_scale_atoms.numel() < size:
        raise ValueError(f"w_scale_atoms holds {w_scale_atoms.numel()} bytes, needs {size}")
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), dev, workspace)
    _call("nvfp4_linear_laid_out", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale_atoms), int(bn), N,
          _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(y), _ptr(ws), ws.numel())
    return y


def nvfp4_linear_single_launch(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                               weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                               bias: Optional[torch.Tensor] = None,
                               y: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear as one kernel launch (quantization inside the GEMM launch, then a
    grid-wide barrier, then the GEMM); same bits as nvfp4_linear. Needs K % 256 == 0."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    N = _nvfp4_weight(w, w_scale, K, dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), dev, workspace)
    _call("nvfp4_linear_single_launch", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale), N,
          _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(y), _ptr(ws), ws.numel())
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
    dev = x.device
    M, K = x.shape
    N = _nvfp4_weight(w, w_scale, K, dev)
    _need(next_workspace, "next_workspace", torch.uint8, 1, device=dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    _scalar(next_input_scale, "next_input_scale", dev)
    _bias(bias, N, dev)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), dev, workspace)
    _call("nvfp4_linear_gelu_quantize", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale), N,
          _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(next_input_scale),
          _ptr(next_workspace), next_workspace.numel(), _ptr(ws), ws.numel())


def nvfp4_linear_quantized_input(M: int, w: torch.Tensor, w_scale: torch.Tensor,
                                 weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                                 workspace: torch.Tensor, bias: Optional[torch.Tensor] = None,
                                 y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear on activations already quantized into `workspace` (by
    nvfp4_linear_gelu_quantize): weight-scale layout, then the GEMM."""
    _need(w, "w", torch.uint8, 2)
    dev = w.device
    K = w.shape[1] * 2
    N = _nvfp4_weight(w, w_scale, K, dev)
    _need(workspace, "workspace", torch.uint8, 1, device=dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    _call("nvfp4_linear_quantized_input", dev, M, K, _ptr(w), _ptr(w_scale), N,
          _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(y), _ptr(workspace),
          workspace.numel())
    return y


def nvfp4_linear_gemm_lowrank(M: int, w: torch.Tensor, weight_scale_2: torch.Tensor,
                              input_scale: torch.Tensor, workspace: torch.Tensor,
                              lr_act: torch.Tensor, lr_up: torch.Tensor,
                              bias: Optional[torch.Tensor] = None,
                              y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear_gemm plus the low-rank branch alpha * lr_act @ lr_up^T: lr_act bf16
    [M, r] (the branch's activations divided by alpha), lr_up bf16 [N, r]."""
    _need(w, "w", torch.uint8, 2)
    dev = w.device
    N, K = w.shape[0], w.shape[1] * 2
    _need(workspace, "workspace", torch.uint8, 1, device=dev)
    _need(lr_act, "lr_act", torch.bfloat16, 2, device=dev)
    r = lr_act.shape[1]
    _need(lr_act, "lr_act", torch.bfloat16, 2, (M, r), dev)
    _need(lr_up, "lr_up", torch.bfloat16, 2, (N, r), dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    _call("nvfp4_linear_gemm_lowrank", dev, M, K, _ptr(w), N, _ptr(weight_scale_2),
          _ptr(input_scale), _ptr(bias), _ptr(lr_act), _ptr(lr_up), r, _ptr(y),
          _ptr(workspace), workspace.numel())
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
    dev = x.device
    M, K = x.shape
    N = _nvfp4_weight(w, w_scale, K, dev)
    _need(lora_down, "lora_down", torch.bfloat16, 2, device=dev)
    r = lora_down.shape[0]
    _need(lora_down, "lora_down", torch.bfloat16, 2, (r, K), dev)
    _need(lora_up, "lora_up", torch.bfloat16, 2, (N, r), dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    if smooth is not None:
        _need(smooth, "smooth", torch.float32, 1, (K,), dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    ws = _workspace(svdq_nvfp4_linear_workspace_size(M, K, N, r), dev, workspace)
    _call("svdq_nvfp4_linear", dev, _ptr(x), M, K, _ptr(smooth), _ptr(lora_down), _ptr(lora_up),
          r, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias),
          _ptr(y), _ptr(ws), ws.numel())
    return y


def w4a16_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                 weight_scale_2: torch.Tensor, bias: Optional[torch.Tensor] = None,
                 y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = bf16(x @ what^T + bias) with what = bf16(fp32(E2M1(w) * E4M3(w_scale) *
    weight_scale_2)): 4-bit weights, bf16 activations (modulation layers).

    x bf16 [M, K]; w uint8 [N, K/2]; w_scale uint8 [N, K/16]; weight_scale_2 fp32
    scalar; bias fp32 [N] or None."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    N = _nvfp4_weight(w, w_scale, K, dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    _call("w4a16_linear", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(weight_scale_2),
          _ptr(bias), _ptr(y))
    return y


def nvfp4_linear_noalloc(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                         weight_scale_2: torch.Tensor, input_scale: torch.Tensor,
                         bias: Optional[torch.Tensor] = None,
                         y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """nvfp4_linear without a workspace argument, for callers that cannot allocate
    device memory: the library's fixed 32 MiB scratch array of the call's device is
    used instead (see include/qlinear.h). Pass ``y`` to avoid the output allocation
    here as well; it is checked (bf16 [M, N], contiguous, on x's device)."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    N = _nvfp4_weight(w, w_scale, K, dev)
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    _call("nvfp4_linear_noalloc", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale), N,
          _ptr(weight_scale_2), _ptr(input_scale), _ptr(bias), _ptr(y))
    return y


def nvfp4_linear_prologue(x: torch.Tensor, w_scale: torch.Tensor, input_scale: torch.Tensor,
                          workspace: torch.Tensor) -> None:
    """The first launch of nvfp4_linear: quantizes x and lays out the weight scales
    into `workspace` (nvfp4_linear_workspace_size(M, K, N) bytes)."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    _need(w_scale, "w_scale", torch.uint8, 2, device=dev)
    N = w_scale.shape[0]
    _need(w_scale, "w_scale", torch.uint8, 2, (N, K // 16), dev)
    _scalar(input_scale, "input_scale", dev)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), dev, workspace)
    _call("nvfp4_linear_prologue", dev, _ptr(x), M, K, _ptr(w_scale), N, _ptr(input_scale),
          _ptr(ws), ws.numel())


def nvfp4_linear_gemm(M: int, w: torch.Tensor, weight_scale_2: torch.Tensor,
                      input_scale: torch.Tensor, workspace: torch.Tensor,
                      bias: Optional[torch.Tensor] = None,
                      y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The second launch of nvfp4_linear: the GEMM on a workspace filled by
    nvfp4_linear_prologue."""
    _need(w, "w", torch.uint8, 2)
    dev = w.device
    N, K = w.shape[0], w.shape[1] * 2
    _scalar(weight_scale_2, "weight_scale_2", dev)
    _scalar(input_scale, "input_scale", dev)
    ws = _workspace(nvfp4_linear_workspace_size(M, K, N), dev, workspace)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    _call("nvfp4_linear_gemm", dev, M, K, _ptr(w), N, _ptr(weight_scale_2), _ptr(input_scale),
          _ptr(bias), _ptr(y), _ptr(ws), ws.numel())
    return y


def nvfp4_global_scale(x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Device fp32 scalar amax(|x|) / (6 * 448) (the calibration rule of the workloads)."""
    _need(x, "x", torch.bfloat16)
    dev = x.device
    if out is None:
        out = torch.empty((1,), dtype=torch.float32, device=dev)
    _scalar(out, "out", dev)
    _call("nvfp4_global_scale", dev, _ptr(x), x.numel(), _ptr(out))
    return out


def prepare_nvfp4_weight(w: torch.Tensor):
    """bf16 [N, K] weight -> (codes [N, K/2], scales [N, K/16], weight_scale_2 [1]),
    quantized on the GPU by the same kernel as the activations."""
    g = nvfp4_global_scale(w)
    wq, ws = nvfp4_quantize_act(w, g)
    return wq, ws, g


# ----------------------------------------------------------------------------- INT4

def int4_quantize_rows(x: torch.Tensor, q: Optional[torch.Tensor] = None,
                       scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 [M, K] -> (INT4 codes uint8 [M, K/2], fp32 group scales [M, K/64])."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    _need(q, "q", torch.uint8, 2, (M, K // 2), dev)
    if scale is None:
        scale = torch.empty((M, K // 64), dtype=torch.float32, device=dev)
    _need(scale, "scale", torch.float32, 2, (M, K // 64), dev)
    _call("int4_quantize_rows", dev, _ptr(x), M, K, _ptr(q), _ptr(scale))
    return q, scale


def prepare_int4_weight(w: torch.Tensor):
    """bf16 weight [N, K] -> (INT4 codes [N, K/2], group scales [N, K/64])."""
    return int4_quantize_rows(w.contiguous())


def int4_linear_workspace_size(M: int, K: int, N: int) -> int:
    return int(_lib.load().int4_linear_workspace_size(M, K, N))


def _int4_weight(w: torch.Tensor, w_scale: torch.Tensor, K: int, dev) -> int:
    _need(w, "w", torch.uint8, 2, device=dev)
    N = w.shape[0]
    if w.shape[1] * 2 != K:
        raise ValueError(f"w must have K/2 = {K // 2} bytes per row, got {w.shape[1]}")
    _need(w_scale, "w_scale", torch.float32, 2, (N, K // 64), dev)
    return N


def int4_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """INT4 W4A4 linear: Y = bf16(sum_g xs ws sum_k qx qw + bias), x quantized at run time."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    N = _int4_weight(w, w_scale, K, dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    ws = _workspace(int4_linear_workspace_size(M, K, N), dev, workspace)
    _call("int4_linear", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(bias), _ptr(y),
          _ptr(ws), ws.numel())
    return y


def int4_linear_gemm_workspace_size(M: int, K: int, N: int) -> int:
    return int(_lib.load().int4_linear_gemm_workspace_size(M, K, N))


def int4_linear_gemm(xq: torch.Tensor, x_scale: torch.Tensor, w: torch.Tensor,
                     w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     y: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The GEMM of int4_linear on activations quantized by int4_quantize_rows."""
    _need(xq, "xq", torch.uint8, 2)
    dev = xq.device
    M, K = xq.shape[0], xq.shape[1] * 2
    _need(x_scale, "x_scale", torch.float32, 2, (M, K // 64), dev)
    N = _int4_weight(w, w_scale, K, dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    ws = _workspace(int4_linear_gemm_workspace_size(M, K, N), dev, workspace)
    _call("int4_linear_gemm", dev, _ptr(xq), _ptr(x_scale), M, K, _ptr(w), _ptr(w_scale), N,
          _ptr(bias), _ptr(y), _ptr(ws), ws.numel())
    return y


# ----------------------------------------------------------------------------- fp8r

def fp8r_quantize_rows(x: torch.Tensor, xq: Optional[torch.Tensor] = None,
                       x_scale: Optional[torch.Tensor] = None):
    """bf16 [M, K] -> (E4M3 codes uint8 [M, K], fp32 row scales [M])."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
    _need(xq, "xq", torch.uint8, 2, (M, K), dev)
    if x_scale is None:
        x_scale = torch.empty((M,), dtype=torch.float32, device=dev)
    _need(x_scale, "x_scale", torch.float32, 1, (M,), dev)
    _call("fp8r_quantize_rows", dev, _ptr(x), M, K, _ptr(xq), _ptr(x_scale))
    return xq, x_scale


def prepare_fp8r_weight(w: torch.Tensor):
    """bf16 [N, K] weight -> (E4M3 codes [N, K], fp32 per-row scales [N])."""
    return fp8r_quantize_rows(w)


def fp8r_linear_workspace_size(M: int, K: int, N: int) -> int:
    return int(_lib.load().fp8r_linear_workspace_size(M, K, N))


def _fp8r_weight(w: torch.Tensor, w_scale: torch.Tensor, K: int, dev) -> int:
    _need(w, "w", torch.uint8, 2, device=dev)
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError(f"w must have K = {K} bytes per row, got {w.shape[1]}")
    _need(w_scale, "w_scale", torch.float32, 1, (N,), dev)
    return N


def fp8r_linear(x: torch.Tensor, w: torch.Tensor, w_scale: torch.Tensor,
                bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = bf16(x_scale[m] * w_scale[n] * (E4M3(x) @ E4M3(w)^T) + bias)."""
    _need(x, "x", torch.bfloat16, 2)
    dev = x.device
    M, K = x.shape
    N = _fp8r_weight(w, w_scale, K, dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    ws = _workspace(fp8r_linear_workspace_size(M, K, N), dev, workspace)
    _call("fp8r_linear", dev, _ptr(x), M, K, _ptr(w), _ptr(w_scale), N, _ptr(bias), _ptr(y),
          _ptr(ws), ws.numel())
    return y


def fp8r_linear_gemm(xq: torch.Tensor, x_scale: torch.Tensor, w: torch.Tensor,
                     w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The GEMM of fp8r_linear on activations quantized by fp8r_quantize_rows."""
    _need(xq, "xq", torch.uint8, 2)
    dev = xq.device
    M, K = xq.shape
    _need(x_scale, "x_scale", torch.float32, 1, (M,), dev)
    N = _fp8r_weight(w, w_scale, K, dev)
    _bias(bias, N, dev)
    y = _out(y, M, N, dev)
    _call("fp8r_linear_gemm", dev, _ptr(xq), _ptr(x_scale), M, K, _ptr(w), _ptr(w_scale), N,
          _ptr(bias), _ptr(y))
    return y


# ----------------------------------------------------------------------------- diagnostics

def ql_encode_e4m3(v: torch.Tensor) -> torch.Tensor:
    _need(v, "v", torch.float32)
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _call("ql_encode_e4m3", v.device, _ptr(v), _ptr(out), v.numel())
    return out


def ql_encode_e2m1(v: torch.Tensor) -> torch.Tensor:
    _need(v, "v", torch.float32)
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _call("ql_encode_e2m1", v.device, _ptr(v), _ptr(out), v.numel())
    return out


def read_device_status() -> int:
    """Reads and clears the current device's status word (0, or QL_ERR_TIMEOUT after a
    kernel's bounded wait expired)."""
    st = _lib.C.c_int(0)
    _lib.check("ql_read_device_status", _lib.load().ql_read_device_status(_lib.C.byref(st)))
    return st.value


def read_gemm_clock() -> Tuple[int, int]:
    """(SM cycles, nanoseconds) of the first CTA of the last GEMM launch on the current
    device; cycles / ns is the SM clock in GHz that launch ran at."""
    c, t = _lib.C.c_int64(0), _lib.C.c_int64(0)
    _lib.check("ql_read_gemm_clock", _lib.load().ql_read_gemm_clock(_lib.C.byref(c),
                                                                      _lib.C.byref(t)))
    return c.value, t.value


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
