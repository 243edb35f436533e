"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
function include/qlinear.h declares, sizes its workspaces, and rejects bad
arguments with the documented status codes before touching the device."""
import ctypes as C
import os
import re

import pytest

from fp8_rowwise_quantized_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlinear.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([a-z][a-z0-9_]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_functions()
    assert len(names) >= 26, names
    for n in names:
        assert hasattr(lib, n), f"missing export {n}"
    assert set(names) == set(_lib.SIGNATURES), set(names) ^ set(_lib.SIGNATURES)


def test_status_strings():
    lib = _lib.load()
    for code in range(8):
        s = lib.ql_status_string(code).decode()
        assert s and s != "unknown status"
    assert lib.ql_status_string(99).decode() == "unknown status"


def test_workspace_sizes():
    lib = _lib.load()
    M, K, N = 4096, 3072, 12288
    ws = lib.nvfp4_linear_workspace_size(M, K, N)
    # codes M*K/2 + activation scale atoms + weight scale atoms (padded), 1 KB aligned
    assert ws >= M * K // 2 + M * K // 16 + N * K // 16
    assert ws < M * K // 2 + 2 * (M * K // 16) + 2 * (N * K // 16) + 8192
    assert ws % 1024 == 0
    assert lib.nvfp4_linear_workspace_size(M, 48, N) == 0       # K % 32 != 0
    assert lib.nvfp4_linear_workspace_size(0, K, N) == 0
    assert lib.fp8r_linear_workspace_size(4096, 3072, 3072) >= 4096 * 3072 + 4096 * 4
    assert lib.fp8r_linear_workspace_size(4096, 3000, 3072) == 0  # K % 16 != 0
    a, b, c = C.c_size_t(), C.c_size_t(), C.c_size_t()
    assert lib.nvfp4_linear_workspace_layout(M, K, N, C.byref(a), C.byref(b), C.byref(c)) == 0
    assert a.value == 0 and b.value >= M * K // 2 and c.value > b.value and c.value < ws


def test_every_dit_layer_fits_the_noalloc_scratch():
    # nvfp4_linear_noalloc holds 32 MiB of scratch per device; every M = 4096
    # diffusion-transformer layer of the workloads fits in it
    lib = _lib.load()
    for K, N in [(3072, 3072), (3072, 9216), (3072, 12288), (12288, 3072)]:
        need = lib.nvfp4_linear_workspace_size(4096, K, N)
        assert 0 < need <= (32 << 20), (K, N, need)


def test_argument_errors_before_device():
    lib = _lib.load()
    fake = 1 << 20          # aligned, never dereferenced: validation fails first
    odd = fake + 8          # not 16-byte aligned
    M, K, N = 128, 256, 256
    ws = lib.nvfp4_linear_workspace_size(M, K, N)
    # null pointer
    assert lib.nvfp4_linear(None, M, K, fake, fake, N, fake, fake, None, fake, fake, ws, None) == 1
    # non-positive size
    assert lib.nvfp4_linear(fake, 0, K, fake, fake, N, fake, fake, None, fake, fake, ws, None) == 1
    # K not a multiple of 32
    assert lib.nvfp4_linear(fake, M, 48, fake, fake, N, fake, fake, None, fake, fake, ws, None) == 2
    # misaligned output
    assert lib.nvfp4_linear(fake, M, K, fake, fake, N, fake, fake, None, odd, fake, ws, None) == 3
    # workspace too small / missing
    assert lib.nvfp4_linear(fake, M, K, fake, fake, N, fake, fake, None, fake, fake, ws - 1, None) == 5
    assert lib.nvfp4_linear(fake, M, K, fake, fake, N, fake, fake, None, fake, None, ws, None) == 5
    assert lib.fp8r_linear(fake, M, 40, fake, fake, N, None, fake, fake, 1 << 30, None) == 2
    assert lib.fp8r_quantize_rows(fake, M, 12, fake, fake, None) == 2
    assert lib.nvfp4_quantize_act(fake, M, 24, fake, fake, fake, None) == 2
    assert lib.nvfp4_quantize_act(odd, M, K, fake, fake, fake, None) == 3
    assert lib.ql_encode_e4m3(None, fake, 10, None) == 1
    # int4: K % 64, null workspace
    assert lib.int4_quantize_rows(fake, M, 96, fake, fake, None) == 2
    assert lib.int4_linear(fake, M, K, fake, fake, N, None, fake, None, 1 << 20, None) == 5
    assert lib.int4_linear_workspace_size(M, 96, N) == 0
    assert lib.int4_linear_gemm_workspace_size(M, 96, N) == 0
    # GEMM workspace: f16 x [M, K], x row factors [M], f16 w [N, K], w row factors [N],
    # each part 1 KB-aligned
    al = lambda b: -(-b // 1024) * 1024
    gws = al(2 * M * K) + al(4 * M) + al(2 * N * K) + al(4 * N)
    assert lib.int4_linear_gemm_workspace_size(M, K, N) == gws
    # int4_linear: activation codes, then their group scales, then the GEMM workspace
    assert lib.int4_linear_workspace_size(M, K, N) == al(M * K // 2) + al(M * (K // 64) * 4) + gws
    assert lib.int4_linear_workspace_size(3, 64, 1) == 1024 * 6
    assert lib.int4_linear(fake, M, K, fake, fake, N, None, fake, odd, 1 << 30, None) == 3
    # int4_linear_gemm: null pointer, K % 64, workspace, misaligned codes / scales / bias / y
    big = 1 << 30
    assert lib.int4_linear_gemm(None, fake, M, K, fake, fake, N, None, fake, fake, big, None) == 1
    assert lib.int4_linear_gemm(fake, fake, M, K, fake, fake, 0, None, fake, fake, big, None) == 1
    assert lib.int4_linear_gemm(fake, fake, M, 96, fake, fake, N, None, fake, fake, big, None) == 2
    assert lib.int4_linear_gemm(fake, fake, M, K, fake, fake, N, None, fake, None, big, None) == 5
    assert lib.int4_linear_gemm(fake, fake, M, K, fake, fake, N, None, fake, fake, gws - 1, None) == 5
    assert lib.int4_linear_gemm(odd, fake, M, K, fake, fake, N, None, fake, fake, big, None) == 3
    assert lib.int4_linear_gemm(fake, fake, M, K, odd, fake, N, None, fake, fake, big, None) == 3
    assert lib.int4_linear_gemm(fake, fake + 2, M, K, fake, fake, N, None, fake, fake, big, None) == 3
    assert lib.int4_linear_gemm(fake, fake, M, K, fake, fake + 2, N, None, fake, fake, big, None) == 3
    assert lib.int4_linear_gemm(fake, fake, M, K, fake, fake, N, fake + 2, fake, fake, big, None) == 3
    assert lib.int4_linear_gemm(fake, fake, M, K, fake, fake, N, None, fake + 1, fake, big, None) == 3
    assert lib.int4_linear_gemm(fake, fake, M, K, fake, fake, N, None, fake, odd, big, None) == 3
    # weight scales laid out once: sizes, tile widths, workspace and alignment
    assert lib.nvfp4_weight_scale_atoms_size(N, K, 96) == 0
    assert lib.nvfp4_weight_scale_atoms_size(N, 40, 128) == 0
    # atoms: ceil(N / bn) tiles x K/64 groups x ceil(bn / 128) atoms of 512 bytes
    assert lib.nvfp4_weight_scale_atoms_size(N, K, 224) == -(-N // 224) * (K // 64) * 2 * 512
    assert lib.nvfp4_weight_scale_atoms_size(N, K, 128) == -(-N // 128) * (K // 64) * 512
    big = 1 << 30
    assert lib.nvfp4_layout_weight_scales(None, N, K, 128, fake, big, None) == 1
    assert lib.nvfp4_layout_weight_scales(fake, N, K, 96, fake, big, None) == 2
    assert lib.nvfp4_layout_weight_scales(fake, N, K, 128, fake, 16, None) == 5
    assert lib.nvfp4_layout_weight_scales(fake, N, K, 128, odd, big, None) == 3
    assert lib.nvfp4_linear_laid_out(fake, M, K, fake, fake, 100, N, fake, fake, None, fake,
                                     fake, big, None) == 2
    assert lib.nvfp4_linear_laid_out(fake, M, K, fake, odd, 128, N, fake, fake, None, fake,
                                     fake, big, None) == 3
    assert lib.nvfp4_linear_laid_out(fake, M, K, fake, fake, 128, N, fake, fake, None, fake,
                                     fake, 16, None) == 5
    assert lib.nvfp4_linear_laid_out(fake, M, K, fake, None, 128, N, fake, fake, None, fake,
                                     fake, big, None) == 1
    # w4a16: null weight, K % 32, misaligned x, odd w_scale
    assert lib.w4a16_linear(fake, 1, K, None, fake, N, fake, None, fake, None) == 1
    assert lib.w4a16_linear(fake, 1, 48, fake, fake, N, fake, None, fake, None) == 2
    assert lib.w4a16_linear(odd, 1, K, fake, fake, N, fake, None, fake, None) == 3
    assert lib.w4a16_linear(fake, 1, K, fake, fake + 1, N, fake, None, fake, None) == 3


def test_argument_errors_of_the_split_fused_and_extension_calls():
    # every check runs before the device is touched: null pointers (1), shapes (2),
    # alignment (3), workspace (5), in the order each entry point documents
    lib = _lib.load()
    fake, odd, big = 1 << 20, (1 << 20) + 8, 1 << 30
    M, K, N = 128, 256, 256
    al = lambda b: -(-b // 1024) * 1024
    # nvfp4_linear_prologue(x, M, K, w_scale, N, input_scale, workspace, bytes, stream)
    assert lib.nvfp4_linear_prologue(None, M, K, fake, N, fake, fake, big, None) == 1
    assert lib.nvfp4_linear_prologue(fake, M, 40, fake, N, fake, fake, big, None) == 2
    assert lib.nvfp4_linear_prologue(odd, M, K, fake, N, fake, fake, big, None) == 3
    assert lib.nvfp4_linear_prologue(fake, M, K, fake, N, fake, fake, 16, None) == 5
    assert lib.nvfp4_linear_prologue(fake, M, K, fake, N, fake, odd, big, None) == 3
    # nvfp4_linear_gemm(M, K, w, N, weight_scale_2, input_scale, bias, y, workspace, bytes, s)
    assert lib.nvfp4_linear_gemm(M, K, None, N, fake, fake, None, fake, fake, big, None) == 1
    assert lib.nvfp4_linear_gemm(M, K, fake, N, fake, fake, None, odd, fake, big, None) == 3
    assert lib.nvfp4_linear_gemm(M, K, fake, N, fake, fake, odd, fake, fake, big, None) == 3
    assert lib.nvfp4_linear_gemm(M, K, fake, N, fake, fake, None, fake, None, big, None) == 5
    # nvfp4_linear_gemm_lowrank(..., bias, lr_act, lr_up, rank, y, workspace, bytes, s)
    lr = lambda act, rank: lib.nvfp4_linear_gemm_lowrank(M, K, fake, N, fake, fake, None, act,
                                                         fake, rank, fake, fake, big, None)
    assert lr(None, 32) == 1
    assert lr(fake, 12) == 2 and lr(fake, 72) == 2 and lr(fake, 0) == 2
    assert lr(odd, 32) == 3
    # nvfp4_linear_single_launch: K % 256 == 0 and a 16-byte aligned w_scale as well
    sl = lambda k, w_scale, nbytes: lib.nvfp4_linear_single_launch(
        fake, M, k, fake, w_scale, N, fake, fake, None, fake, fake, nbytes, None)
    assert sl(288, fake, big) == 2
    assert sl(K, odd, big) == 3
    assert sl(K, fake, 16) == 5
    # nvfp4_linear_gelu_quantize(x, M, K, w, w_scale, N, ws2, is, bias, next_is,
    #                            next_workspace, next_bytes, workspace, bytes, s)
    gq = lambda n, next_is, next_ws, next_bytes, ws: lib.nvfp4_linear_gelu_quantize(
        fake, M, K, fake, fake, n, fake, fake, None, next_is, next_ws, next_bytes, ws, big, None)
    assert gq(N, None, fake, big, fake) == 1
    assert gq(200, fake, fake, big, fake) == 2             # N % 256 != 0
    assert gq(N, fake, odd, big, fake) == 3
    assert gq(N, fake, fake, 16, fake) == 5
    assert gq(N, fake, fake, big, None) == 5
    # nvfp4_linear_quantized_input(M, K, w, w_scale, N, ws2, is, bias, y, workspace, bytes, s)
    qi = lambda k, ws, nbytes: lib.nvfp4_linear_quantized_input(
        M, k, fake, fake, N, fake, fake, None, fake, ws, nbytes, None)
    assert qi(K, None, big) == 1
    assert qi(48, fake, big) == 2
    assert qi(K, fake, 16) == 5
    assert qi(K, odd, big) == 3
    # svdq_nvfp4_linear(x, M, K, smooth, down, up, rank, w, w_scale, N, ws2, is, bias, y,
    #                   workspace, bytes, s); its workspace adds lr_act bf16 [M, rank]
    need = lib.svdq_nvfp4_linear_workspace_size(M, K, N, 32)
    assert need == lib.nvfp4_linear_workspace_size(M, K, N) + al(M * 32 * 2)
    assert lib.svdq_nvfp4_linear_workspace_size(M, K, N, 4) == 0
    assert lib.svdq_nvfp4_linear_workspace_size(M, K, N, 72) == 0
    sv = lambda smooth, down, rank, nbytes: lib.svdq_nvfp4_linear(
        fake, M, K, smooth, down, fake, rank, fake, fake, N, fake, fake, None, fake, fake, nbytes,
        None)
    assert sv(None, None, 32, big) == 1
    assert sv(None, fake, 30, big) == 2
    assert sv(odd, fake, 32, big) == 3                     # the smoothing vector
    assert sv(None, fake, 32, need - 1) == 5
    # fp8r_linear_gemm(xq, x_scale, M, K, w, w_scale, N, bias, y, s)
    assert lib.fp8r_linear_gemm(None, fake, M, K, fake, fake, N, None, fake, None) == 1
    assert lib.fp8r_linear_gemm(fake, fake, M, 40, fake, fake, N, None, fake, None) == 2
    assert lib.fp8r_linear_gemm(odd, fake, M, K, fake, fake, N, None, fake, None) == 3
    # calibration and the element encoders
    assert lib.nvfp4_global_scale(None, 10, fake, None) == 1
    assert lib.nvfp4_global_scale(fake, 0, fake, None) == 1
    assert lib.ql_encode_e2m1(fake, None, 10, None) == 1
    assert lib.ql_encode_e2m1(fake, fake, 0, None) == 1


def test_no_device_reports_error_instead_of_crashing():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    lib = _lib.load()
    fake = 1 << 20
    rc = lib.nvfp4_quantize_act(fake, 128, 256, fake, fake, fake, None)
    assert rc in (4, 6)           # device check or CUDA error, never a crash
    assert lib.ql_last_error_message().decode()
    st = C.c_int(-1)
    assert lib.ql_read_device_status(C.byref(st)) in (4, 6)


def test_tile_choice_of_the_dit_layers():
    # the cost model's picks for the benchmarked layers (host logic, no device):
    # 256 x 224 CTA-pair tiles for the MLP up projection and the fused QKV, 256 x 256 for
    # the MLP down projection, 256 x 192 for the attention projection; below 512 rows
    # one CTA per 128-row tile; at most 64 rows the skinny kernels with the narrowest
    # width whose tiles fit one wave of 148 SMs
    import fp8_rowwise_quantized_b200 as q
    assert q.tile_config(4096, 12288, 3072) == (224, 2)
    assert q.tile_config(4096, 9216, 3072) == (224, 2)
    assert q.tile_config(4096, 3072, 12288) == (256, 2)
    assert q.tile_config(4096, 3072, 3072) == (192, 2)
    assert q.tile_config(256, 12288, 3072) == (192, 1)
    assert q.tile_config(16, 12288, 3072) == (96, 1)     # 128 tiles
    assert q.tile_config(16, 3072, 3072) == (64, 1)      # 48 tiles
    assert q.tile_config(64, 18432, 3072) == (128, 1)    # 144 tiles
    assert q.tile_config(65, 3072, 3072)[0] >= 128       # 65 rows: no skinny kernel
    for M, N in [(1, 3072), (16, 12288), (64, 18432)]:
        bn, cg = q.tile_config(M, N, 3072)
        assert cg == 1 and -(-N // bn) <= 148


def test_tile_config_is_host_only_and_follows_override():
    import fp8_rowwise_quantized_b200 as q
    bn, cg = q.tile_config(4096, 12288, 3072)
    assert bn in (128, 192, 224, 256) and cg == 2       # 256-row pair tiles once M >= 512
    assert q.tile_config(128, 256, 256)[1] == 1        # one CTA per 128-row tile below that
    q.set_tile_override(192, 1)
    try:
        assert q.tile_config(4096, 12288, 3072) == (192, 1)
    finally:
        q.set_tile_override(0, 0)
    assert q.tile_config(4096, 12288, 3072) == (bn, cg)
    lib = _lib.load()
    assert lib.ql_tile_config(1, 0, 1, 1, None, None) == _lib.QL_ERR_INVALID_ARG


def test_binding_rejects_host_tensors_without_computing():
    # there is no CPU path: every compute call given host tensors raises before any
    # work is done, instead of falling back to another implementation
    import torch
    import fp8_rowwise_quantized_b200 as q
    M, K, N = 16, 256, 128
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    w4 = torch.zeros((N, K // 2), dtype=torch.uint8)
    s4 = torch.zeros((N, K // 16), dtype=torch.uint8)
    one = torch.ones(1, dtype=torch.float32)
    w8 = torch.zeros((N, K), dtype=torch.uint8)
    rows = torch.ones(N, dtype=torch.float32)
    i4s = torch.ones((N, K // 64), dtype=torch.float32)
    down = torch.zeros((32, K), dtype=torch.bfloat16)
    up = torch.zeros((N, 32), dtype=torch.bfloat16)
    nws = torch.zeros(1 << 20, dtype=torch.uint8)
    calls = {
        "nvfp4_quantize_act": lambda: q.nvfp4_quantize_act(x, one),
        "nvfp4_global_scale": lambda: q.nvfp4_global_scale(x),
        "nvfp4_linear": lambda: q.nvfp4_linear(x, w4, s4, one, one),
        "nvfp4_layout_weight_scales": lambda: q.nvfp4_layout_weight_scales(s4, 128),
        "nvfp4_linear_laid_out": lambda: q.nvfp4_linear_laid_out(x, w4, nws, 128, one, one),
        "nvfp4_linear_single_launch": lambda: q.nvfp4_linear_single_launch(x, w4, s4, one, one),
        "nvfp4_linear_noalloc": lambda: q.nvfp4_linear_noalloc(x, w4, s4, one, one),
        "nvfp4_linear_gelu_quantize": lambda: q.nvfp4_linear_gelu_quantize(
            x, w4, s4, one, one, one, nws),
        "nvfp4_linear_quantized_input": lambda: q.nvfp4_linear_quantized_input(
            M, w4, s4, one, one, nws),
        "svdq_nvfp4_linear": lambda: q.svdq_nvfp4_linear(x, w4, s4, one, one, down, up),
        "w4a16_linear": lambda: q.w4a16_linear(x, w4, s4, one),
        "fp8r_quantize_rows": lambda: q.fp8r_quantize_rows(x),
        "fp8r_linear": lambda: q.fp8r_linear(x, w8, rows),
        "int4_quantize_rows": lambda: q.int4_quantize_rows(x),
        "int4_linear": lambda: q.int4_linear(x, w4, i4s),
    }
    for name, call in calls.items():
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
