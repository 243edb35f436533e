"""GPU parity of the NVFP4 and fp8r linear layers (tensor-core GEMMs) against the
fp64 oracle, through the C ABI. Small shapes are compared element by element in
full (several tiles plus ragged tails in M, N and K; every tile width); the
full diffusion-transformer sizes are compared on sampled rows, with properties
that hold at any size checked on the whole output."""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import (Fp8rCase, Nvfp4Case, bf16_bits, check_linear, sample_rows, scalar_dev,
                         to_dev)

pytestmark = pytest.mark.gpu


def nan_output(M, N):
    # every element must be written: start from NaN and require all finite after
    return torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")


def run_nvfp4(c: Nvfp4Case, rows=None, workspace=None):
    d = c.device_args()
    y = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                       bias=d["bias"], y=nan_output(c.M, c.N), workspace=workspace)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y).all()), "unwritten or non-finite outputs"
    y_ref, y64, T = c.reference(rows)
    yc = y if rows is None else y[torch.from_numpy(rows).cuda()]
    return y, check_linear(yc, y64, T, f"nvfp4 {c.M}x{c.K}x{c.N}")


@pytest.mark.parametrize("M,K,N", [
    (128, 256, 256),     # the tiny layer: 2 N tiles
    (1, 32, 8),          # smallest K, one row, narrow N
    (17, 96, 136),       # ragged everything; K not a multiple of 256
    (200, 288, 392),     # two M tiles, partial K tile
    (256, 512, 384),     # tile width 128, three N tiles
    (130, 1024, 1536),   # tile width 192
    (300, 768, 4096),    # tile width 256 (single TMEM accumulator)
    (64, 3072, 200),     # N not a multiple of 8 -> scalar tail stores
    (512, 256, 384),     # CTA-pair tiles (M >= 512), exact fit
    (600, 512, 520),     # CTA pair: last pair tile half empty (follower rows all out)
    (777, 1056, 1000),   # CTA pair, ragged M, N and K
    (1024, 768, 1536),   # CTA pair, tile width 192
    (520, 512, 4096),    # CTA pair, tile width 256 (single TMEM accumulator)
])
def test_nvfp4_linear_small_full(M, K, N):
    run_nvfp4(Nvfp4Case(M, K, N, seed=M + N))


def test_nvfp4_linear_tiny_with_bias_and_saturation():
    run_nvfp4(Nvfp4Case(128, 256, 256, seed=0, bias=True))
    run_nvfp4(Nvfp4Case(128, 256, 256, seed=1, input_scale_div=4.0))


@pytest.mark.parametrize("name,M,K,N,bias", [
    ("attn_proj", 4096, 3072, 3072, True),
    ("attn_qkv", 4096, 3072, 9216, True),
    ("mlp_up", 4096, 3072, 12288, False),
])
def test_nvfp4_linear_dit_sizes_sampled(name, M, K, N, bias):
    c = Nvfp4Case(M, K, N, seed=0, bias=bias)
    rows = sample_rows(M, 20, seed=1)
    y, frob = run_nvfp4(c, rows)
    # whole output: written (finite, checked in run_nvfp4), of the expected
    # magnitude and nonzero almost everywhere (the sampled rows carry the exact check)
    yb = oracle.bf16_bits_to_f64(bf16_bits(y))
    assert np.abs(yb).max() < 1e4 and (yb != 0).mean() > 0.99


# Skinny / batched sweep of the layer at K = 3072: a few text tokens up to four
# 4096-token latents, with the attention-projection and MLP-up widths.
@pytest.mark.parametrize("M,N", [(16, 3072), (16, 12288), (256, 3072), (256, 12288)])
def test_nvfp4_linear_skinny_full(M, N):
    run_nvfp4(Nvfp4Case(M, 3072, N, seed=M + N))


@pytest.mark.parametrize("M,N", [(1024, 3072), (1024, 12288), (8192, 3072), (8192, 12288),
                                 (16384, 3072), (16384, 12288)])
def test_nvfp4_linear_batched_sampled(M, N):
    c = Nvfp4Case(M, 3072, N, seed=M + N)
    y, _ = run_nvfp4(c, sample_rows(M, 16, seed=M))
    yb = oracle.bf16_bits_to_f64(bf16_bits(y))
    assert np.abs(yb).max() < 1e4 and (yb != 0).mean() > 0.99


# Skinny kernels (M <= 64): stages hold only 16 / 32 / 64 rows of A, tiles of 64, 96
# or 128 columns on one CTA; every combination through the tile override, with
# ragged M, N and K and a bias.
@pytest.mark.parametrize("bn", [64, 96, 128])
@pytest.mark.parametrize("M", [1, 16, 17, 32, 40, 64])
def test_nvfp4_linear_skinny_kernels_full(bn, M):
    q.set_tile_override(bn, 1)
    try:
        assert q.tile_config(M, 1000, 800) == (bn, 1)
        run_nvfp4(Nvfp4Case(M, 800, 1000, seed=M + bn, bias=True))
    finally:
        q.set_tile_override(0, 0)


def test_skinny_choice_keeps_one_wave():
    # the automatic choice for M <= 64: the narrowest width whose tiles fit 148 SMs
    assert q.tile_config(16, 12288, 3072) == (96, 1)
    assert q.tile_config(16, 3072, 3072) == (64, 1)
    assert q.tile_config(64, 18432, 3072) == (128, 1)


def test_nvfp4_mlp_down_from_gelu_of_up():
    # the down projection's input is GELU of the up projection's GPU output,
    # re-quantized at run time with a re-calibrated input scale
    up = Nvfp4Case(4096, 3072, 12288, seed=0)
    d = up.device_args()
    y_up = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"])
    h = torch.nn.functional.gelu(y_up.float()).to(torch.bfloat16).cpu()
    down = Nvfp4Case(4096, 12288, 3072, seed=1, x=h)
    run_nvfp4(down, sample_rows(4096, 20, seed=2))


def test_nvfp4_linear_split_calls_match_fused():
    c = Nvfp4Case(512, 3072, 3072, seed=5, bias=True)
    d = c.device_args()
    ws = torch.empty(q.nvfp4_linear_workspace_size(512, 3072, 3072), dtype=torch.uint8,
                     device="cuda")
    y1 = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                        bias=d["bias"], workspace=ws)
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws)
    y2 = q.nvfp4_linear_gemm(512, d["w"], d["weight_scale_2"], d["input_scale"], ws,
                             bias=d["bias"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)  # same kernels, same order: bit-identical


@pytest.mark.parametrize("M", [16, 40])
def test_skinny_linear_matches_split_calls(M):
    # nvfp4_linear lays out the weight scales inside the skinny GEMM; the split
    # prologue + GEMM calls take them from the workspace: same bits
    c = Nvfp4Case(M, 3072, 3072, seed=M, bias=True)
    d = c.device_args()
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, 3072, 3072), dtype=torch.uint8,
                     device="cuda")
    y1 = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                        bias=d["bias"], workspace=ws)
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws)
    y2 = q.nvfp4_linear_gemm(M, d["w"], d["weight_scale_2"], d["input_scale"], ws,
                             bias=d["bias"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    _, y64, T = c.reference()
    check_linear(y1, y64, T, "skinny nvfp4_linear")


@pytest.mark.parametrize("M,K,bn", [(1, 800, 64), (17, 800, 96), (40, 3072, 128),
                                    (64, 800, 128), (16, 3072, 0)])
def test_skinny_linear_leaves_the_quantized_activations(M, K, bn):
    # the skinny layer quantizes its activations inside the GEMM (one launch); the
    # CTAs of the first column of tiles leave the codes and scale atoms in the
    # workspace: the codes are the oracle's, and codes and atoms are byte for byte
    # what nvfp4_linear_prologue writes (ragged K: 800 is not a multiple of 256)
    N = 1000
    if bn:
        q.set_tile_override(bn, 1)
    try:
        c = Nvfp4Case(M, K, N, seed=M + K, bias=True)
        d = c.device_args()
        n = q.nvfp4_linear_workspace_size(M, K, N)
        codes_off, sf_off, wgt_off = q.nvfp4_linear_workspace_layout(M, K, N)
        ws1 = torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda")
        ws2 = ws1.clone()
        y = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                           bias=d["bias"], workspace=ws1)
        q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws2)
        torch.cuda.synchronize()
    finally:
        q.set_tile_override(0, 0)
    xq, _ = c.oracle_act()
    n_codes = M * (K // 2)
    assert np.array_equal(ws1[codes_off:codes_off + n_codes].cpu().numpy(), xq.reshape(-1))
    kg = (K + 255) // 256 * 4
    n_atoms = (M + 127) // 128 * kg * 512
    assert sf_off + n_atoms <= wgt_off
    assert torch.equal(ws1[sf_off:sf_off + n_atoms], ws2[sf_off:sf_off + n_atoms])
    assert torch.equal(ws1[codes_off:codes_off + n_codes], ws2[codes_off:codes_off + n_codes])
    _, y64, T = c.reference()
    check_linear(y, y64, T, "skinny nvfp4_linear, one launch")


def test_skinny_layer_output_feeds_the_next_layer_at_once():
    # a skinny GEMM lets the next kernel on the stream launch at its start; the next
    # layer's prologue must still read this layer's finished output. Two skinny layers
    # back to back, no synchronisation between them, the first output starting as NaN.
    from synthetic import make_linear_inputs
    M, K1, N1, N2 = 16, 256, 512, 256
    assert q.tile_config(M, N1, K1)[0] < 128 and q.tile_config(M, N2, N1)[0] < 128
    inp1 = make_linear_inputs(M, K1, N1, seed=21)
    inp2 = make_linear_inputs(M, N1, N2, seed=22)
    g1 = oracle.nvfp4_global_scale(inp1.w)
    w1q, w1s = oracle.nvfp4_quantize(inp1.w, g1)
    g2 = oracle.nvfp4_global_scale(inp2.w)
    w2q, w2s = oracle.nvfp4_quantize(inp2.w, g2)
    gx1 = oracle.nvfp4_global_scale(inp1.x)
    # the second layer's input scale: calibrated on the oracle's first-layer output
    xq1, xs1 = oracle.nvfp4_quantize(inp1.x, gx1)
    y1_ref, _, _ = oracle.nvfp4_linear(xq1, xs1, w1q, w1s, gx1, g1)
    gx2 = oracle.nvfp4_global_scale(torch.from_numpy(y1_ref.view(np.int16)).view(torch.bfloat16))
    x1 = to_dev(inp1.x)
    d1 = dict(w=to_dev(w1q), w_scale=to_dev(w1s), weight_scale_2=scalar_dev(g1),
              input_scale=scalar_dev(float(gx1)))
    d2 = dict(w=to_dev(w2q), w_scale=to_dev(w2s), weight_scale_2=scalar_dev(g2),
              input_scale=scalar_dev(float(gx2)))
    for _ in range(3):
        y1 = nan_output(M, N1)
        y2 = nan_output(M, N2)
        q.nvfp4_linear(x1, d1["w"], d1["w_scale"], d1["weight_scale_2"], d1["input_scale"], y=y1)
        q.nvfp4_linear(y1, d2["w"], d2["w_scale"], d2["weight_scale_2"], d2["input_scale"], y=y2)
        torch.cuda.synchronize()
        assert bool(torch.isfinite(y1).all()) and bool(torch.isfinite(y2).all())
        # the second layer against the oracle on the first layer's actual output
        xq2, xs2 = oracle.nvfp4_quantize(y1.cpu(), gx2)
        _, y64, T = oracle.nvfp4_linear(xq2, xs2, w2q, w2s, gx2, g2)
        check_linear(y2, y64, T, "second skinny layer")
    assert q.read_device_status() == 0


def test_nvfp4_linear_repeatable():
    c = Nvfp4Case(1024, 3072, 3072, seed=6)
    d = c.device_args()
    ys = [q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"])
          for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def run_fp8r(c: Fp8rCase, rows=None):
    d = c.device_args()
    y = q.fp8r_linear(d["x"], d["w"], d["w_scale"], bias=d["bias"], y=nan_output(c.M, c.N))
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y).all()), "unwritten or non-finite outputs"
    y_ref, y64, T = c.reference(rows)
    yc = y if rows is None else y[torch.from_numpy(rows).cuda()]
    return y, check_linear(yc, y64, T, f"fp8r {c.M}x{c.K}x{c.N}")


@pytest.mark.parametrize("M,K,N,bias", [
    (128, 256, 256, False),
    (1, 16, 8, True),
    (77, 208, 136, True),
    (200, 400, 392, False),
    (130, 1024, 1536, True),
    (300, 768, 4096, False),
    (64, 512, 200, False),
    (600, 400, 520, True),     # CTA pair, ragged
    (1000, 1024, 1536, False),  # CTA pair, tile width 192
    (520, 256, 4096, True),    # CTA pair, tile width 256
])
def test_fp8r_linear_small_full(M, K, N, bias):
    run_fp8r(Fp8rCase(M, K, N, seed=M + K, bias=bias))


def test_fp8r_linear_4096x3072x3072_sampled():
    c = Fp8rCase(4096, 3072, 3072, seed=0)
    y, _ = run_fp8r(c, sample_rows(4096, 24, seed=3))
    yb = oracle.bf16_bits_to_f64(bf16_bits(y))
    assert (yb != 0).mean() > 0.99


def test_fp8r_gemm_from_prequantized_matches_linear():
    c = Fp8rCase(256, 3072, 3072, seed=4, bias=True)
    d = c.device_args()
    y1 = q.fp8r_linear(d["x"], d["w"], d["w_scale"], bias=d["bias"])
    xq, xs = q.fp8r_quantize_rows(d["x"])
    y2 = q.fp8r_linear_gemm(xq, xs, d["w"], d["w_scale"], bias=d["bias"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


TILES = [(128, 1), (192, 1), (224, 1), (256, 1), (128, 2), (192, 2), (224, 2), (256, 2)]


@pytest.mark.parametrize("bn,cg", TILES)
def test_nvfp4_linear_every_tile_config(bn, cg):
    # ragged in M, N and K for every tile width and for one SM or a CTA pair,
    # including the 256-column tile whose two TMEM buffers share a slab
    try:
        q.set_tile_override(bn, cg)
        run_nvfp4(Nvfp4Case(700, 1280, 1000, seed=bn + cg, bias=True))
        run_nvfp4(Nvfp4Case(1536, 3072, 3072, seed=3), sample_rows(1536, 8, seed=bn))
    finally:
        q.set_tile_override(0, 0)


@pytest.mark.parametrize("bn,cg", TILES)
def test_fp8r_linear_every_tile_config(bn, cg):
    try:
        q.set_tile_override(bn, cg)
        run_fp8r(Fp8rCase(700, 1024, 1000, seed=bn * cg, bias=True))
    finally:
        q.set_tile_override(0, 0)


def test_tile_override_rejects_bad_values():
    for bn, cg in [(80, 1), (96, 2), (64, 2), (128, 3), (320, 1)]:
        with pytest.raises(q.QLinearError):
            q.set_tile_override(bn, cg)


# ----------------------------------------------------------------------------- weight scales laid out once

def _laid_out_vs_linear(M, K, N, bn, seed, bias):
    c = Nvfp4Case(M, K, N, seed=seed, bias=bias)
    d = c.device_args()
    cg = 2 if M >= 512 else 1
    q.set_tile_override(bn, cg)
    try:
        y_ref = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                               d["input_scale"], bias=d["bias"])
    finally:
        q.set_tile_override(0, 0)
    atoms = q.nvfp4_layout_weight_scales(d["w_scale"], bn)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    q.nvfp4_linear_laid_out(d["x"], d["w"], atoms, bn, d["weight_scale_2"], d["input_scale"],
                            bias=d["bias"], y=y)
    torch.cuda.synchronize()
    assert q.read_device_status() == 0
    return c, y, y_ref


@pytest.mark.parametrize("bn", [128, 192, 224, 256])
def test_laid_out_weight_scales_same_bits_as_nvfp4_linear(bn):
    # CTA pairs, ragged M and N; the same tile width through nvfp4_linear (which lays
    # the scales out per call) and through the atoms laid out once
    c, y, y_ref = _laid_out_vs_linear(600, 768, 520, bn, seed=bn, bias=True)
    assert torch.equal(y, y_ref)
    _, y64, T = c.reference()
    check_linear(y, y64, T, f"nvfp4_linear_laid_out bn={bn}")


@pytest.mark.parametrize("M", [17, 300])
def test_laid_out_single_cta_tiles(M):
    # one CTA per tile (M < 512), including a lone tile with fewer than 128 rows
    c, y, y_ref = _laid_out_vs_linear(M, 1024, 1000, 192, seed=M, bias=False)
    assert torch.equal(y, y_ref)
    _, y64, T = c.reference()
    check_linear(y, y64, T, f"nvfp4_linear_laid_out M={M}")


def test_laid_out_atoms_equal_the_workspace_atoms():
    # the atoms laid out once are byte for byte the weight part nvfp4_linear_prologue
    # writes into its workspace for the same tile width
    M, K, N = 4096, 3072, 12288
    c = Nvfp4Case(256, K, N, seed=4)
    d = c.device_args()
    bn, _ = q.tile_config(M, N, K)
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    q.nvfp4_linear_prologue(x, d["w_scale"], d["input_scale"], ws)
    _, _, wgt_off = q.nvfp4_linear_workspace_layout(M, K, N)
    atoms = q.nvfp4_layout_weight_scales(d["w_scale"], bn)
    torch.cuda.synchronize()
    n = q.nvfp4_weight_scale_atoms_size(N, K, bn)
    assert atoms.numel() == n
    assert torch.equal(ws[wgt_off:wgt_off + n], atoms)
