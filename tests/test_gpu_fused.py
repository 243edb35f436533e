"""nvfp4_linear_single_launch (K % 256 == 0): the GEMM kernel first quantizes the
activations and lays out the row-major weight scales into its workspace with every
warp of the grid, meets at a grid-wide barrier, then multiplies.

Checks, through the C ABI:
  * the codes and block scales the launch leaves in its workspace are bit-exact
    against the oracle's quantization, for CTA-pair and single-CTA tiles;
  * the output equals the two-launch path (quantize, then GEMM) bit for bit;
  * a workspace full of leftover bytes gives the same result, and every
    synchronisation word is back to zero after the call;
  * a CUDA graph that captured the call gives, on each replay, the result of an
    eager call on the replayed input.
The element-wise parity against the fp64 oracle of all shapes, K % 256 == 0 ones
included, is in test_gpu_linear.py.
"""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
from gpu_helpers import Nvfp4Case, check_linear, unpack_act_scale_atoms

pytestmark = pytest.mark.gpu


def _call(d, ws, y=None):
    return q.nvfp4_linear_single_launch(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                          bias=d["bias"], y=y, workspace=ws)


def _act_scale_bytes(M, K):
    KG = -(-K // 256) * 4
    return -(-M // 128) * KG * 512


@pytest.mark.parametrize("M,K,N", [
    (600, 512, 520),    # CTA pairs (256-row blocks), ragged M and N
    (130, 1024, 1536),  # single-CTA tiles (128-row blocks)
    (2048, 3072, 768),  # eight 256-row blocks, K of the diffusion layers
])
def test_workspace_codes_and_scales_bit_exact(M, K, N):
    c = Nvfp4Case(M, K, N, seed=M + 7, bias=True)
    d = c.device_args()
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    y = _call(d, ws)
    torch.cuda.synchronize()
    codes_off, sf_off, _ = q.nvfp4_linear_workspace_layout(M, K, N)
    buf = ws.cpu().numpy()
    xq, xs = c.oracle_act()
    got_q = buf[codes_off:codes_off + M * K // 2].reshape(M, K // 2)
    assert np.array_equal(got_q, xq)
    got_s = unpack_act_scale_atoms(buf[sf_off:sf_off + _act_scale_bytes(M, K)], M, K)
    assert np.array_equal(got_s, xs)
    _, y64, T = c.reference()
    check_linear(y, y64, T, "single-launch nvfp4_linear")


def test_rejects_k_not_multiple_of_256():
    c = Nvfp4Case(128, 288, 256, seed=2)
    d = c.device_args()
    with pytest.raises(q.QLinearError):
        _call(d, None)


def test_equals_two_launch_path_bit_for_bit():
    M, K, N = 1024, 3072, 1536
    c = Nvfp4Case(M, K, N, seed=11, bias=True)
    d = c.device_args()
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    y1 = _call(d, ws)
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws)
    y2 = q.nvfp4_linear_gemm(M, d["w"], d["weight_scale_2"], d["input_scale"], ws, bias=d["bias"])
    y3 = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                        bias=d["bias"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(y1, y3)


@pytest.mark.parametrize("fill", ["ones", "random"])
def test_leftover_workspace_bytes_and_sync_words_reset(fill):
    M, K, N = 777, 1024, 1000
    c = Nvfp4Case(M, K, N, seed=3)
    d = c.device_args()
    size = q.nvfp4_linear_workspace_size(M, K, N)
    if fill == "ones":
        ws = torch.full((size,), 0xFF, dtype=torch.uint8, device="cuda")
    else:
        g = torch.Generator(device="cuda").manual_seed(5)
        ws = torch.randint(0, 256, (size,), dtype=torch.uint8, device="cuda", generator=g)
    clean = torch.zeros(size, dtype=torch.uint8, device="cuda")
    y_dirty = _call(d, ws)
    y_clean = _call(d, clean)
    torch.cuda.synchronize()
    assert torch.equal(y_dirty, y_clean)
    _, y64, T = c.reference()
    check_linear(y_dirty, y64, T, f"workspace filled with {fill}")
    # the synchronisation words sit between the activation scales and the
    # weight-scale atoms; after the call they are all zero again
    _, sf_off, wsf_off = q.nvfp4_linear_workspace_layout(M, K, N)
    sync_start = -(-(sf_off + _act_scale_bytes(M, K)) // 1024) * 1024
    n_words = 8
    words = ws[sync_start:sync_start + 8 * n_words].cpu().numpy()
    assert sync_start + 8 * n_words <= wsf_off
    assert not words.any()


def test_cuda_graph_replay_matches_eager():
    M, K, N = 512, 3072, 3072
    c = Nvfp4Case(M, K, N, seed=21, bias=True)
    d = c.device_args()
    ws = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    x_static = d["x"]
    _call(d, ws, y)  # warm-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _call(d, ws, y)
    g = torch.Generator().manual_seed(9)
    for i in range(3):
        x_new = (torch.randn(M, K, generator=g) * (1.0 + i)).to(torch.bfloat16).cuda()
        x_static.copy_(x_new)
        graph.replay()
        torch.cuda.synchronize()
        y_graph = y.clone()
        ws_eager = torch.empty_like(ws)
        y_eager = _call(dict(d, x=x_new), ws_eager)
        torch.cuda.synchronize()
        assert torch.equal(y_graph, y_eager), f"replay {i}"
    assert q.read_device_status() == 0
