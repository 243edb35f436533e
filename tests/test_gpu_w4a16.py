"""GPU parity of the W4A16 linear (NVFP4 weights dequantized to bf16, bf16
activations; the modulation-layer kernel family of the Nunchaku page) against the
fp64 oracle, through the C ABI.

  * one-hot activation rows make Y[m, n] the dequantized weight itself, so the
    GPU's dequantization is checked bit for bit against the oracle's;
  * random activations check the whole output with the linear's acceptance bound
    (per element 1e-3 * sum_k |x w| + one bf16 ulp, Frobenius 5e-3): ragged N,
    every row-pass width (M = 1, 2, 3..4, 5..8 and several passes), bias, K from
    one chunk to the MLP width;
  * the modulation-layer sizes (K = 3072, N = 9216 and 18432) in full."""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import bf16_bits, check_linear, scalar_dev, to_dev
from synthetic import make_linear_inputs

pytestmark = pytest.mark.gpu


class W4a16Case:
    def __init__(self, M, K, N, seed=0, bias=False):
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=bias)
        self.M, self.K, self.N = M, K, N
        self.x = inp.x
        self.gw = oracle.nvfp4_global_scale(inp.w)
        self.wq, self.ws = oracle.nvfp4_quantize(inp.w, self.gw)
        self.bias = None if inp.bias is None else inp.bias.numpy()

    def run(self, x=None):
        x = self.x if x is None else x
        y = torch.full((x.shape[0], self.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        q.w4a16_linear(to_dev(x), to_dev(self.wq), to_dev(self.ws), scalar_dev(self.gw),
                       bias=None if self.bias is None else to_dev(self.bias), y=y)
        torch.cuda.synchronize()
        assert bool(torch.isfinite(y).all()), "unwritten or non-finite outputs"
        assert q.read_device_status() == 0
        return y

    def check(self):
        y = self.run()
        _, y64, T = oracle.w4a16_linear(self.x, self.wq, self.ws, self.gw, self.bias)
        return check_linear(y, y64, T, f"w4a16 {self.M}x{self.K}x{self.N}")


def test_w4a16_dequantization_bit_exact_through_one_hot_rows():
    c = W4a16Case(1, 1024, 300, seed=3)
    wb = oracle.w4a16_dequantize_bf16(c.wq, c.ws, c.gw)        # bf16 bits [N, K]
    cols = np.arange(0, c.K, 7)
    x = torch.zeros((len(cols), c.K), dtype=torch.bfloat16)
    x[torch.arange(len(cols)), torch.from_numpy(cols)] = 1.0
    y = bf16_bits(c.run(x))                                     # [len(cols), N]
    # a -0 weight (code 0x8) gives +0 in Y: the fp32 sum starts from +0
    want = wb[:, cols].T.copy()
    want[want == 0x8000] = 0
    assert (wb == 0x8000).any() and (want != 0).mean() > 0.9
    np.testing.assert_array_equal(y, want)


@pytest.mark.parametrize("M,K,N,bias", [
    (1, 32, 1, False),        # one chunk, one output
    (1, 96, 7, True),         # chunks not a multiple of the warp, ragged N
    (2, 1056, 130, False),
    (3, 3072, 515, True),     # row pass of 4 with one row masked
    (4, 512, 64, False),
    (5, 768, 333, True),      # row pass of 8, three rows masked
    (8, 3072, 1000, False),
    (13, 640, 257, True),     # two row passes
    (16, 3072, 384, False),
    (2, 12288, 200, True),    # long rows
])
def test_w4a16_linear_small_full(M, K, N, bias):
    W4a16Case(M, K, N, seed=M + N, bias=bias).check()


@pytest.mark.parametrize("M,N", [(1, 18432), (2, 18432), (1, 9216), (4, 9216)])
def test_w4a16_modulation_sizes_full(M, N):
    W4a16Case(M, 3072, N, seed=N + M, bias=True).check()


def test_w4a16_rejects_bad_arguments():
    x = torch.zeros((2, 48), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((8, 24), dtype=torch.uint8, device="cuda")
    ws = torch.zeros((8, 3), dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QLinearError):
        q.w4a16_linear(x, w, ws, scalar_dev(1.0))  # K % 32 != 0
