"""GPU parity of the INT4 W4A4 linear (the INT4 variant of the Nunchaku page's
4-bit layer; reading: signed 4-bit codes, one fp32 scale = amax / 7 per 64-element
group) against the oracle, through the C ABI: codes and group scales bit-exact; the
linear within the acceptance bound of the other layers (per element 1e-3 * T plus
one bf16 ulp, Frobenius 5e-3), small shapes in full with ragged M and N, the
diffusion-transformer sizes on sampled rows."""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import check_linear, sample_rows, to_dev
from synthetic import make_linear_inputs

pytestmark = pytest.mark.gpu


class Int4Case:
    def __init__(self, M, K, N, seed=0, bias=False):
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=bias)
        self.M, self.K, self.N = M, K, N
        self.x = inp.x
        self.wq, self.ws = oracle.int4_quantize(inp.w)
        self.bias = None if inp.bias is None else inp.bias.numpy()

    def run(self):
        y = torch.full((self.M, self.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        q.int4_linear(to_dev(self.x), to_dev(self.wq), to_dev(self.ws),
                      bias=None if self.bias is None else to_dev(self.bias), y=y)
        torch.cuda.synchronize()
        assert bool(torch.isfinite(y).all()), "unwritten or non-finite outputs"
        assert q.read_device_status() == 0
        return y

    def reference(self, rows=None):
        xq, xs = oracle.int4_quantize(self.x)
        if rows is not None:
            xq, xs = xq[rows], xs[rows]
        return oracle.int4_linear(xq, xs, self.wq, self.ws, self.bias)


@pytest.mark.parametrize("M,K", [(1, 64), (7, 128), (130, 3072), (513, 1024)])
def test_int4_quantize_bit_exact(M, K):
    g = torch.Generator().manual_seed(M + K)
    x = torch.randn(M, K, generator=g)
    x[:, ::37] *= 30.0
    if M > 2:
        x[1] = 0.0                      # a zero row: scale 0, codes 0
        x[2, :64] = 0.0                 # a zero group
    x = x.to(torch.bfloat16)
    qg, sg = q.int4_quantize_rows(x.cuda())
    torch.cuda.synchronize()
    qo, so = oracle.int4_quantize(x)
    np.testing.assert_array_equal(sg.cpu().numpy(), so)
    np.testing.assert_array_equal(qg.cpu().numpy(), qo)


@pytest.mark.parametrize("M,K,N,bias", [
    (1, 64, 8, False),        # one group, one row
    (17, 192, 130, True),     # ragged M and N, three groups
    (130, 1024, 257, True),   # two row tiles, three column tiles
    (256, 3072, 384, False),
])
def test_int4_linear_small_full(M, K, N, bias):
    c = Int4Case(M, K, N, seed=M + N, bias=bias)
    y = c.run()
    _, y64, T = c.reference()
    check_linear(y, y64, T, f"int4 {M}x{K}x{N}")


@pytest.mark.parametrize("M,K,N,bias", [(4096, 3072, 3072, True), (4096, 3072, 12288, False)])
def test_int4_linear_dit_sizes_sampled(M, K, N, bias):
    c = Int4Case(M, K, N, seed=1, bias=bias)
    y = c.run()
    rows = sample_rows(M, 12, seed=2)
    _, y64, T = c.reference(rows)
    check_linear(y[torch.from_numpy(rows).cuda()], y64, T, f"int4 {M}x{K}x{N}")


def test_int4_gemm_from_prequantized_matches_linear():
    c = Int4Case(300, 1024, 520, seed=3, bias=True)
    x = to_dev(c.x)
    y1 = c.run()
    xq, xs = q.int4_quantize_rows(x)
    y2 = q.int4_linear_gemm(xq, xs, to_dev(c.wq), to_dev(c.ws), bias=to_dev(c.bias))
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_int4_rejects_k_not_multiple_of_64():
    x = torch.zeros((4, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q.QLinearError):
        q.int4_quantize_rows(x)


def test_int4_linear_odd_groups_ragged_tiles():
    # nine 64-element groups (the last two-group pipeline stage holds one), three row
    # tiles and five column tiles of 128, ragged in both
    c = Int4Case(300, 576, 520, seed=5, bias=True)
    y = c.run()
    _, y64, T = c.reference()
    check_linear(y, y64, T, "int4 300x576x520")


def test_int4_gemm_unaligned_output_matches_aligned():
    # an output that is not 16-byte aligned takes the element-wise store path; it must
    # give the same bits and write nothing outside Y
    M, K, N = 200, 320, 264
    c = Int4Case(M, K, N, seed=6, bias=True)
    xq, xs = q.int4_quantize_rows(to_dev(c.x))
    w, ws, b = to_dev(c.wq), to_dev(c.ws), to_dev(c.bias)
    y1 = q.int4_linear_gemm(xq, xs, w, ws, bias=b)
    buf = torch.full((M * N + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    y2 = buf[1:1 + M * N].view(M, N)
    q.int4_linear_gemm(xq, xs, w, ws, bias=b, y=y2)
    torch.cuda.synchronize()
    assert y2.data_ptr() % 16 != 0
    assert torch.equal(y1, y2)
    assert bool(torch.isnan(buf[:1]).all()) and bool(torch.isnan(buf[1 + M * N:]).all())
    _, y64, T = c.reference()
    check_linear(y1, y64, T, "int4 200x320x264")


def _f16_operand(codes, scales, K):
    """numpy statement of the GEMM's f16 operand: per row e = E - 12 for the largest
    group scale m 2^E (m in [0.5, 1)), values RN16(RN32(q * (s * 2^-e))), factor 2^e."""
    rows = codes.shape[0]
    lo = (codes.astype(np.int16) << 12).astype(np.int16) >> 12
    hi = (codes.astype(np.int16) << 8).astype(np.int16) >> 12
    qv = np.empty((rows, K), dtype=np.float32)
    qv[:, 0::2] = lo
    qv[:, 1::2] = hi
    mx = np.abs(scales).max(axis=1)
    e = np.where(mx > 0, np.frexp(mx)[1] - 12, 0).astype(np.int32)
    s_scaled = np.ldexp(scales.astype(np.float64), -e[:, None]).astype(np.float32)
    vals = (qv * np.repeat(s_scaled, 64, axis=1)).astype(np.float32).astype(np.float16)
    return vals, np.ldexp(np.float32(1.0), e).astype(np.float32)


def test_int4_gemm_f16_operands_bit_exact():
    # the workspace of int4_linear_gemm holds f16 x [M, K], x factors [M], f16 w [N, K],
    # w factors [N] (1 KB-aligned parts); both dequantizations match numpy bit for bit,
    # including a zero row and a row whose groups span 2^30 in scale
    M, K, N = 70, 320, 130
    c = Int4Case(M, K, N, seed=8)
    x = c.x.clone()
    x[3] = 0
    x[5] = x[5] * torch.logspace(-9, 0, K, base=10.0).to(torch.bfloat16)
    x = x.to(torch.bfloat16)
    xq, xs = q.int4_quantize_rows(to_dev(x))
    ws = torch.empty(q.int4_linear_gemm_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    q.int4_linear_gemm(xq, xs, to_dev(c.wq), to_dev(c.ws), workspace=ws)
    torch.cuda.synchronize()
    al = lambda b: -(-b // 1024) * 1024
    buf = ws.cpu().numpy()
    o = 0
    xh = buf[o:o + 2 * M * K].view(np.float16).reshape(M, K); o += al(2 * M * K)
    xf = buf[o:o + 4 * M].view(np.float32); o += al(4 * M)
    wh = buf[o:o + 2 * N * K].view(np.float16).reshape(N, K); o += al(2 * N * K)
    wf = buf[o:o + 4 * N].view(np.float32)
    ex, efx = _f16_operand(xq.cpu().numpy(), xs.cpu().numpy(), K)
    ew, efw = _f16_operand(c.wq, c.ws, K)
    np.testing.assert_array_equal(xh.view(np.uint16), ex.view(np.uint16))
    np.testing.assert_array_equal(xf, efx)
    np.testing.assert_array_equal(wh.view(np.uint16), ew.view(np.uint16))
    np.testing.assert_array_equal(wf, efw)
    assert np.abs(xh.astype(np.float32)).max() < 2.0 ** 15


def test_int4_linear_same_sign_products():
    # every product x w >= 0, so the operands' rounding errors cannot cancel in sign:
    # the result still meets the linear's bound (each product within 2^-10 of exact)
    M, K, N = 256, 3072, 256
    g = torch.Generator().manual_seed(9)
    c = Int4Case(M, K, N, seed=9)
    c.x = (torch.rand(M, K, generator=g) * 4.0).to(torch.bfloat16)
    w = (torch.rand(N, K, generator=g) * 0.05).to(torch.bfloat16)
    c.wq, c.ws = oracle.int4_quantize(w)
    y = c.run()
    _, y64, T = c.reference()
    check_linear(y, y64, T, "int4 same-sign 256x3072x256")
