"""GPU parity of the quantization kernels against the oracle (bit-exact), through
the C ABI: element encoders (exhaustive over the ranges where codes change),
NVFP4 activation quantization, the prologue's workspace contents, FP8 row-wise
quantization and the calibration reduction."""
import numpy as np
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
import oracle
from gpu_helpers import Nvfp4Case, scalar_dev, to_dev, unpack_act_scale_atoms
from synthetic import make_activations, make_linear_inputs

pytestmark = pytest.mark.gpu


def _bits_ranges(lo: float, hi: float):
    """fp32 bit patterns of [lo, hi) for positive lo < hi, and the negatives."""
    a = int(np.float32(lo).view(np.uint32))
    b = int(np.float32(hi).view(np.uint32))
    return [(a, b - a), (a | 0x80000000, b - a)]


def _compare_encoder(first, count, fmt, chunk=1 << 25):
    enc_gpu = q.ql_encode_e2m1 if fmt == "e2m1" else q.ql_encode_e4m3
    enc_ref = oracle.e2m1_encode_bits_range if fmt == "e2m1" else oracle.e4m3_encode_bits_range
    done = 0
    while done < count:
        n = min(chunk, count - done)
        start = first + done
        bits = torch.arange(start, start + n, dtype=torch.int64, device="cuda")
        v = bits.to(torch.int32, copy=False) if start + n < (1 << 31) else (bits - (1 << 32)).to(torch.int32)
        got = enc_gpu(v.view(torch.float32)).cpu().numpy()
        ref = enc_ref(start, n)
        bad = np.nonzero(got != ref)[0]
        if bad.size:
            i = bad[0]
            b = np.uint32(start + i)
            raise AssertionError(f"{fmt}: {bad.size} mismatches in chunk at {start:#x}; first "
                                 f"{float(b.view(np.float32))!r} ({int(b):#010x}) gpu {got[i]:#x} "
                                 f"oracle {ref[i]:#x}")
        done += n


def test_encoders_exhaustive_where_codes_change():
    # every fp32 with 2^-11 <= |v| < 2^10 (E4M3: all codes, ties, saturation onset)
    for first, count in _bits_ranges(2.0 ** -11, 2.0 ** 10):
        _compare_encoder(first, count, "e4m3")
    # every fp32 with 2^-4 <= |v| < 2^4 (E2M1: all codes, ties, saturation onset)
    for first, count in _bits_ranges(2.0 ** -4, 2.0 ** 4):
        _compare_encoder(first, count, "e2m1")


def test_encoders_strided_elsewhere():
    # the rest of the finite range, every 4099th pattern, plus zeros and extremes
    for fmt in ("e4m3", "e2m1"):
        bits = np.arange(0, 0x7F800000, 4099, dtype=np.uint32)
        bits = np.concatenate([bits, np.uint32([0, 1, 0x7F7FFFFF, 0x00800000])])
        bits = np.concatenate([bits, bits | np.uint32(0x80000000)])
        v = bits.view(np.float32)
        enc_gpu = q.ql_encode_e2m1 if fmt == "e2m1" else q.ql_encode_e4m3
        enc_ref = oracle.e2m1_encode if fmt == "e2m1" else oracle.e4m3_encode
        got = enc_gpu(to_dev(v)).cpu().numpy()
        ref = enc_ref(v)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, (fmt, [(float(v[i]), hex(got[i]), hex(ref[i])) for i in bad[:8]])


@pytest.mark.parametrize("M,K", [(128, 256), (1, 16), (3, 48), (127, 272), (129, 1040),
                                 (4096, 3072), (4096, 12288)])
def test_nvfp4_quantize_act_bit_exact(M, K):
    x = make_activations(M, K, seed=M + K)
    g = oracle.nvfp4_global_scale(x)
    xq_ref, xs_ref = oracle.nvfp4_quantize(x, g)
    xq, xs = q.nvfp4_quantize_act(to_dev(x), scalar_dev(g))
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(xs.cpu().numpy(), xs_ref)


def test_nvfp4_quantize_saturating_and_zero_rows():
    M, K = 64, 512
    x = make_activations(M, K, seed=3)
    x[5] = 0.0
    x[6, :16] = -0.0
    g = oracle.nvfp4_global_scale(x) / 4  # activations beyond the calibration
    xq_ref, xs_ref = oracle.nvfp4_quantize(x, g)
    assert (xs_ref == 0x7E).any()
    xq, xs = q.nvfp4_quantize_act(to_dev(x), scalar_dev(g))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(xs.cpu().numpy(), xs_ref)


def test_nvfp4_quantize_weight_on_gpu_matches_oracle():
    inp = make_linear_inputs(16, 3072, 3072, seed=1)
    wq, ws, g = q.prepare_nvfp4_weight(to_dev(inp.w))
    g_ref = oracle.nvfp4_global_scale(inp.w)
    assert g.item() == np.float32(g_ref)
    wq_ref, ws_ref = oracle.nvfp4_quantize(inp.w, g_ref)
    assert np.array_equal(wq.cpu().numpy(), wq_ref)
    assert np.array_equal(ws.cpu().numpy(), ws_ref)


@pytest.mark.parametrize("M,K,N", [(128, 256, 256), (200, 288, 392), (4096, 3072, 12288)])
def test_nvfp4_prologue_workspace_codes_bit_exact(M, K, N):
    c = Nvfp4Case(M, K, N, seed=2)
    d = c.device_args()
    ws = torch.zeros(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    q.nvfp4_linear_prologue(d["x"], d["w_scale"], d["input_scale"], ws)
    torch.cuda.synchronize()
    codes_off, act_off, _ = q.nvfp4_linear_workspace_layout(M, K, N)
    buf = ws.cpu().numpy()
    xq_ref, xs_ref = c.oracle_act()
    assert np.array_equal(buf[codes_off:codes_off + M * K // 2].reshape(M, K // 2), xq_ref)
    assert np.array_equal(unpack_act_scale_atoms(buf[act_off:], M, K), xs_ref)


@pytest.mark.parametrize("M,K", [(4096, 3072), (1, 8), (33, 200), (300, 12288)])
def test_fp8r_quantize_rows_bit_exact(M, K):
    x = make_activations(M, K, seed=M * 7 + K)
    if M > 2:
        x[2] = 0.0
    xq_ref, s_ref = oracle.fp8r_quantize_rows(x)
    xq, s = q.fp8r_quantize_rows(to_dev(x))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)


def test_global_scale_matches_oracle():
    x = make_activations(4096, 3072, seed=9)
    got = q.nvfp4_global_scale(to_dev(x)).item()
    assert np.float32(got) == np.float32(oracle.nvfp4_global_scale(x))
