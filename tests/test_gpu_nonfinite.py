"""Non-finite activations (NaN, +-Inf) are outside the tested arithmetic: the
layers give them no meaning, but they must not fault, hang or spread. Every row of
x is quantized on its own (NVFP4 blocks, fp8r row scales) and contracts into its
own row of Y, so rows holding NaN or Inf may come out as anything while every
other row is bit for bit the output of the same call on clean input."""
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
from gpu_helpers import Fp8rCase, Nvfp4Case, scalar_dev, to_dev

pytestmark = pytest.mark.gpu

BAD_ROWS = [0, 77, 130, 511]


def poisoned(x):
    xb = x.clone()
    xb[0, 5] = float("nan")
    xb[77, 100] = float("inf")
    xb[130, 3000] = float("-inf")
    xb[511, :] = float("nan")
    return xb


def clean_rows(M):
    keep = torch.ones(M, dtype=torch.bool)
    keep[BAD_ROWS] = False
    return keep.cuda()


def test_nvfp4_linear_nonfinite_rows_stay_in_their_rows():
    c = Nvfp4Case(600, 3072, 1536, seed=21, bias=True)
    d = c.device_args()
    call = lambda x: q.nvfp4_linear(x, d["w"], d["w_scale"], d["weight_scale_2"],
                                    d["input_scale"], bias=d["bias"])
    y_clean = call(d["x"])
    y_bad = call(poisoned(d["x"]))
    torch.cuda.synchronize()
    assert q.read_device_status() == 0
    keep = clean_rows(600)
    assert torch.equal(y_bad[keep], y_clean[keep])


def test_fp8r_linear_nonfinite_rows_stay_in_their_rows():
    c = Fp8rCase(600, 3072, 1536, seed=22, bias=True)
    d = c.device_args()
    call = lambda x: q.fp8r_linear(x, d["w"], d["w_scale"], bias=d["bias"])
    y_clean = call(d["x"])
    y_bad = call(poisoned(d["x"]))
    torch.cuda.synchronize()
    assert q.read_device_status() == 0
    keep = clean_rows(600)
    assert torch.equal(y_bad[keep], y_clean[keep])


def test_w4a16_linear_nonfinite_rows_stay_in_their_rows():
    c = Nvfp4Case(520, 3072, 1000, seed=23)
    x = to_dev(c.x)
    w, ws, g = to_dev(c.wq), to_dev(c.ws), scalar_dev(c.gw)
    y_clean = q.w4a16_linear(x, w, ws, g)
    y_bad = q.w4a16_linear(poisoned(x), w, ws, g)
    torch.cuda.synchronize()
    assert q.read_device_status() == 0
    keep = clean_rows(520)
    assert torch.equal(y_bad[keep], y_clean[keep])
