"""nvfp4_linear_noalloc: the NVFP4 linear for callers that cannot allocate device
memory (a plugin whose host owns all device memory, a serving loop that must not
enter the allocator, a C caller without a memory manager). It runs the same
kernels as nvfp4_linear on a fixed scratch array inside the library instead of a
caller workspace.

Checks, through the C ABI: two calls in a row (different layer sizes, so the
second call reuses scratch the first one filled) each agree with nvfp4_linear on
the same inputs, within the tolerance of the other parity tests (against the
fp64 oracle) and bit for bit; a problem that needs more scratch than the array
holds is rejected with QL_ERR_WORKSPACE. This file is collected last so that a
run that stops at the first failure has run every other test; it passes in a
fresh process as well as after them.
"""
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
from fp8_rowwise_quantized_b200 import _lib
from gpu_helpers import Nvfp4Case, check_linear

pytestmark = pytest.mark.gpu


def _nan_output(M, N):
    return torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")


def test_noalloc_matches_nvfp4_linear_on_two_calls_in_a_row():
    cases = [Nvfp4Case(1024, 3072, 3072, seed=31, bias=True), Nvfp4Case(200, 288, 392, seed=32)]
    args = [c.device_args() for c in cases]
    # the entry point with a caller workspace, for reference
    refs = [q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                           bias=d["bias"]) for d in args]
    # two calls in a row of the entry point without one
    outs = []
    for c, d in zip(cases, args):
        outs.append(q.nvfp4_linear_noalloc(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                                           d["input_scale"], bias=d["bias"],
                                           y=_nan_output(c.M, c.N)))
    torch.cuda.synchronize()
    for c, ref, out in zip(cases, refs, outs):
        assert bool(torch.isfinite(out).all())
        _, y64, T = c.reference()
        check_linear(ref, y64, T, "nvfp4_linear")
        check_linear(out, y64, T, "nvfp4_linear_noalloc")
        assert torch.equal(out, ref)  # same kernels on the same inputs
    assert q.read_device_status() == 0


def test_noalloc_on_a_side_stream_after_a_first_call():
    # a first call on the default stream, then one on a side stream: the scratch
    # path gives the same bits as nvfp4_linear issued on that same stream
    c = Nvfp4Case(512, 1024, 640, seed=33, bias=True)
    d = c.device_args()
    q.nvfp4_linear_noalloc(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                           bias=d["bias"])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ref = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"],
                             bias=d["bias"])
        out = q.nvfp4_linear_noalloc(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                                     d["input_scale"], bias=d["bias"], y=_nan_output(c.M, c.N))
    side.synchronize()
    assert torch.equal(out, ref)
    _, y64, T = c.reference()
    check_linear(out, y64, T, "nvfp4_linear_noalloc on a side stream")
    assert q.read_device_status() == 0


def test_noalloc_checks_the_output_and_bias():
    c = Nvfp4Case(64, 256, 128, seed=34)
    d = c.device_args()
    wrong_y = torch.empty((c.M, c.N + 8), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        q.nvfp4_linear_noalloc(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                               d["input_scale"], y=wrong_y)
    with pytest.raises(ValueError):
        q.nvfp4_linear_noalloc(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                               d["input_scale"],
                               y=torch.empty((c.M, c.N), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        q.nvfp4_linear_noalloc(d["x"], d["w"], d["w_scale"], d["weight_scale_2"],
                               d["input_scale"],
                               bias=torch.zeros(c.N - 1, dtype=torch.float32, device="cuda"))


def test_noalloc_rejects_problems_beyond_its_scratch():
    M, K, N = 16384, 12288, 3072  # needs about 130 MB of scratch
    assert q.nvfp4_linear_workspace_size(M, K, N) > (32 << 20)
    lib = _lib.load()
    fake = torch.empty(16, dtype=torch.uint8, device="cuda").data_ptr()
    rc = lib.nvfp4_linear_noalloc(fake, M, K, fake, fake, N, fake, fake, None, fake, None)
    assert rc == _lib.QL_ERR_WORKSPACE
    assert "more than" in lib.ql_last_error_message().decode()
