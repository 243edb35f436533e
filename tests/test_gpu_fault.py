"""Failure detection without a GPU fault: the GEMM kernels bound every wait. The
test hook makes one launch wait on a barrier that nothing completes; the wait
must expire after its short limit, the kernel must return, the device status
word must report QL_ERR_TIMEOUT, and the context must stay usable."""
import pytest
import torch

import fp8_rowwise_quantized_b200 as q
from fp8_rowwise_quantized_b200 import _lib
from gpu_helpers import Nvfp4Case, check_linear

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    c = Nvfp4Case(256, 512, 384, seed=11)
    d = c.device_args()
    assert q.read_device_status() == 0
    try:
        q.set_fault_injection(True, timeout_ms=200)
        q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"])
        torch.cuda.synchronize()
    finally:
        q.set_fault_injection(False, 0)
    assert q.read_device_status() == _lib.QL_ERR_TIMEOUT
    assert q.read_device_status() == 0  # reading clears it
    # the context is intact: a normal call afterwards is correct
    y = q.nvfp4_linear(d["x"], d["w"], d["w_scale"], d["weight_scale_2"], d["input_scale"])
    torch.cuda.synchronize()
    _, y64, T = c.reference()
    check_linear(y, y64, T, "after fault injection")
    assert q.read_device_status() == 0
