"""Helpers of the GPU parity tests: seeded inputs, oracle references and the
acceptance checks.

Acceptance (stated for the quantized linear):
  * quantized codes and block / row scales: bit-exact against the oracle;
  * bf16 outputs: relative Frobenius error <= 5e-3, and per element
    |y - y_ref| <= 1e-3 * sum_k |x_k w_k| (scaled) + one bf16 ulp of |y_ref|,
    where y_ref is the oracle's fp64 value.
"""
import numpy as np
import torch

import oracle

FROB_TOL = 5e-3
ELEM_TOL = 1e-3


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().cuda()


def scalar_dev(v: float) -> torch.Tensor:
    return torch.tensor([v], dtype=torch.float32, device="cuda")


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_linear(y_gpu: torch.Tensor, y64: np.ndarray, T: np.ndarray, what: str = "",
                 extra: np.ndarray = None):
    """Element and Frobenius tolerance of a bf16 GPU output against the fp64 oracle.
    `extra` adds a per-element allowance (e.g. for a branch evaluated in 16 bits)."""
    y = oracle.bf16_bits_to_f64(bf16_bits(y_gpu))
    assert y.shape == y64.shape, (y.shape, y64.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    err = np.abs(y - y64)
    bound = ELEM_TOL * T + oracle.bf16_ulp(y64)
    if extra is not None:
        bound = bound + extra
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:8]
        detail = [(tuple(i), float(y[tuple(i)]), float(y64[tuple(i)]), float(bound[tuple(i)]))
                  for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance, e.g. {detail}")
    frob = np.linalg.norm(y - y64) / max(np.linalg.norm(y64), 1e-300)
    assert frob <= FROB_TOL, f"{what}: relative Frobenius error {frob}"
    return frob


def unpack_act_scale_atoms(buf: np.ndarray, M: int, K: int) -> np.ndarray:
    """Row-major [M, K/16] view of the activation scale atoms the linear's
    prologue writes into its workspace (internal layout: atoms of 128 rows x 4
    scales, byte 16*(r%32) + 4*(r/32) + j, atom index row_group * KG + kg with KG
    = 64-element groups of K rounded up to 256)."""
    KG = -(-K // 256) * 4
    nb = K // 16
    r = np.arange(M)[:, None]
    b = np.arange(nb)[None, :]
    kg, j = b // 4, b % 4
    rr = r % 128
    off = ((r // 128) * KG + kg) * 512 + (rr % 32) * 16 + (rr // 32) * 4 + j
    return buf[off]


def sample_rows(M: int, n_random: int, seed: int = 0) -> np.ndarray:
    """Rows that cover first / last / tile-boundary rows plus random ones."""
    fixed = {0, 1, 31, 32, 127, 128, 129, M // 2, M - 129, M - 128, M - 2, M - 1}
    rng = np.random.default_rng(seed)
    extra = set(rng.choice(M, size=min(n_random, M), replace=False).tolist())
    rows = sorted(r for r in fixed | extra if 0 <= r < M)
    return np.array(rows, dtype=np.int64)


class Nvfp4Case:
    """Seeded NVFP4 layer: oracle-quantized weight, oracle-calibrated input scale."""

    def __init__(self, M, K, N, seed=0, bias=False, input_scale_div=1.0, x=None):
        from synthetic import make_linear_inputs
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=bias)
        self.x = inp.x if x is None else x
        self.M, self.K, self.N = M, K, N
        self.gw = oracle.nvfp4_global_scale(inp.w)
        self.wq, self.ws = oracle.nvfp4_quantize(inp.w, self.gw)
        self.gx = np.float32(oracle.nvfp4_global_scale(self.x) / input_scale_div)
        self.bias = None if inp.bias is None else inp.bias.numpy()

    def oracle_act(self):
        return oracle.nvfp4_quantize(self.x, self.gx)

    def device_args(self):
        return dict(x=to_dev(self.x), w=to_dev(self.wq), w_scale=to_dev(self.ws),
                    weight_scale_2=scalar_dev(self.gw), input_scale=scalar_dev(float(self.gx)),
                    bias=None if self.bias is None else to_dev(self.bias))

    def reference(self, rows=None):
        xq, xs = self.oracle_act()
        if rows is not None:
            xq, xs = xq[rows], xs[rows]
        return oracle.nvfp4_linear(xq, xs, self.wq, self.ws, self.gx, self.gw, self.bias)


class Fp8rCase:
    def __init__(self, M, K, N, seed=0, bias=False):
        from synthetic import make_linear_inputs
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=bias)
        self.x = inp.x
        self.M, self.K, self.N = M, K, N
        self.wq, self.wsc = oracle.fp8r_quantize_rows(inp.w)
        self.bias = None if inp.bias is None else inp.bias.numpy()

    def device_args(self):
        return dict(x=to_dev(self.x), w=to_dev(self.wq), w_scale=to_dev(self.wsc),
                    bias=None if self.bias is None else to_dev(self.bias))

    def reference(self, rows=None):
        xq, xs = oracle.fp8r_quantize_rows(self.x)
        if rows is not None:
            xq, xs = xq[rows], xs[rows]
        return oracle.fp8r_linear(xq, xs, self.wq, self.wsc, self.bias)
