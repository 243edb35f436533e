"""The seeded input recipe of the tests and the benchmark (synthetic/__init__.py):
the outlier-channel count, the draw order, determinism and the distributions' scales."""
import torch

from synthetic import WORKLOADS, make_activations, make_linear_inputs, outlier_count


def test_outlier_count_is_one_percent_rounded_half_to_even():
    assert outlier_count(256) == 2                 # the tiny layer's fixed count
    assert outlier_count(3072) == 31               # 30.72
    assert outlier_count(12288) == 123             # 122.88
    assert outlier_count(50) == 0 and outlier_count(150) == 2   # 0.5 -> 0, 1.5 -> 2


def test_draws_are_seeded_and_x_comes_first():
    a = make_linear_inputs(64, 3072, 32, seed=3, with_bias=True)
    b = make_linear_inputs(64, 3072, 32, seed=3, with_bias=True)
    assert torch.equal(a.x, b.x) and torch.equal(a.w, b.w) and torch.equal(a.bias, b.bias)
    assert not torch.equal(a.x, make_linear_inputs(64, 3072, 32, seed=4).x)
    # X does not depend on N or on the bias draw that follows it
    assert torch.equal(a.x, make_linear_inputs(64, 3072, 999, seed=3).x)
    assert torch.equal(a.x, make_activations(64, 3072, seed=3))


def test_dtypes_scales_and_outlier_channels():
    inp = make_linear_inputs(2048, 3072, 512, seed=0, with_bias=True)
    assert inp.x.dtype == torch.bfloat16 and inp.w.dtype == torch.bfloat16
    assert inp.bias.dtype == torch.float32 and inp.bias.shape == (512,)
    assert make_linear_inputs(8, 256, 8).bias is None
    x = inp.x.float()
    out = torch.zeros(3072, dtype=torch.bool)
    out[inp.outlier_idx] = True
    assert int(out.sum()) == 31
    ratio = x[:, out].std() / x[:, ~out].std()
    assert 18.0 < ratio < 22.0                     # outlier channels x 20
    assert 0.95 < x[:, ~out].std() < 1.05          # the rest standard normal
    assert 0.019 < inp.w.float().std() < 0.021     # W ~ N(0, 0.02^2)
    assert 0.008 < inp.bias.std() < 0.012          # bias ~ N(0, 0.01^2)


def test_named_workloads_are_the_dit_layer_sizes():
    assert WORKLOADS["nvfp4_mlp_up"] == dict(M=4096, K=3072, N=12288, bias=False)
    assert WORKLOADS["nvfp4_mlp_down"] == dict(M=4096, K=12288, N=3072, bias=False)
    assert WORKLOADS["nvfp4_attn_qkv"]["N"] == 3 * WORKLOADS["nvfp4_attn_proj"]["N"]
