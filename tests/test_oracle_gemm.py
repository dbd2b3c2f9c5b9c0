"""Pins of the oracle's int8 GEMM (a2), dequant epilogue (a3) and the whole
dense linear (a1+a2+a3) -- "Online INT8 W8A8 ...", Changes (gemm_a8w8);
"Qwen3.6-27B-Quark-W8A8-INT8", Quantization Details.

The int32 accumulators are pinned to numpy's int64 matmul (a library
routine); the dequantized fp64 value to the method's own error bound
against the unquantized fp64 product; the fp32/bf16 values to one
rounding step per operation.
"""
import numpy as np
import torch

from moe_gemm_absmax_b200 import inputs


def test_gemm_s32_equals_numpy_int64(orc):
    rng = np.random.default_rng(0)
    for (M, N, K) in [(1, 1, 1), (3, 5, 7), (16, 40, 512), (9, 33, 1000)]:
        a = rng.integers(-127, 128, (M, K), dtype=np.int8)
        b = rng.integers(-127, 128, (N, K), dtype=np.int8)
        ref = a.astype(np.int64) @ b.astype(np.int64).T
        assert np.array_equal(orc.gemm_s32(a, b), ref.astype(np.int32))


def test_gemm_s32_extremes_fit_int32(orc):
    K = 17408                                    # the widest K of the workloads
    a = np.full((2, K), 127, np.int8)
    b = np.full((3, K), -127, np.int8)
    b[1] = 127
    acc = orc.gemm_s32(a, b)
    assert acc[0, 0] == -127 * 127 * K and acc[0, 1] == 127 * 127 * K
    assert abs(int(acc[0, 0])) < 2 ** 31


def test_gemm_s32_at_samples(orc):
    rng = np.random.default_rng(1)
    a = rng.integers(-127, 128, (20, 256), dtype=np.int8)
    b = rng.integers(-127, 128, (30, 256), dtype=np.int8)
    ms = rng.integers(0, 20, 50)
    ns = rng.integers(0, 30, 50)
    full = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(orc.gemm_s32_at(a, b, ms, ns), full[ms, ns])


def test_dequant_rounding_steps(orc):
    rng = np.random.default_rng(2)
    acc = rng.integers(-2 ** 28, 2 ** 28, (8, 64)).astype(np.int32)
    sx = (rng.random(8) * 0.1).astype(np.float32)
    sw = (rng.random(64) * 1e-3).astype(np.float32)
    y, y32, y64 = orc.dequant(acc, sx, sw)
    exact = acc.astype(np.float64) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    assert np.array_equal(y64, exact)
    # three roundings (int->fp32, two products): relative error <= 3 * 2^-24
    assert np.all(np.abs(y32 - exact) <= 3.0001 * 2.0 ** -24 * np.abs(exact))
    # numpy float32 products are IEEE round-to-nearest: same value bit for bit
    np32 = (acc.astype(np.float32) * sx[:, None]) * sw[None, :]
    assert np.array_equal(y32, np32)
    ref_bf16 = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y, ref_bf16)


def test_linear_error_bound_against_unquantized_product(orc):
    """|x W^T - y64| <= sum_k (|x_k| s_w/2 + |W_nk| s_x/2 + s_x s_w/4): each
    operand is within half a step of its code, so the product error is the
    sum of the cross terms."""
    xb, w = inputs.tiny_linear(0)
    qw, sw = orc.quant_rows_f32(w)
    y, y32, qx, sx = orc.linear(xb, qw, sw)
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    W = w.astype(np.float64)
    ref = x @ W.T
    acc = orc.gemm_s32(qx, qw)
    y64 = acc.astype(np.float64) * sx[:, None] * sw[None, :]
    slack = 1 + 1e-5                                   # fp32 rounding of x/s and s itself
    bound = (np.abs(x) @ np.ones_like(W).T) * sw[None, :] / 2 * slack \
        + sx[:, None] * (np.ones_like(x) @ np.abs(W).T) / 2 * slack \
        + x.shape[1] * sx[:, None] * sw[None, :] / 4
    assert np.all(np.abs(ref - y64) <= bound + 1e-12)
    # edge rows of the workload: the all-zero row gives exact zeros
    assert not y[0].any() and sx[0] == 0
    # and the fp32/bf16 outputs are the documented rounding of the same value
    y_b, y32_b, _ = orc.dequant(acc, sx, sw)
    assert np.array_equal(y, y_b) and np.array_equal(y32, y32_b)


def test_linear_close_to_fp64_reference(orc):
    """W8A8 with per-token/per-channel scales stays close to the bf16 x fp32 product."""
    xb, w = inputs.dense_linear(3, 8, 1024, 256)
    qw, sw = orc.quant_rows_f32(w)
    y, y32, qx, sx = orc.linear(xb, qw, sw)
    ref = inputs.bf16_bits_to_f32(xb).astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(y32 - ref) / np.linalg.norm(ref)
    assert rel < 0.05
