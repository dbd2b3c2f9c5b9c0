"""GPU parity of the quantization kernels (a0, a1) and the project
exponential against the CPU oracle: codes and scales bit for bit."""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import to_dev_bf16

pytestmark = pytest.mark.gpu


def _check_act(orc, xb):
    q, s = w8a8.quant_act(to_dev_bf16(xb))
    qo, so = orc.quant_rows_bf16(xb)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


def test_quant_act_tiny_with_edge_rows(orc):
    xb, _ = inputs.tiny_linear(0)
    _check_act(orc, xb)


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("K", [5120, 17408])
def test_quant_act_decode_shapes(orc, M, K):
    xb, _ = inputs.dense_linear(M + K, M, K, 16, with_weights=False)
    _check_act(orc, xb)


@pytest.mark.parametrize("M,K", [(129, 2048), (3, 16), (512, 5120), (37, 17408), (2, 65536)])
def test_quant_act_ragged_and_long(orc, M, K):
    xb, _ = inputs.dense_linear(7, M, K, 16, with_weights=False)
    _check_act(orc, xb)


def test_quant_act_special_values(orc):
    rows = np.zeros((6, 32), np.float32)
    rows[1, 3] = -1e-40                       # subnormal single nonzero
    rows[2] = np.array([127, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, 126.5] * 4, np.float32) / 16   # exact ties
    rows[3] = -np.abs(np.linspace(0.1, 3, 32))                  # absmax negative
    rows[4] = np.float32(3.0e38) * np.sign(np.sin(np.arange(32)))  # near the fp32 limit
    rows[5, ::2] = -0.0
    _check_act(orc, inputs.to_bf16_bits(rows))


@pytest.mark.parametrize("N,K", [(512, 512), (100, 17408), (33, 5120), (8, 48)])
def test_quant_rows_f32_weights(orc, N, K):
    w = inputs.weights(np.random.default_rng(N * K), (N, K))
    q, s = w8a8.quant_rows_f32(torch.from_numpy(w).cuda())
    qo, so = orc.quant_rows_f32(w)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


def test_exp_proj_bit_exact(orc):
    x = np.concatenate([np.arange(0, 0x42B00000, 40009, dtype=np.uint32),
                        np.arange(0x80000000, 0xC2AE0000, 40009, dtype=np.uint32)]).view(np.float32)
    x = np.concatenate([x, np.float32([88.0, -87.0, 100.0, -100.0, 0.0, -0.0])])
    y = w8a8.exp_proj(torch.from_numpy(x).cuda()).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), orc.exp_proj(x).view(np.uint32))


def test_quant_near_ties_take_the_exact_path(orc):
    """Values a few ulps from a half-integer multiple of the scale: the
    reciprocal-multiply fast path must hand them to the exact division."""
    rng = np.random.default_rng(11)
    rows = []
    for scale in (1 / 16, 0.0123, 3.7e-3):
        n = rng.integers(-126, 126, 256).astype(np.float64)
        eps = rng.choice([0.0, 2.0 ** -23, -(2.0 ** -23), 2.0 ** -20, -(2.0 ** -20), 2.0 ** -15, -(2.0 ** -15)], 256)
        v = ((n + 0.5) * (1.0 + eps) * scale).astype(np.float32)
        v[0] = np.float32(127 * scale)            # fixes absmax, hence s = fp32(127 scale / 127)
        rows.append(v)
    w = np.stack(rows)
    q, s = w8a8.quant_rows_f32(torch.from_numpy(w).cuda())
    qo, so = orc.quant_rows_f32(w)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("M,K", [(300, 512), (400, 17408), (296, 2064), (700, 1024), (300, 104448)])
def test_quant_act_many_rows(orc, M, K):
    """Row counts of a prefill batch: rows staged in shared memory (one and two
    CTA widths), the warp-per-row kernel, and rows too long to stage."""
    xb, _ = inputs.dense_linear(M * 3 + K, M, K, 16, with_weights=False)
    _check_act(orc, xb)


@pytest.mark.parametrize("N,K", [(300, 256), (320, 17408), (600, 1024)])
def test_quant_rows_f32_many_rows(orc, N, K):
    w = inputs.weights(np.random.default_rng(N + K), (N, K))
    q, s = w8a8.quant_rows_f32(torch.from_numpy(w).cuda())
    qo, so = orc.quant_rows_f32(w)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


def test_quant_act_row_stride(orc):
    """x is every other row block of a wider buffer (ldx > K), many rows."""
    xb, _ = inputs.dense_linear(5, 320, 6144, 16, with_weights=False)
    full = to_dev_bf16(xb)
    view = full[:, 1024:1024 + 4096]
    q, s = w8a8.quant_act(view)
    qo, so = orc.quant_rows_bf16(np.ascontiguousarray(xb[:, 1024:1024 + 4096]))
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


def test_quant_special_values_many_rows(orc):
    """Special rows repeated past the row count that switches kernels."""
    rows = np.zeros((6, 64), np.float32)
    rows[1, 3] = -1e-40
    rows[2] = np.array([127, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, 126.5] * 8, np.float32) / 16
    rows[3] = -np.abs(np.linspace(0.1, 3, 64))
    rows[4] = np.float32(3.0e38) * np.sign(np.sin(np.arange(64)))
    rows[5, ::2] = -0.0
    _check_act(orc, inputs.to_bf16_bits(np.tile(rows, (60, 1))))
    q, s = w8a8.quant_rows_f32(torch.from_numpy(np.tile(rows, (60, 1))).cuda())
    qo, so = orc.quant_rows_f32(np.tile(rows, (60, 1)))
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
