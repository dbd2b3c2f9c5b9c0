"""GPU parity of the FWHT128-domain path: rotated codes and bf16 group
scales bit for bit (a12); the group-scaled GEMM (a13) equal to the oracle's
ascending-group fp32 sum within one bf16 ulp."""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import assert_bf16_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _fwht_gpu(xb):
    q, s = w8a8.fwht128_quant(to_dev_bf16(xb))
    return q, s


@pytest.mark.parametrize("M", [1, 2048, 3])
def test_fwht128_quant_bit_exact(orc, M):
    xb, wb = inputs.hadamard_linear(M, M)
    q, s = _fwht_gpu(xb)
    qo, so, _ = orc.fwht128_quant(xb)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(from_dev_bf16(s), so)


def test_fwht128_quant_weights_and_zero_blocks(orc):
    _, wb = inputs.hadamard_linear(0, 1)
    wb = wb.copy()
    wb[5, 128:256] = 0
    q, s = _fwht_gpu(wb)
    qo, so, _ = orc.fwht128_quant(wb)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(from_dev_bf16(s), so)


@pytest.mark.parametrize("M", [1, 5, 8, 2048, 200, 300, 777])
def test_linear_g128(orc, M):
    xb, wb = inputs.hadamard_linear(M + 11, M)
    qx, sx = _fwht_gpu(xb)
    qw, sw = _fwht_gpu(wb)
    y = from_dev_bf16(w8a8.linear_g128(qx, sx, qw, sw))
    qxo, sxo, _ = orc.fwht128_quant(xb)
    qwo, swo, _ = orc.fwht128_quant(wb)
    rows = np.arange(M) if M <= 2048 else np.unique(np.concatenate([np.random.default_rng(M).integers(0, M, 48),
                                                                  [0, 127, 128, M - 1]]))
    yo, y32 = orc.gemm_g128(qxo[rows], sxo[rows], qwo, swo)
    exact = assert_bf16_close(y[rows], y32, what=f"g128 M={M}")
    assert exact == 1.0


# ---- the unrotated group-128 grid (the head's format: one bf16 scale per row and 128 of K, no rotation)

@pytest.mark.parametrize("M", [1, 3, 2048])
def test_group128_quant_bit_exact(orc, M):
    xb, wb = inputs.hadamard_linear(M + 3, M)
    xb = xb.copy()
    xb[0, 256:384] = 0   # a zero block
    q, s = w8a8.group128_quant(to_dev_bf16(xb))
    qo, so = orc.group128_quant(xb)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(from_dev_bf16(s), so)


@pytest.mark.parametrize("M,N", [(1, 4096), (4, 4096), (8, 1040), (9, 4096), (200, 1040), (2048, 4096),
                                 (520, 1040), (256, 136)])
def test_linear_group128(orc, M, N):
    xb, wb = inputs.hadamard_linear(M + 29, M, N=N)
    qx, sx = w8a8.group128_quant(to_dev_bf16(xb))
    qw, sw = w8a8.group128_quant(to_dev_bf16(wb))
    y = from_dev_bf16(w8a8.linear_group128(qx, sx, qw, sw))
    qxo, sxo = orc.group128_quant(xb)
    qwo, swo = orc.group128_quant(wb)
    assert np.array_equal(qw.cpu().numpy(), qwo) and np.array_equal(from_dev_bf16(sw), swo)
    rows = np.arange(M) if M <= 2048 else np.unique(np.concatenate([np.random.default_rng(M).integers(0, M, 48),
                                                                  [0, 127, 128, M - 1]]))
    yo, y32 = orc.gemm_group128(qxo[rows], sxo[rows], qwo, swo)
    assert assert_bf16_close(y[rows], y32, what=f"group128 M={M}") == 1.0
    assert np.array_equal(y[rows], yo)


def test_linear_group128_is_128x_the_rotated_form():
    """Same codes and scales through both entry points: the unrotated GEMM is
    the rotated one without its 1/128 (bit for bit in fp32, so after bf16 too)."""
    xb, wb = inputs.hadamard_linear(3, 16, N=512)
    qx, sx = w8a8.group128_quant(to_dev_bf16(xb))
    qw, sw = w8a8.group128_quant(to_dev_bf16(wb))
    a = w8a8.linear_group128(qx, sx, qw, sw).float()
    b = w8a8.linear_g128(qx, sx, qw, sw).float()
    assert torch.equal(a, b * 128)
