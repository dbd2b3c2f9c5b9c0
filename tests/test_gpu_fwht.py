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


@pytest.mark.parametrize("M", [1, 5, 8, 2048, 200])
def test_linear_g128(orc, M):
    xb, wb = inputs.hadamard_linear(M + 11, M)
    qx, sx = _fwht_gpu(xb)
    qw, sw = _fwht_gpu(wb)
    y = from_dev_bf16(w8a8.linear_g128(qx, sx, qw, sw))
    qxo, sxo, _ = orc.fwht128_quant(xb)
    qwo, swo, _ = orc.fwht128_quant(wb)
    rows = np.arange(M) if M <= 256 else np.unique(np.concatenate([np.random.default_rng(M).integers(0, M, 48),
                                                                  [0, 127, 128, M - 1]]))
    yo, y32 = orc.gemm_g128(qxo[rows], sxo[rows], qwo, swo)
    exact = assert_bf16_close(y[rows], y32, what=f"g128 M={M}")
    assert exact == 1.0
