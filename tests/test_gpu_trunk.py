"""GPU parity of the trunk's two-level format and of the shared expert
against the CPU oracle, bit for bit: the weight codes, u8 group scales and
bf16 row scales (the minimax search decided in the same fp32 steps); the
trunk GEMM's bf16 output (one fp32 fma per 128-group in ascending order, the
u8 x bf16 weight scale exact); the shared expert's rotated codes and scales
and its bf16 output."""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import assert_bf16_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _trunk_both(orc, wb):
    q, su8, s2 = w8a8.trunk_weight_quant(to_dev_bf16(wb))
    qo, su8o, s2o = orc.trunk_weight_quant(wb)
    assert np.array_equal(_bits(s2), s2o)
    assert np.array_equal(su8.cpu().numpy(), su8o)
    assert np.array_equal(q.cpu().numpy(), qo)
    return (q, su8, s2), (qo, su8o, s2o)


@pytest.mark.parametrize("N,K", [(37, 512), (64, 2048), (5, 8192)])
def test_trunk_weight_quant_bit_exact(orc, N, K):
    rng = np.random.default_rng(N + K)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[1] = 0                                  # a zero row
    w[2, 700 % K:700 % K + 9] *= 40.0         # a loud group
    w[3, :256] *= 1e-3                        # a quiet group
    _trunk_both(orc, inputs.to_bf16_bits(w))


@pytest.mark.parametrize("M,N,K", [(1, 512, 2048), (4, 1040, 512), (8, 4096, 2048), (9, 512, 2048),
                                   (200, 1040, 512), (2048, 4096, 2048), (300, 1040, 512), (513, 264, 1024)])
def test_linear_trunk(orc, M, N, K):
    xb, wb = inputs.hadamard_linear(M + N, M, K=K, N=N)
    (q, su8, s2), (qo, su8o, s2o) = _trunk_both(orc, wb)
    qx, sx = w8a8.fwht128_quant(to_dev_bf16(xb))
    y = from_dev_bf16(w8a8.linear_trunk(qx, sx, q, su8, s2))
    qxo, sxo, _ = orc.fwht128_quant(xb)
    rows = np.arange(M) if M <= 2048 else np.unique(np.concatenate([np.random.default_rng(M).integers(0, M, 40),
                                                                  [0, 127, 128, M - 1]]))
    yo, y32 = orc.gemm_trunk(qxo[rows], sxo[rows], qo, su8o, s2o)
    assert assert_bf16_close(y[rows], y32, what=f"trunk M={M}") == 1.0
    assert np.array_equal(y[rows], yo)


def _shared_weights(orc, seed, H, I):
    rng = np.random.default_rng([seed, 3])
    w13b = inputs.to_bf16_bits(inputs.weights(rng, (2 * I, H)))
    w2b = inputs.to_bf16_bits(inputs.weights(rng, (H, I)))
    g13, o13 = _trunk_both(orc, w13b)
    g2 = w8a8.fwht128_quant(to_dev_bf16(w2b))
    o2 = orc.fwht128_quant(w2b)
    assert np.array_equal(g2[0].cpu().numpy(), o2[0]) and np.array_equal(_bits(g2[1]), o2[1])
    return (*g13, g2[0], g2[1]), (*o13, o2[0], o2[1])


@pytest.mark.parametrize("M,H,I", [(1, 256, 128), (5, 512, 256), (8, 2048, 512), (20, 256, 384),
                                   (40, 512, 128), (300, 768, 256)])
def test_shared_expert(orc, M, H, I):
    gw, ow = _shared_weights(orc, M + H, H, I)
    rng = np.random.default_rng(M * 7 + I)
    xb = inputs.to_bf16_bits(rng.standard_normal((M, H)).astype(np.float32))
    y, dbg = w8a8.shared_expert_forward(to_dev_bf16(xb), *gw, debug=True)
    y = from_dev_bf16(y)
    ref = orc.shared_expert_forward(xb, *ow)
    assert np.array_equal(dbg["qx"].cpu().numpy(), ref["qx"]) and np.array_equal(_bits(dbg["sx"]), ref["sx"])
    assert np.array_equal(dbg["qa"].cpu().numpy(), ref["qa"]) and np.array_equal(_bits(dbg["sa"]), ref["sa"])
    assert assert_bf16_close(y, ref["y32"], what="shared expert y") == 1.0
    assert np.array_equal(y, ref["y"])


def test_shared_expert_rejects_bad_shapes():
    x = torch.zeros((2, 384), dtype=torch.bfloat16, device="cuda")
    w13 = torch.zeros((256, 384), dtype=torch.int8, device="cuda")
    u13 = torch.zeros((256, 1), dtype=torch.uint8, device="cuda")
    r13 = torch.zeros(256, dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros((384, 128), dtype=torch.int8, device="cuda")
    s2 = torch.zeros((384, 1), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w8a8.W8A8Error):
        w8a8.shared_expert_forward(x, w13, u13, r13, w2, s2)
