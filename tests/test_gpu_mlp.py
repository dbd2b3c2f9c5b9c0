"""GPU parity of the dense gated MLP block (gate_up with SiLU(gate) * up,
requant, down) against the CPU oracle: the x codes and scales, the gated
intermediate's codes and scales and the bf16 output bit for bit -- the
kernels take the oracle's fp32 steps in its order -- on every path: the
weight-streaming GEMV (M <= 8), the one-CTA tcgen05 GEMM and the CTA-pair
GEMM (M >= 256)."""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import assert_bf16_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _weights(orc, seed, H, I):
    rng = np.random.default_rng([seed, 9])
    w13 = inputs.weights(rng, (2 * I, H))
    w2 = inputs.weights(rng, (H, I))
    g13, g2 = w8a8.quant_rows_f32(torch.from_numpy(w13).cuda()), w8a8.quant_rows_f32(torch.from_numpy(w2).cuda())
    o13, o2 = orc.quant_rows_f32(w13), orc.quant_rows_f32(w2)
    assert np.array_equal(g13[0].cpu().numpy(), o13[0]) and np.array_equal(g2[0].cpu().numpy(), o2[0])
    return (g13[0], g13[1], g2[0], g2[1]), (o13[0], o13[1], o2[0], o2[1])


def _check(orc, xb, gw, ow, rows=None):
    y, dbg = w8a8.mlp_forward(to_dev_bf16(xb), *gw, debug=True)
    y = from_dev_bf16(y)
    rows = np.arange(xb.shape[0]) if rows is None else rows
    ref = orc.mlp_forward(xb[rows], *ow)
    assert np.array_equal(dbg["qx"].cpu().numpy()[rows], ref["qx"])
    assert np.array_equal(dbg["sx"].cpu().numpy()[rows].view(np.uint32), ref["sx"].view(np.uint32))
    assert np.array_equal(dbg["qa"].cpu().numpy()[rows], ref["qa"])
    assert np.array_equal(dbg["sa"].cpu().numpy()[rows].view(np.uint32), ref["sa"].view(np.uint32))
    assert assert_bf16_close(y[rows], ref["y32"], what="mlp y") == 1.0
    assert np.array_equal(y[rows], ref["y"])


@pytest.mark.parametrize("M,H,I", [(1, 256, 96), (5, 256, 128), (8, 512, 256), (3, 128, 16),
                                   # one-CTA tcgen05 GEMMs (9 <= M < 256), ragged rows
                                   (13, 256, 128), (40, 512, 96), (200, 256, 256),
                                   # CTA-pair GEMMs (M >= 256): several tiles, ragged M and N
                                   (256, 256, 128), (300, 512, 176), (520, 768, 384)])
def test_mlp_small_configs(orc, M, H, I):
    xb, _ = inputs.dense_linear(M * 3 + H + I, M, H, 16, with_weights=False)
    gw, ow = _weights(orc, M + H, H, I)
    _check(orc, xb, gw, ow)


def test_mlp_zero_token_row():
    xb, _ = inputs.dense_linear(4, 6, 256, 16, with_weights=False)
    xb[3] = 0
    rng = np.random.default_rng(5)
    w13, w2 = inputs.weights(rng, (256, 256)), inputs.weights(rng, (256, 128))
    g13, g2 = w8a8.quant_rows_f32(torch.from_numpy(w13).cuda()), w8a8.quant_rows_f32(torch.from_numpy(w2).cuda())
    y = from_dev_bf16(w8a8.mlp_forward(to_dev_bf16(xb), g13[0], g13[1], g2[0], g2[1]))
    assert not y[3].any()


@pytest.fixture(scope="module")
def mlp_full(orc):
    """The dense MLP of the workload: H = 5120, I = 17408 (gate_up 34816 x 5120, down 5120 x 17408)."""
    return _weights(orc, 0, inputs.DOWN["N"], inputs.DOWN["K"])


@pytest.mark.parametrize("M", [1, 8])
def test_mlp_full_size_decode(orc, mlp_full, M):
    xb, _ = inputs.dense_linear(70 + M, M, inputs.DOWN["N"], 16, with_weights=False)
    _check(orc, xb, *mlp_full)


def test_mlp_full_size_prefill_sampled(orc, mlp_full):
    M = 512
    xb, _ = inputs.dense_linear(77, M, inputs.DOWN["N"], 16, with_weights=False)
    rows = np.unique(np.concatenate([np.random.default_rng(3).integers(0, M, 6), [0, 255, 256, M - 1]]))
    _check(orc, xb, *mlp_full, rows=rows)


def test_mlp_rejects_bad_shapes():
    x = torch.zeros((2, 250), dtype=torch.bfloat16, device="cuda")
    w13 = torch.zeros((256, 250), dtype=torch.int8, device="cuda")
    w2 = torch.zeros((250, 128), dtype=torch.int8, device="cuda")
    s = torch.ones(256, dtype=torch.float32, device="cuda")
    with pytest.raises(w8a8.W8A8Error):
        w8a8.mlp_forward(x, w13, s, w2, s[:250].contiguous())
