"""Pins of the oracle's dense gated MLP block (the dense analogue of a8-a10:
"Online INT8 W8A8 ...", Changes -- gemm1 with fused gated SiLU over
interleaved w13 rows, per-token int8 quant, gemm2).

Pinned against (1) a numpy recomposition from the separately pinned
primitives (activation quant, int64 matmul, fp32 products, SiLU, row quant),
bit for bit, and (2) the routed-MoE oracle with one expert and top-1, whose
routing weight is exactly 1.
"""
import numpy as np

from moe_gemm_absmax_b200 import inputs


def _mlp(seed, M=5, H=256, I=96):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, H)).astype(np.float32)
    w13 = (rng.standard_normal((2 * I, H)) * 0.02).astype(np.float32)
    w2 = (rng.standard_normal((H, I)) * 0.02).astype(np.float32)
    return inputs.to_bf16_bits(x), w13, w2


def test_mlp_matches_numpy_recomposition(orc):
    xb, w13, w2 = _mlp(0)
    q13, s13 = orc.quant_rows_f32(w13)
    q2, s2 = orc.quant_rows_f32(w2)
    res = orc.mlp_forward(xb, q13, s13, q2, s2)
    qx, sx = orc.quant_rows_bf16(xb)
    acc1 = qx.astype(np.int64) @ q13.astype(np.int64).T
    v = (acc1.astype(np.float32) * sx[:, None]) * s13[None, :]
    a = orc.silu(v[:, 0::2]).reshape(v.shape[0], -1) * v[:, 1::2]
    qa, sa = orc.quant_rows_f32(a)
    acc2 = qa.astype(np.int64) @ q2.astype(np.int64).T
    y = (acc2.astype(np.float32) * sa[:, None]) * s2[None, :]
    assert np.array_equal(res["qx"], qx) and np.array_equal(res["sx"], sx)
    assert np.array_equal(res["qa"], qa) and np.array_equal(res["sa"], sa)
    assert np.array_equal(res["y32"], y)
    assert np.array_equal(res["y"], orc.f32_to_bf16(y))


def test_mlp_is_single_expert_top1_moe(orc):
    xb, w13, w2 = _mlp(1, M=7)
    q13, s13 = orc.quant_rows_f32(w13)
    q2, s2 = orc.quant_rows_f32(w2)
    res = orc.mlp_forward(xb, q13, s13, q2, s2)
    logits = np.zeros((xb.shape[0], 1), np.uint16)
    moe = orc.moe_forward(xb, logits, q13[None], s13[None], q2[None], s2[None], 1)
    assert np.array_equal(res["y"], moe["y"]) and np.array_equal(res["y32"], moe["y32"])
    assert np.array_equal(res["qa"], moe["qa"][:, 0]) and np.array_equal(res["sa"], moe["sa"][:, 0])


def test_mlp_zero_token_and_error_bound(orc):
    """A zero token gives a zero row; the others stay within a loose bound of
    the unquantized fp64 MLP (int8 codes: a few percent of the row scale)."""
    xb, w13, w2 = _mlp(2, M=4)
    xb[2] = 0
    q13, s13 = orc.quant_rows_f32(w13)
    q2, s2 = orc.quant_rows_f32(w2)
    res = orc.mlp_forward(xb, q13, s13, q2, s2)
    assert not res["y32"][2].any()
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    v = x @ w13.astype(np.float64).T
    g, u = v[:, 0::2], v[:, 1::2]
    a = g / (1.0 + np.exp(-g)) * u
    y = a @ w2.astype(np.float64).T
    scale = np.abs(y).max(axis=1, keepdims=True) + 1e-30
    assert np.all(np.abs(res["y32"].astype(np.float64) - y) <= 0.05 * scale)
