"""Pins of the oracle's shared expert on the rotated grid ("Qwen3.6-35B-A3B
IQ8R - radiance container", file table, Experts row: stored like the routed
experts, with its gate/up projection in the trunk's format; recipe rows ffn_gate_up_shexp
(two-level trunk format) and ffn_down_shexp (group=128 scale=bf16
transform=fwht128)).

Pinned bit for bit against a recomposition from the separately pinned
primitives (FWHT128 group quantizer, trunk GEMM, SiLU, fp32-row FWHT
quantizer, group-128 GEMM), against the unrotated fp64 gated MLP of the same
bf16 weights within a loose quantization bound, and by a zero token giving a
zero row.
"""
import numpy as np

from moe_gemm_absmax_b200 import inputs


def _case(orc, seed, M=4, H=512, I=256):
    rng = np.random.default_rng(seed)
    xb = inputs.to_bf16_bits(rng.standard_normal((M, H)).astype(np.float32))
    w13b = inputs.to_bf16_bits((rng.standard_normal((2 * I, H)) * 0.02).astype(np.float32))
    w2b = inputs.to_bf16_bits((rng.standard_normal((H, I)) * 0.02).astype(np.float32))
    q13, u13, r13 = orc.trunk_weight_quant(w13b)
    q2, s2, _ = orc.fwht128_quant(w2b)
    return xb, w13b, w2b, (q13, u13, r13, q2, s2)


def test_shared_expert_matches_recomposition(orc):
    xb, _, _, w = _case(orc, 0)
    res = orc.shared_expert_forward(xb, *w)
    q13, u13, r13, q2, s2 = w
    qx, sx, _ = orc.fwht128_quant(xb)
    _, v = orc.gemm_trunk(qx, sx, q13, u13, r13)
    a = orc.silu(v[:, 0::2]).reshape(v.shape[0], -1) * v[:, 1::2]
    qa, sa = orc.fwht128_quant_f32(a)
    y, y32 = orc.gemm_g128(qa, sa, q2, s2)
    assert np.array_equal(res["qx"], qx) and np.array_equal(res["sx"], sx)
    assert np.array_equal(res["qa"], qa) and np.array_equal(res["sa"], sa)
    assert np.array_equal(res["y32"], y32) and np.array_equal(res["y"], y)


def test_shared_expert_near_unrotated_fp64_mlp(orc):
    xb, w13b, w2b, w = _case(orc, 1, M=3)
    res = orc.shared_expert_forward(xb, *w)
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    v = x @ inputs.bf16_bits_to_f32(w13b).astype(np.float64).T
    g, u = v[:, 0::2], v[:, 1::2]
    ref = (g / (1.0 + np.exp(-g)) * u) @ inputs.bf16_bits_to_f32(w2b).astype(np.float64).T
    err = np.abs(res["y32"].astype(np.float64) - ref)
    assert np.all(err <= 0.05 * np.abs(ref).max(axis=1, keepdims=True))
    assert err.max() > 0


def test_shared_expert_zero_token(orc):
    xb, _, _, w = _case(orc, 2, M=3)
    xb[1] = 0
    res = orc.shared_expert_forward(xb, *w)
    assert not res["y32"][1].any() and res["y32"][0].any()
