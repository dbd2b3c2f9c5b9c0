"""Pins of the oracle's routed experts on the FWHT128 grid: "Qwen3.6-35B-A3B
IQ8R - radiance container", file table (Experts row: int8 codes on the
rotated grid, one bf16 scale per row and 128-wide slice of K; Activations
row: quantized after the same rotation, the routed experts taking the trunk
quantizer's codes)
and the recipe rows of the routed experts' gate_up and down weights
(group=128 scale=bf16 transform=fwht128).

Pinned (1) bit for bit against a recomposition from the separately pinned
primitives (router, FWHT128 group quantizer, group-128 GEMM, SiLU, slot-order
fp32 combine), (2) against the unrotated fp64 MoE of the same bf16 weights
within a loose quantization bound -- a dropped 1/128, a rotation along the
wrong axis or a transposed operand is off by orders of magnitude -- and (3)
by the invariants of the routed layer (a zero token, identical experts).
The fp32 quantizer of the gated intermediate is pinned to the bf16 one on
bf16-representable rows and to its own round-trip bound elsewhere.
"""
import numpy as np

from moe_gemm_absmax_b200 import inputs


def _small(seed, T=5, E=8, H=256, I=128):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) * 0.02).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    return inputs.to_bf16_bits(x), inputs.to_bf16_bits(logits), inputs.to_bf16_bits(w13), inputs.to_bf16_bits(w2)


def _rotate_experts(orc, w13b, w2b):
    E, I2, H = w13b.shape
    q13, s13, _ = orc.fwht128_quant(w13b.reshape(E * I2, H))
    q2, s2, _ = orc.fwht128_quant(w2b.reshape(E * H, -1))
    I = I2 // 2
    return (q13.reshape(E, I2, H), s13.reshape(E, I2, H // 128), q2.reshape(E, H, I),
            s2.reshape(E, H, I // 128))


def test_fwht128_quant_f32_equals_bf16_path_on_bf16_rows(orc):
    xb, _ = inputs.hadamard_linear(4, 6, K=384, N=8)
    q, s, _ = orc.fwht128_quant(xb)
    qf, sf = orc.fwht128_quant_f32(inputs.bf16_bits_to_f32(xb))
    assert np.array_equal(q, qf) and np.array_equal(s, sf)


def test_fwht128_quant_f32_round_trip_bound(orc):
    rng = np.random.default_rng(7)
    a = (rng.standard_normal((4, 256)) * 10.0 ** rng.uniform(-3, 2, (4, 1))).astype(np.float32)
    q, s = orc.fwht128_quant_f32(a)
    sf = inputs.bf16_bits_to_f32(s).astype(np.float64)
    for m in range(4):
        for g in range(2):
            blk = orc.fwht128(a[m, g * 128:(g + 1) * 128]).astype(np.float64)
            codes = q[m, g * 128:(g + 1) * 128]
            j = int(np.argmax(np.abs(blk)))
            assert abs(int(codes[j])) == 127 and np.sign(codes[j]) == np.sign(blk[j])
            assert np.all(np.abs(blk - codes * sf[m, g]) <= sf[m, g] * (0.5 + 128 * 2.0 ** -23))


def _recompose(orc, xb, lb, q13, s13, q2, s2, k):
    T, H = xb.shape
    ids, wts = orc.route(lb, k)
    out = np.zeros((T, H), np.float32)
    for t in range(T):
        qx, sx, _ = orc.fwht128_quant(xb[t:t + 1])
        for j in range(k):
            e = ids[t, j]
            _, v = orc.gemm_g128(qx, sx, q13[e], s13[e])
            v = v[0]
            a = orc.silu(v[0::2]) * v[1::2]
            qa, sa = orc.fwht128_quant_f32(a[None, :])
            _, y2 = orc.gemm_g128(qa, sa, q2[e], s2[e])
            out[t] = out[t] + wts[t, j] * y2[0]
    return out


def test_moe_g128_matches_recomposition(orc):
    xb, lb, w13b, w2b = _small(0)
    q13, s13, q2, s2 = _rotate_experts(orc, w13b, w2b)
    res = orc.moe_g128_forward(xb, lb, q13, s13, q2, s2, 2)
    ref = _recompose(orc, xb, lb, q13, s13, q2, s2, 2)
    assert np.array_equal(res["y32"], ref)
    assert np.array_equal(res["y"], orc.f32_to_bf16(ref))
    qx, sx, _ = orc.fwht128_quant(xb)
    assert np.array_equal(res["qx"], qx) and np.array_equal(res["sx"], sx)
    ids, wts = orc.route(lb, 2)
    assert np.array_equal(res["ids"], ids) and np.array_equal(res["wts"], wts)


def test_moe_g128_near_unrotated_fp64_moe(orc):
    """The rotations cancel (H H^T = 128 I on both GEMMs): the result stays
    within a few percent of each row's scale of the fp64 MoE over the same
    bf16 weights, unrotated and unquantized."""
    xb, lb, w13b, w2b = _small(1, T=4, E=4, H=384, I=256)
    q13, s13, q2, s2 = _rotate_experts(orc, w13b, w2b)
    k = 2
    res = orc.moe_g128_forward(xb, lb, q13, s13, q2, s2, k)
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    w13 = inputs.bf16_bits_to_f32(w13b).astype(np.float64)
    w2 = inputs.bf16_bits_to_f32(w2b).astype(np.float64)
    ids, wts = res["ids"], res["wts"].astype(np.float64)
    ref = np.zeros_like(x)
    for t in range(x.shape[0]):
        for j in range(k):
            e = ids[t, j]
            v = w13[e] @ x[t]
            g, u = v[0::2], v[1::2]
            ref[t] += wts[t, j] * (w2[e] @ (g / (1.0 + np.exp(-g)) * u))
    scale = np.abs(ref).max(axis=1, keepdims=True)
    err = np.abs(res["y32"].astype(np.float64) - ref)
    assert np.all(err <= 0.05 * scale)
    assert err.max() > 0   # quantized: not the identity


def test_moe_g128_zero_token_and_identical_experts(orc):
    xb, lb, w13b, w2b = _small(2, T=4, E=6)
    xb[1] = 0
    # every expert a copy of expert 0: the output is the same whatever the routing
    w13b[:] = w13b[0]
    w2b[:] = w2b[0]
    q13, s13, q2, s2 = _rotate_experts(orc, w13b, w2b)
    res = orc.moe_g128_forward(xb, lb, q13, s13, q2, s2, 3)
    assert not res["y32"][1].any()
    lb2 = lb[:, ::-1].copy()
    res2 = orc.moe_g128_forward(xb, lb2, q13, s13, q2, s2, 3)
    # the same y2 in every slot; only the weights' fp32 rounding differs
    assert np.allclose(res["y32"], res2["y32"], rtol=2e-6, atol=1e-7 * np.abs(res["y32"]).max())
    single = orc.moe_g128_forward(xb, lb, q13, s13, q2, s2, 1)
    assert np.allclose(res["y32"], single["y32"], rtol=2e-6, atol=1e-7 * np.abs(res["y32"]).max())


def test_moe_g128_debug_outputs_per_slot(orc):
    xb, lb, w13b, w2b = _small(3, T=3)
    q13, s13, q2, s2 = _rotate_experts(orc, w13b, w2b)
    res = orc.moe_g128_forward(xb, lb, q13, s13, q2, s2, 2, tokens=[2, 0])
    assert res["qa"].shape == (2, 2, 128) and res["sa"].shape == (2, 2, 1)
    full = orc.moe_g128_forward(xb, lb, q13, s13, q2, s2, 2)
    assert np.array_equal(res["y"], full["y"][[2, 0]])
    assert np.array_equal(res["qa"], full["qa"][[2, 0]]) and np.array_equal(res["sa"], full["sa"][[2, 0]])
    assert np.abs(res["qa"]).max() == 127
