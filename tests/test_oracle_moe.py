"""Pins of the oracle's routed MoE layer (a5-a11): "Online INT8 W8A8 ...",
Changes (routing -> per-token int8 quant -> gemm1 with fused gated SiLU over
interleaved w13 -> per-token int8 quant -> gemm2 with scatter/combine).

The pipeline is recomposed here in numpy (int64 matmuls, IEEE fp32
elementwise products, slot-order accumulation) from the separately pinned
primitives (quant row, SiLU, router), and must agree bit for bit.  Further
invariants: a single expert with top-1 is the dense gated MLP, identical
experts make the output independent of routing, a zero token gives zeros,
and relabelling the experts changes nothing.
"""
import numpy as np
import torch

from moe_gemm_absmax_b200 import inputs


def _small(seed, T=6, E=8, H=256, I=64):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13 = (rng.standard_normal((E, 2 * I, H)) * 0.02).astype(np.float32)
    w2 = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    return inputs.to_bf16_bits(x), inputs.to_bf16_bits(logits), w13, w2


def _quant_experts(orc, w13, w2):
    E, I2, H = w13.shape
    q13, s13 = orc.quant_rows_f32(w13.reshape(E * I2, H))
    q2, s2 = orc.quant_rows_f32(w2.reshape(E * H, -1))
    return q13.reshape(w13.shape), s13.reshape(E, I2), q2.reshape(w2.shape), s2.reshape(E, H)


def _numpy_moe(orc, xb, lb, q13, s13, q2, s2, k):
    T, H = xb.shape
    ids, wts = orc.route(lb, k)
    x = inputs.bf16_bits_to_f32(xb)
    out = np.zeros((T, H), np.float32)
    for t in range(T):
        qx, sx = orc.quant_row_f32(x[t])
        for j in range(k):
            e = ids[t, j]
            acc1 = q13[e].astype(np.int64) @ qx.astype(np.int64)
            v = (acc1.astype(np.float32) * sx) * s13[e]
            a = orc.silu(v[0::2]) * v[1::2]
            qa, sa = orc.quant_row_f32(a)
            acc2 = q2[e].astype(np.int64) @ qa.astype(np.int64)
            y2 = (acc2.astype(np.float32) * sa) * s2[e]
            out[t] = out[t] + wts[t, j] * y2
    return out


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_moe_matches_numpy_recomposition(orc):
    xb, lb, w13, w2 = _small(0)
    q13, s13, q2, s2 = _quant_experts(orc, w13, w2)
    for k in (1, 2, 3):
        res = orc.moe_forward(xb, lb, q13, s13, q2, s2, k)
        ref = _numpy_moe(orc, xb, lb, q13, s13, q2, s2, k)
        assert np.array_equal(res["y32"], ref)
        assert np.array_equal(res["y"], _bf16(ref))


def test_moe_token_subset_equals_full(orc):
    xb, lb, w13, w2 = _small(1, T=9)
    q13, s13, q2, s2 = _quant_experts(orc, w13, w2)
    full = orc.moe_forward(xb, lb, q13, s13, q2, s2, 2)
    part = orc.moe_forward(xb, lb, q13, s13, q2, s2, 2, tokens=np.array([7, 2, 4]))
    for key in ("y", "y32", "ids", "wts", "qx", "sx", "qa", "sa"):
        assert np.array_equal(part[key], full[key][[7, 2, 4]])


def test_single_expert_top1_is_dense_gated_mlp(orc):
    """E = 1, k = 1: weight 1 exactly; y = down(quant(SiLU(gate)·up)) with
    the dense a1 -> a2/a3 composition written out in numpy."""
    xb, lb, w13, w2 = _small(2, E=1)
    q13, s13, q2, s2 = _quant_experts(orc, w13, w2)
    res = orc.moe_forward(xb, lb, q13, s13, q2, s2, 1)
    assert np.all(res["wts"] == 1.0) and np.all(res["ids"] == 0)
    qx, sx = orc.quant_rows_bf16(xb)
    acc1 = qx.astype(np.int64) @ q13[0].astype(np.int64).T
    v = (acc1.astype(np.float32) * sx[:, None]) * s13[0][None, :]
    a = orc.silu(v[:, 0::2]).reshape(v.shape[0], -1) * v[:, 1::2]
    qa, sa = orc.quant_rows_f32(a)
    acc2 = qa.astype(np.int64) @ q2[0].astype(np.int64).T
    y = (acc2.astype(np.float32) * sa[:, None]) * s2[0][None, :]
    assert np.array_equal(res["y32"], np.float32(1.0) * y)


def test_identical_experts_ignore_routing(orc):
    xb, lb, w13, w2 = _small(3, E=6)
    w13[:] = w13[0]
    w2[:] = w2[0]
    q13, s13, q2, s2 = _quant_experts(orc, w13, w2)
    res = orc.moe_forward(xb, lb, q13, s13, q2, s2, 3)
    one = orc.moe_forward(xb, lb, q13[:1], s13[:1], q2[:1], s2[:1], 1)
    # sum_j w_j * y2 with sum_j w_j = 1 (to fp32 rounding)
    tol = 8 * 2.0 ** -24 * res["yabs"] + 1e-30
    assert np.all(np.abs(res["y32"] - one["y32"]) <= tol)


def test_zero_token_gives_zero_row(orc):
    xb, lb, w13, w2 = _small(4)
    xb[2] = 0
    q13, s13, q2, s2 = _quant_experts(orc, w13, w2)
    res = orc.moe_forward(xb, lb, q13, s13, q2, s2, 2)
    assert res["sx"][2] == 0 and not res["qx"][2].any()
    assert not res["y32"][2].any()


def test_expert_relabelling_invariance(orc):
    xb, lb, w13, w2 = _small(5, E=8)
    q13, s13, q2, s2 = _quant_experts(orc, w13, w2)
    perm = np.random.default_rng(9).permutation(8)
    res = orc.moe_forward(xb, lb, q13, s13, q2, s2, 2)
    res_p = orc.moe_forward(xb, np.ascontiguousarray(lb[:, perm]), q13[perm], s13[perm], q2[perm], s2[perm], 2)
    lf = inputs.bf16_bits_to_f32(lb)
    distinct = all(len(set(r.tolist())) == r.size for r in lf)
    assert distinct
    assert np.array_equal(perm[res_p["ids"]], res["ids"])
    # codes do not depend on the labels; the weights only through the
    # index-order softmax sum, i.e. to fp32 rounding
    assert np.array_equal(res["qa"], res_p["qa"]) and np.array_equal(res["sa"], res_p["sa"])
    assert np.allclose(res["wts"], res_p["wts"], rtol=4 * 2.0 ** -23, atol=0)
    assert np.all(np.abs(res["y32"] - res_p["y32"]) <= 16 * 2.0 ** -24 * res["yabs"])
