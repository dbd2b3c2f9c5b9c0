"""Pins of the oracle's two-level trunk format: "Qwen3.6-35B-A3B IQ8R -
radiance container", file table (Trunk: int8 codes -127..127 with a u8 scale
per row and 256 of K under a bf16 scale a row, each 128 of K rotated by the
unnormalised Hadamard, round to nearest) and the recipe rows of the trunk
linears (codes=i8 group=256 scale=u8 scale2=bf16 block2=1x* transform=fwht128
clamp=sym rule=search).

The weight quantizer is pinned by brute force over all 255 u8 values in fp64
(the chosen one has the smallest largest error of its group), by the codes
being the nearest codes under the chosen scale, by the row scale being one
bf16 rounding of absmax / (127 * 255), and by the error bound that the search
can only improve on.  The GEMM is pinned by exact power-of-two cases, by
equality with the separately pinned group-128 GEMM where every u8 * scale2 is
a bf16 value, and by the quantization bound of the unrotated fp64 product.
"""
import numpy as np

from moe_gemm_absmax_b200 import inputs


def _rows(seed, N=3, K=512):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K)).astype(np.float32) * 0.02
    if N >= 3 and K >= 512:
        w[1, 300:310] *= 30.0      # one group much louder than the rest of its row
        w[2, :256] *= 1e-3         # one group much quieter
    return inputs.to_bf16_bits(w)


def test_trunk_quant_search_is_minimax_and_codes_nearest(orc):
    wb = _rows(0)
    q, su8, s2 = orc.trunk_weight_quant(wb)
    _, _, v = orc.fwht128_quant(wb)          # the rotated rows, fp32
    v = v.astype(np.float64)
    s2f = inputs.bf16_bits_to_f32(s2).astype(np.float64)
    N, K = v.shape
    codes = np.arange(-127, 128, dtype=np.float64)
    us = np.arange(1, 256, dtype=np.float64)
    for n in range(N):
        rmax = np.abs(v[n]).max()
        assert abs(s2f[n] - rmax / 32385) <= 2.0 ** -8 * rmax / 32385
        for j in range(K // 256):
            blk = v[n, j * 256:(j + 1) * 256]
            # every candidate's largest error, in fp64 (s = u * scale2 is exact)
            s = us[:, None] * s2f[n]
            c = np.clip(np.rint(blk[None, :] / s), -127, 127)
            worst = np.abs(blk[None, :] - c * s).max(axis=1)
            u = int(su8[n, j])
            assert 1 <= u <= 255
            assert worst[u - 1] <= worst.min() * (1 + 2.0 ** -20) + 1e-30
            # nearest codes under the chosen scale (away from exact ties)
            sc = u * s2f[n]
            err = np.abs(blk[:, None] - codes[None, :] * sc)
            best = codes[np.argmin(err, axis=1)]
            second = np.sort(err, axis=1)[:, 1]
            clear = second - err.min(axis=1) > 2.0 ** -20 * sc
            assert np.array_equal(q[n, j * 256:(j + 1) * 256][clear], best[clear])
            # the search can only improve on the smallest scale that covers the group
            gmax = np.abs(blk).max()
            assert worst[u - 1] <= (gmax / 127 + s2f[n]) / 2 * (1 + 1e-6)


def test_trunk_quant_zero_row_and_full_row_group(orc):
    wb = _rows(1, N=2, K=256)
    wb[0] = 0
    q, su8, s2 = orc.trunk_weight_quant(wb)
    assert s2[0] == 0 and su8[0, 0] == 0 and not q[0].any()
    # the group holding the row maximum takes (nearly) the largest u8
    assert su8[1, 0] >= 250
    assert np.abs(q[1]).max() == 127


def test_gemm_trunk_exact_with_power_of_two_scales(orc):
    rng = np.random.default_rng(3)
    qx = rng.integers(-127, 128, (3, 512), dtype=np.int8)
    qw = rng.integers(-127, 128, (4, 512), dtype=np.int8)
    sx = inputs.to_bf16_bits(np.full((3, 4), 2.0 ** -5, np.float32))
    su8 = np.array([[1, 4], [2, 2], [8, 1], [128, 16]], np.uint8)
    s2 = inputs.to_bf16_bits(np.full(4, 2.0 ** -12, np.float32))
    _, y32 = orc.gemm_trunk(qx, sx, qw, su8, s2)
    # the same sum in exact arithmetic: per 256-group scale u8 * 2^-12
    sw = np.repeat(su8.astype(np.float64), 2, axis=1) * 2.0 ** -12     # per 128-group
    p = np.stack([qx[:, g * 128:(g + 1) * 128].astype(np.int64) @ qw[:, g * 128:(g + 1) * 128].astype(np.int64).T
                  for g in range(4)], axis=-1)
    exact = (p * 2.0 ** -5 * sw[None, :, :]).sum(-1) / 128
    assert np.array_equal(y32.astype(np.float64), exact)


def test_gemm_trunk_equals_group128_gemm_when_scales_are_bf16(orc):
    rng = np.random.default_rng(4)
    qx = rng.integers(-127, 128, (5, 768), dtype=np.int8)
    qw = rng.integers(-127, 128, (6, 768), dtype=np.int8)
    sx = inputs.to_bf16_bits(rng.uniform(0.01, 0.1, (5, 6)).astype(np.float32))
    su8 = (2 ** rng.integers(0, 8, (6, 3))).astype(np.uint8)        # powers of two: u8 * bf16 is bf16
    s2 = inputs.to_bf16_bits(rng.uniform(1e-4, 1e-3, 6).astype(np.float32))
    sw = inputs.to_bf16_bits((np.repeat(su8.astype(np.float32), 2, axis=1)
                              * inputs.bf16_bits_to_f32(s2)[:, None]).astype(np.float32))
    assert np.array_equal(inputs.bf16_bits_to_f32(sw).astype(np.float64),
                          np.repeat(su8.astype(np.float64), 2, axis=1)
                          * inputs.bf16_bits_to_f32(s2).astype(np.float64)[:, None])
    y, y32 = orc.gemm_trunk(qx, sx, qw, su8, s2)
    yg, yg32 = orc.gemm_g128(qx, sx, qw, sw)
    assert np.array_equal(y32, yg32) and np.array_equal(y, yg)


def test_gemm_trunk_within_quantization_bound(orc):
    xb, wb = inputs.hadamard_linear(8, 4, K=512, N=32)
    qx, sx, xr = orc.fwht128_quant(xb)
    qw, su8, s2 = orc.trunk_weight_quant(wb)
    _, _, wr = orc.fwht128_quant(wb)
    _, y32 = orc.gemm_trunk(qx, sx, qw, su8, s2)
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    w = inputs.bf16_bits_to_f32(wb).astype(np.float64)
    ref = x @ w.T
    sxf = inputs.bf16_bits_to_f32(sx).astype(np.float64)
    swf = np.repeat(su8.astype(np.float64), 2, axis=1) * inputs.bf16_bits_to_f32(s2).astype(np.float64)[:, None]
    bound = np.zeros_like(ref)
    for g in range(4):
        sl = slice(g * 128, (g + 1) * 128)
        bound += (np.abs(xr[:, sl]).astype(np.float64).sum(1)[:, None] * swf[None, :, g] / 2
                  + sxf[:, None, g] * np.abs(wr[:, sl]).astype(np.float64).sum(1)[None, :] / 2
                  + 128 * sxf[:, None, g] * swf[None, :, g] / 4)
    bound = bound / 128 * (1 + 1e-5) + 1e-5 * np.abs(ref) + 1e-9
    assert np.all(np.abs(y32.astype(np.float64) - ref) <= bound)
