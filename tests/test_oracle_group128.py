"""Pins of the oracle's group-128 grid without the rotation (the head's
format: "Qwen3.6-35B-A3B IQ8R - radiance container", file table, Head row:
int8 codes with one bf16 scale per row and 128 of K, no rotation; recipe row
output.weight: codes=i8 group=128 scale=bf16 clamp=sym, no transform).

The quantizer is pinned by brute force (each code is the nearest of the 255
codes to x / s, the absmax element maps to +-127, the bf16 scale is within
one bf16 rounding of absmax / 127) and, on inputs whose rotation is exact, to
the separately pinned FWHT128 quantizer; the GEMM by exact integer results
with power-of-two scales and by the quantization bound of the fp64 product.
"""
import numpy as np
import scipy.linalg

from moe_gemm_absmax_b200 import inputs

H128 = scipy.linalg.hadamard(128).astype(np.float64)


def test_group128_quant_brute_force(orc):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((3, 384)) * 10.0 ** rng.uniform(-2, 2, (3, 1))).astype(np.float32)
    x[1, 128:256] *= 40.0
    xb = inputs.to_bf16_bits(x)
    q, s = orc.group128_quant(xb)
    xf = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    sf = inputs.bf16_bits_to_f32(s).astype(np.float64)
    codes = np.arange(-127, 128, dtype=np.float64)
    for m in range(3):
        for g in range(3):
            blk = xf[m, g * 128:(g + 1) * 128]
            c = q[m, g * 128:(g + 1) * 128].astype(np.int64)
            amax = np.abs(blk).max()
            assert abs(sf[m, g] - amax / 127) <= 2.0 ** -8 * amax / 127
            j = int(np.argmax(np.abs(blk)))
            assert abs(c[j]) == 127 and np.sign(c[j]) == np.sign(blk[j])
            err = np.abs(blk[:, None] - codes[None, :] * sf[m, g])
            best = codes[np.argmin(err, axis=1)]
            second = np.sort(err, axis=1)[:, 1]
            clear = second - err.min(axis=1) > 2.0 ** -20 * sf[m, g]   # not within a hair of a tie
            assert np.array_equal(c[clear], best[clear])


def test_group128_quant_zero_block_and_ties(orc):
    xb = np.zeros((2, 256), np.uint16)
    # block 1 of row 1: absmax 127 -> scale exactly 1; halves round to even
    v = np.zeros(128, np.float32)
    v[0], v[1], v[2], v[3], v[4] = 127.0, 2.5, 3.5, -2.5, -0.5
    xb[1, 128:] = inputs.to_bf16_bits(v)
    q, s = orc.group128_quant(xb)
    assert not q[0].any() and not s[0].any() and not q[1, :128].any() and s[1, 0] == 0
    assert inputs.bf16_bits_to_f32(s[1, 1]) == 1.0
    assert list(q[1, 128:133]) == [127, 2, 4, -2, 0]


def test_group128_quant_equals_fwht_quant_when_the_rotation_is_exact(orc):
    """x with two +-1 entries per block: H x has entries in {-2..2}, exact in
    bf16, so quantizing H x on the plain grid gives the rotated quantizer's codes."""
    rng = np.random.default_rng(5)
    x = np.zeros((4, 256), np.float32)
    for m in range(4):
        for g in range(2):
            idx = rng.choice(128, 2, replace=False) + 128 * g
            x[m, idx] = rng.choice([-1.0, 1.0], 2)
    xb = inputs.to_bf16_bits(x)
    hx = (x.reshape(4, 2, 128).astype(np.float64) @ H128.T).reshape(4, 256)
    qr, sr, _ = orc.fwht128_quant(xb)
    qp, sp = orc.group128_quant(inputs.to_bf16_bits(hx.astype(np.float32)))
    assert np.array_equal(qr, qp) and np.array_equal(sr, sp)


def test_gemm_group128_exact_with_power_of_two_scales(orc):
    rng = np.random.default_rng(3)
    qx = rng.integers(-127, 128, (3, 384), dtype=np.int8)
    qw = rng.integers(-127, 128, (5, 384), dtype=np.int8)
    sx = inputs.to_bf16_bits(np.full((3, 3), 2.0 ** -4, np.float32))
    sw = inputs.to_bf16_bits(np.full((5, 3), 2.0 ** -6, np.float32))
    _, y32 = orc.gemm_group128(qx, sx, qw, sw)
    exact = (qx.astype(np.int64) @ qw.astype(np.int64).T) * 2.0 ** -10
    assert np.array_equal(y32.astype(np.float64), exact)
    _, r32 = orc.gemm_g128(qx, sx, qw, sw)
    assert np.array_equal(y32, r32 * 128)   # the rotated form differs by its 1/128 only


def test_gemm_group128_within_quantization_bound(orc):
    xb, wb = inputs.hadamard_linear(7, 4, K=512, N=48)
    qx, sx = orc.group128_quant(xb)
    qw, sw = orc.group128_quant(wb)
    _, y32 = orc.gemm_group128(qx, sx, qw, sw)
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    w = inputs.bf16_bits_to_f32(wb).astype(np.float64)
    ref = x @ w.T
    sxf = inputs.bf16_bits_to_f32(sx).astype(np.float64)
    swf = inputs.bf16_bits_to_f32(sw).astype(np.float64)
    bound = np.zeros_like(ref)
    for g in range(4):
        sl = slice(g * 128, (g + 1) * 128)
        bound += (np.abs(x[:, sl]).sum(1)[:, None] * swf[None, :, g] / 2
                  + sxf[:, None, g] * np.abs(w[:, sl]).sum(1)[None, :] / 2
                  + 128 * sxf[:, None, g] * swf[None, :, g] / 4)
    bound = bound * (1 + 1e-5) + 1e-5 * np.abs(ref) + 1e-9
    assert np.all(np.abs(y32.astype(np.float64) - ref) <= bound)
    assert np.abs(y32.astype(np.float64) - ref).max() > 0
