"""Pins of the oracle's FWHT128 group quantization (a12) and group-128
scaled GEMM (a13): "Qwen3.6-35B-A3B IQ8R - radiance container", file table
(Trunk row: every 128-wide slice of K turned by the unnormalised Hadamard
matrix; Experts row: one bf16 scale for each row and 128-wide slice on that
rotated grid; Activations row: quantized after the same rotation) and the conversion recipe (transform=fwht128 group=128
scale=bf16 clamp=sym).

The transform is pinned to scipy's Sylvester Hadamard matrix (a library
routine), to H H = 128 I, to exact integer arithmetic, and to the fp64
product within the fp32 error bound; the group quantization to its
round-trip bound and the +-127 absmax code; the GEMM to the unrotated fp64
product within the quantization error bound (H H^T = 128 I makes the 1/128
exact).
"""
import numpy as np
import scipy.linalg

from moe_gemm_absmax_b200 import inputs

H128 = scipy.linalg.hadamard(128).astype(np.float64)


def test_sylvester_matrix_is_self_inverse_up_to_128():
    assert np.array_equal(H128 @ H128, 128 * np.eye(128))


def test_fwht_of_unit_vectors_are_hadamard_columns(orc):
    for i in (0, 1, 5, 64, 127):
        e = np.zeros(128, np.float32)
        e[i] = 1
        assert np.array_equal(orc.fwht128(e), H128[:, i].astype(np.float32))


def test_fwht_exact_on_small_integers_and_involution(orc):
    rng = np.random.default_rng(0)
    for _ in range(20):
        v = rng.integers(-1000, 1000, 128).astype(np.float32)
        r = orc.fwht128(v)
        assert np.array_equal(r.astype(np.float64), H128 @ v.astype(np.float64))
        assert np.array_equal(orc.fwht128(r), 128 * v)


def test_fwht_fp32_error_bound(orc):
    rng = np.random.default_rng(1)
    for _ in range(50):
        v = (rng.standard_normal(128) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        r = orc.fwht128(v).astype(np.float64)
        ref = H128 @ v.astype(np.float64)
        # 7 stages, each a rounded add of partial sums bounded by sum |v|
        assert np.all(np.abs(r - ref) <= 7 * 2.0 ** -24 * np.abs(v).astype(np.float64).sum())


def test_fwht128_quant_properties(orc):
    xb, _ = inputs.hadamard_linear(0, 8)
    q, s, xr = orc.fwht128_quant(xb)
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    M, K = x.shape
    ref = (x.reshape(M, K // 128, 128) @ H128.T).reshape(M, K)
    assert np.all(np.abs(xr - ref) <= 7 * 2.0 ** -24 * np.abs(x).reshape(M, -1, 128).sum(-1).repeat(128, 1))
    sf = inputs.bf16_bits_to_f32(s).astype(np.float64)
    assert q.min() >= -127 and q.max() <= 127
    for m in range(M):
        for g in range(K // 128):
            blk = xr[m, g * 128:(g + 1) * 128].astype(np.float64)
            codes = q[m, g * 128:(g + 1) * 128]
            j = int(np.argmax(np.abs(blk)))
            assert abs(int(codes[j])) == 127 and np.sign(codes[j]) == np.sign(blk[j])
            # bf16 scale = the bf16 rounding of fp32(absmax / 127): within 2^-8 relative
            # (8 significant bits), which keeps absmax / s inside [126.5, 127.5)
            amax = np.abs(blk).max()
            assert abs(sf[m, g] - amax / 127) <= 2.0 ** -8 * amax / 127 * (1 + 1e-6)
            err = np.abs(blk - codes * sf[m, g])
            assert np.all(err <= sf[m, g] * (0.5 + 128 * 2.0 ** -23))


def test_fwht128_quant_zero_block(orc):
    xb = np.zeros((2, 256), np.uint16)
    xb[1, 128:] = inputs.to_bf16_bits(np.linspace(-1, 1, 128).astype(np.float32))
    q, s, _ = orc.fwht128_quant(xb)
    assert not q[0].any() and not s[0].any() and not q[1, :128].any() and s[1, 0] == 0
    assert s[1, 1] != 0


def test_gemm_g128_within_quantization_bound(orc):
    xb, wb = inputs.hadamard_linear(2, 4, K=512, N=64)
    qx, sx, xr = orc.fwht128_quant(xb)
    qw, sw, wr = orc.fwht128_quant(wb)
    y, y32 = orc.gemm_g128(qx, sx, qw, sw)
    x = inputs.bf16_bits_to_f32(xb).astype(np.float64)
    w = inputs.bf16_bits_to_f32(wb).astype(np.float64)
    ref = x @ w.T
    sxf = inputs.bf16_bits_to_f32(sx).astype(np.float64)
    swf = inputs.bf16_bits_to_f32(sw).astype(np.float64)
    G = 512 // 128
    bound = np.zeros_like(ref)
    for g in range(G):
        sl = slice(g * 128, (g + 1) * 128)
        bound += (np.abs(xr[:, sl]).astype(np.float64).sum(1)[:, None] * swf[None, :, g] / 2
                  + sxf[:, None, g] * np.abs(wr[:, sl]).astype(np.float64).sum(1)[None, :] / 2
                  + 128 * sxf[:, None, g] * swf[None, :, g] / 4)
    bound = bound / 128 * (1 + 1e-5) + 1e-5 * np.abs(ref) + 1e-9
    assert np.all(np.abs(y32.astype(np.float64) - ref) <= bound)


def test_gemm_g128_exact_with_power_of_two_scales(orc):
    """With scales that are powers of two every fp32 step is exact, so
    y = (1/128) sum_g p_g sx sw equals the integer result."""
    rng = np.random.default_rng(3)
    qx = rng.integers(-127, 128, (3, 384), dtype=np.int8)
    qw = rng.integers(-127, 128, (5, 384), dtype=np.int8)
    sx = inputs.to_bf16_bits(np.full((3, 3), 2.0 ** -4, np.float32))
    sw = inputs.to_bf16_bits(np.full((5, 3), 2.0 ** -6, np.float32))
    y, y32 = orc.gemm_g128(qx, sx, qw, sw)
    exact = (qx.astype(np.int64) @ qw.astype(np.int64).T) * 2.0 ** -10 / 128
    assert np.array_equal(y32.astype(np.float64), exact)
