"""Pins of the oracle's absmax quantization (a0 / a1 / a9) and bf16 rounding.

Each property follows from the scheme's definition (per-token / per-channel
symmetric int8 with scale absmax/127, round to nearest even, codes clamped
to -127..127: "Qwen3.6-27B-Quark-W8A8-INT8", Quantization Scheme; "Online
INT8 W8A8 ...", Precision split) and is checked without the oracle's own
formulas: exact fp64 bounds, brute-force nearest-code search, symmetry,
power-of-two scaling, hand-built half-way cases and torch's bf16 cast.
"""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs


def _rows(seed, M=64, K=300):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[3, rng.choice(K, 3, replace=False)] *= 50.0          # outliers
    x[5] *= 1e-30                                           # tiny but normal
    x[6] = -np.abs(x[6])                                    # absmax on a negative value
    x[7, :] = 0.0
    x[7, 11] = 1e-3                                         # single nonzero
    return x


def test_round_trip_bound_and_range(orc):
    x = _rows(0)
    q, s = orc.quant_rows_f32(x)
    assert q.min() >= -127 and q.max() <= 127
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s[:, None].astype(np.float64))
    # |x - q s| <= s/2 up to the fp32 rounding of x/s (relative 2^-23 of |x|/s <= 127.x)
    bound = s[:, None].astype(np.float64) * (0.5 + 128 * 2.0 ** -23)
    assert np.all(err <= bound)


def test_absmax_maps_to_127(orc):
    x = _rows(1)
    q, s = orc.quant_rows_f32(x)
    for m in range(x.shape[0]):
        if not np.any(x[m]):
            continue
        j = int(np.argmax(np.abs(x[m])))
        assert int(q[m, j]) == (127 if x[m, j] > 0 else -127)
        # the stored scale is the fp32 quotient absmax/127, correctly rounded
        assert s[m] == np.float32(np.float32(np.abs(x[m, j])) / np.float32(127.0))


def test_zero_and_single_nonzero_rows(orc):
    x = np.zeros((2, 40), np.float32)
    x[1, 13] = -0.75
    q, s = orc.quant_rows_f32(x)
    assert s[0] == 0.0 and not q[0].any()
    assert s[1] == np.float32(0.75) / np.float32(127)
    assert q[1, 13] == -127 and np.count_nonzero(q[1]) == 1


def test_sign_symmetry_and_power_of_two_invariance(orc):
    x = _rows(2)
    q, s = orc.quant_rows_f32(x)
    qn, sn = orc.quant_rows_f32(-x)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    for j in (-7, -1, 3, 20):
        f = np.float32(2.0 ** j)
        qj, sj = orc.quant_rows_f32(x * f)
        assert np.array_equal(qj, q)
        assert np.array_equal(sj, s * f)


def test_brute_force_nearest_code(orc):
    """Every code is the nearest of the 255 levels q*s (ties to the even
    code), found by exhaustive search in exact fp64 arithmetic."""
    rng = np.random.default_rng(3)
    levels = np.arange(-127, 128, dtype=np.float64)
    for trial in range(200):
        K = int(rng.integers(1, 9))
        v = (rng.standard_normal(K) * rng.choice([1e-3, 1.0, 40.0])).astype(np.float32)
        q, s = orc.quant_row_f32(v)
        if s == 0:
            assert not q.any()
            continue
        for k in range(K):
            d = np.abs(np.float64(v[k]) - levels * np.float64(s))
            best = np.flatnonzero(d == d.min())
            if best.size == 2:                                  # exact tie: even code
                best = best[(levels[best] % 2) == 0]
            assert int(levels[best[0]]) == int(q[k]), (v, q, s)


def test_half_way_cases_round_to_even(orc):
    # scale chosen so that absmax/127 = 1/16 exactly: x/s = n + 1/2 exactly
    row = np.array([127, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, 126.5, -0.5, -1.5], np.float32) / 16
    q, s = orc.quant_row_f32(row)
    assert s == np.float32(1 / 16)
    assert q.tolist() == [127, 2, 4, -2, -4, 0, 2, 126, 0, -2]


def test_bf16_rows_match_fp32_rows(orc):
    """The bf16 entry widens exactly, so it equals the fp32 entry on the same values."""
    xb, _ = inputs.dense_linear(4, 8, 512, 16)
    q1, s1 = orc.quant_rows_bf16(xb)
    q2, s2 = orc.quant_rows_f32(inputs.bf16_bits_to_f32(xb))
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_negative_zero_and_clamp_range(orc):
    row = np.array([-0.0, 0.0, -3.0, 3.0], np.float32)
    q, s = orc.quant_row_f32(row)
    assert q.tolist() == [0, 0, -127, 127]
    assert -128 not in orc.quant_rows_f32(np.array([[-1.0, 1.0, -1.0]], np.float32))[0]


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(5)
    f = (rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000)).astype(np.float32)
    # exact ties and carries into the exponent
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x3F80FFFF, 0x7F7FFFFF, 0x00008000,
                     0x00018000, 0x7F7F8000], np.uint32).view(np.float32)
    f = np.concatenate([f, ties])
    ours = orc.f32_to_bf16(f)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(orc.bf16_to_f32(ours), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())
