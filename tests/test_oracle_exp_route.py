"""Pins of the oracle's exponential, SiLU and router (a5, a6).

exp_proj is the project's own fp32 exponential (Cody & Waite reduction,
degree-7 Taylor polynomial); it is pinned to the fp64 ``exp`` of numpy by
an error bound in units in the last place over a dense sweep of fp32 bit
patterns.  The router ("Online INT8 W8A8 ...", Precision split: the router
gate stays bf16; Changes: routing, scatter/combine) is pinned by brute
force over all k-subsets of a small expert set and by invariants.
"""
import itertools

import numpy as np

from moe_gemm_absmax_b200 import inputs


def _ulp_err(y32, ref64):
    ref32 = ref64.astype(np.float32)
    return np.abs(y32.astype(np.float64) - ref64) / np.spacing(np.abs(ref32)).astype(np.float64)


def test_exp_proj_error_bound_sweep(orc):
    hi = np.arange(0, 0x42B00000, 997, dtype=np.uint32)           # [0, 88)
    lo = np.arange(0x80000000, 0xC2AE0000, 997, dtype=np.uint32)  # (-87, -0]
    x = np.concatenate([hi, lo]).view(np.float32)
    x = np.concatenate([x, np.float32([88.0, -87.0, 1.0, -1.0, 0.5, -0.5])])
    y = orc.exp_proj(x)
    err = _ulp_err(y, np.exp(x.astype(np.float64)))
    assert err.max() <= 2.0, float(err.max())


def test_exp_proj_clamps_and_exact_points(orc):
    y = orc.exp_proj(np.float32([0.0, -0.0, 100.0, 88.0, -100.0, -87.0]))
    assert y[0] == 1.0 and y[1] == 1.0
    assert y[2] == y[3] and y[4] == y[5]
    assert np.isfinite(y).all() and (y > 0).all()


def test_silu_against_fp64(orc):
    rng = np.random.default_rng(0)
    g = np.concatenate([rng.standard_normal(100000) * 4, rng.standard_normal(1000) * 60,
                        [0.0, 1e-30, -1e-30, 86.0, -86.0]]).astype(np.float32)
    y = orc.silu(g)
    g64 = g.astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64))
    # exp within 2 ulp, then 1 + e and g / d each round once
    inside = g >= -87.0
    ok = np.abs(y - ref) <= 4 * np.spacing(np.abs(ref.astype(np.float32))) + 1e-44
    assert ok[inside].all()
    # below -87 the clamped exponential makes SiLU(g) = g / e^88-ish: a value
    # within |g| e^-87 of the true (smaller still) one
    assert np.all(np.abs(y[~inside] - ref[~inside]) <= np.abs(g64[~inside]) * np.exp(-87.0))
    assert orc.silu(np.float32([0.0]))[0] == 0.0


def _brute_route(lf, k):
    """All k-subsets; the chosen one has the largest logits, ties broken
    toward lower indices (lexicographic on the sorted key)."""
    E = lf.size
    best = None
    for sub in itertools.combinations(range(E), k):
        key = sorted(((-lf[e], e) for e in sub))
        if best is None or key < best[0]:
            best = (key, sub)
    return [e for _, e in best[0]]


def test_route_brute_force_small(orc):
    rng = np.random.default_rng(1)
    for trial in range(60):
        E, k = 8, int(rng.integers(1, 4))
        logits = rng.standard_normal((1, E)).astype(np.float32)
        if trial % 3 == 0:
            logits = np.round(logits * 2) / 2                  # force ties
        lb = inputs.to_bf16_bits(logits)
        ids, w = orc.route(lb, k)
        lf = inputs.bf16_bits_to_f32(lb)[0].astype(np.float64)
        assert ids[0].tolist() == _brute_route(lf, k)
        p = np.exp(lf - lf.max())
        p /= p.sum()
        ref = p[ids[0]] / p[ids[0]].sum()
        assert np.allclose(w[0], ref, rtol=2e-6, atol=0)


def test_route_invariants_full_size(orc):
    xb, lb, _, _ = inputs.moe_layer(0, 64, with_weights=False)
    ids, w = orc.route(lb, 8)
    lf = inputs.bf16_bits_to_f32(lb)
    for t in range(64):
        assert len(set(ids[t].tolist())) == 8
        sel = lf[t, ids[t]]
        assert np.all(np.diff(sel) <= 0)                      # descending
        assert sel.min() >= np.delete(lf[t], ids[t]).max()    # nothing larger left out
        assert abs(float(w[t].astype(np.float64).sum()) - 1.0) <= 8 * 2.0 ** -24
        assert np.all(w[t] > 0)


def test_route_constant_logits_tie_break(orc):
    lb = inputs.to_bf16_bits(np.zeros((2, 256), np.float32))
    ids, w = orc.route(lb, 8)
    assert ids.tolist() == [list(range(8))] * 2
    assert np.all(w == np.float32(0.125))


def test_histogram(orc):
    rng = np.random.default_rng(2)
    ids = rng.integers(0, 256, (100, 8)).astype(np.int32)
    assert np.array_equal(orc.histogram(ids, 256), np.bincount(ids.reshape(-1), minlength=256))
